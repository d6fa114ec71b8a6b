// dQ of the block-sparse attention backward for 128-token tiles on tcgen05 (bf16 in, fp32 out),
// head_dim 128: the gradient of Eq. 12 of "Improving Video Sparse Attention with Fine-grained
// Router and Sparse Rebasing" with respect to Q, with P = exp(S / sqrt(D) - lse) recomputed from
// the forward's LSE and Delta = rowsum(dO * O) (the router gets no gradient, its §2.1), for the
// tile of 128 tokens (4x4x8) that the deep-read blog infers for VSA2 (its section 07).
//
// A 128-token query tile fills the M side of a full-rate MMA and one selected 128-token KV tile
// its N side, so all three GEMMs are M=128, N=128 with all of their output used:
//   S  [128 q, 128 kv] = Q . K_j^T     A = Q  (TMEM), B = K_j (K-major)
//   dP [128 q, 128 kv] = dO . V_j^T    A = dO (TMEM), B = V_j (K-major)
//   dQ [128 q, 128 d] += dS . K_j      A = dS (TMEM, written by the softmax over S), B = K_j (MN-major)
// It also writes -Delta and -lse * log2(e) per token for the dK/dV kernel.
//
// CTA (persistent, one query tile at a time): warps 0-7 form dS = P * (dP - Delta); warp w reads
// TMEM lane quarter w%4 (32 query rows) and key half w/4, and writes its dS in bf16 over the S
// columns it read itself. Warp 8 loads the K tiles (held until the dQ MMAs have read them) and
// draws query tiles from a global counter, warp 10 the V tiles; warp 9 issues the MMAs in the
// order S/dP(0), dQ(0), S/dP(1), dQ(1), ...: S and dP have one buffer each, reused once dQ(n)
// has read dS(n).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int FT = 352;            // 11 warps
constexpr uint32_t TILE_B = 8192;  // one 64x64 bf16 box (64 rows x 128 B)
constexpr uint32_t BLK_B = 32768;  // a 128-token K or V tile: [d half][128 rows x 128 B]
constexpr int KST = 3, VST = 2;    // ring stages
constexpr int IDXCAP = 256;        // KV indices of a row kept in shared memory (per producer)
constexpr int QD = 4;              // item queue entries
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + KST * BLK_B;
constexpr uint32_t OFF_IDX = OFF_V + VST * BLK_B;            // [producer][2 rows][IDXCAP] int32
constexpr uint32_t OFF_RED = OFF_IDX + 2 * 2 * IDXCAP * 4;   // [channel half][128 rows] fp32
constexpr uint32_t OFF_BAR = OFF_RED + 2 * 128 * 4;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr uint32_t OFF_IQ = OFF_FLAG + 64;  // [QD] items, then [2] hand-over
constexpr uint32_t SMEM_USED = OFF_IQ + (QD + 2) * 4;
constexpr uint32_t SMEM_DYN = SMEM_USED + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");

// TMEM columns (all 128 lanes). dS(n) is written in bf16 over the S buffer: key half h at
// columns 64h .. 64h + 31, so each warp overwrites only columns it has read itself.
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_Q = 256, TM_DO = 320, TM_DQ = 384;
constexpr uint32_t TM_COLS = 512;

struct Bars {
  uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  uint64_t sfull, dsfull, bdone, qready, done;
  uint64_t iqfull[QD], iqempty[QD];
};
static_assert(sizeof(Bars) <= 512, "barrier area");

struct Row {
  int beg, len;
};
// Sanitised CSR row of query tile i of head bh; every role reads it the same way.
__device__ __forceinline__ Row load_row(const int32_t* kv_off, int bh, int i, int N, int cap, const DevCtx& ctx,
                                        bool report) {
  int b = kv_off[(size_t)bh * (N + 1) + i];
  int e = kv_off[(size_t)bh * (N + 1) + i + 1];
  if (b < 0 || e < b || e > cap || e - b > N) {
    if (report) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return Row{0, 0};
  }
  return Row{b, e - b};
}

__global__ void __launch_bounds__(FT, 1)
    attn_bwd_dq_b128_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const __nv_bfloat16* __restrict__ qg, const __nv_bfloat16* __restrict__ og,
                            const __nv_bfloat16* __restrict__ dog, const float* __restrict__ lse,
                            float* __restrict__ ndelta, float* __restrict__ nlse2, const int32_t* __restrict__ kv_off,
                            const int32_t* __restrict__ kv_idx, float* __restrict__ dq_out, int N, int L, int topk,
                            int items, float c2, float scale, int* __restrict__ work_ctr, DevCtx ctx) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);  // [0] abort, [4] tmem base
  volatile int* abort = flag_sh;
  volatile int* iq = reinterpret_cast<volatile int*>(dsm + OFF_IQ);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int i = 0; i < KST; ++i) mbar_init(&B.kfull[i], 1), mbar_init(&B.kempty[i], 1);
    for (int i = 0; i < VST; ++i) mbar_init(&B.vfull[i], 1), mbar_init(&B.vempty[i], 1);
    mbar_init(&B.sfull, 1);
    mbar_init(&B.dsfull, 8);
    mbar_init(&B.bdone, 1);
    mbar_init(&B.qready, 8);
    mbar_init(&B.done, 1);
    for (int i = 0; i < QD; ++i) mbar_init(&B.iqfull[i], 1), mbar_init(&B.iqempty[i], 3);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(reinterpret_cast<uint32_t*>(flag_sh + 4), TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(flag_sh + 4);

  auto row_of = [&](int it) { return it >= 0 ? load_row(kv_off, it / N, it % N, N, cap, ctx, false) : Row{0, 0}; };

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------------ TMA producers
    // Warp 8: the K tiles, in the query tile's list order (each held until the dQ MMAs have read
    // it); it also draws the query tiles from the global counter (two items ahead of its loads)
    // and passes them on through the queue. Warp 10: the V tiles, taking the items from the queue
    // one ahead. Each copies the index row of the next item into its own shared-memory rows
    // (cp.async) while it loads the current one.
    const bool kprod = warp == 8;
    int32_t* ibuf = reinterpret_cast<int32_t*>(dsm + OFF_IDX) + (kprod ? 0 : 2 * IDXCAP);
    const CUtensorMap* tm = kprod ? &tm_k : &tm_v;
    if (lane == 0) tma_prefetch_desc(tm);
    auto copy_row = [&](int it, const Row& r, int b) {  // whole warp
      const int32_t* src = kv_idx + (size_t)(it / N) * cap + r.beg;
      const int n = min(r.len, IDXCAP);
      for (int e = lane; e < n; e += 32)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(ibuf + b * IDXCAP + e)), "l"(src + e)
                     : "memory");
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int kq = 0;  // queue entries written (warp 8) or taken (warp 10)
    bool ended = false, ok = true;
    auto next_id = [&]() -> int {  // whole warp
      if (ended) return -1;
      int id = -1, good = 1;
      if (lane == 0) {
        const int e = kq % QD;
        if (kprod) {
          id = atomicAdd(work_ctr, 1);
          if (id >= items) id = -1;
          if (mbar_wait(&B.iqempty[e], ((kq / QD) & 1) ^ 1, abort, ctx)) {
            iq[e] = id;
            mbar_arrive(&B.iqfull[e]);
          } else {
            good = 0;
          }
        } else {
          if (mbar_wait(&B.iqfull[e], (kq / QD) & 1, abort, ctx))
            id = iq[e];
          else
            good = 0;
          mbar_arrive(&B.iqempty[e]);
        }
      }
      id = __shfl_sync(0xffffffffu, id, 0);
      good = __shfl_sync(0xffffffffu, good, 0);
      ++kq;
      if (!good) ok = false;
      if (id < 0 || !good) {
        ended = true;
        id = -1;
      }
      return id;
    };
    int item = next_id();
    Row cur = row_of(item);
    if (item >= 0) copy_row(item, cur, 0);
    int nxt_id = next_id();
    Row nxt = row_of(nxt_id);
    int c = 0;  // ring position: tiles requested so far
    uint64_t* full = kprod ? B.kfull : B.vfull;
    uint64_t* empty = kprod ? B.kempty : B.vempty;
    const int nst = kprod ? KST : VST;
    uint8_t* ring = dsm + (kprod ? OFF_K : OFF_V);
    for (int b = 0; ok && item >= 0; b ^= 1) {
      asm volatile("cp.async.wait_all;" ::: "memory");  // this item's indices (copied an item ago)
      __syncwarp();
      if (nxt_id >= 0 && nxt.len > 0) copy_row(nxt_id, nxt, b ^ 1);
      const int nn_id = kprod ? next_id() : -1;  // warp 10 takes items one ahead only
      const Row nn = row_of(nn_id);
      if (lane == 0 && cur.len > 0) {
        const int bh = item / N;
        const int32_t* gidx = kv_idx + (size_t)bh * cap + cur.beg;
        const int32_t* sidx = ibuf + b * IDXCAP;
        for (int e = 0; ok && e < cur.len; ++e) {
          int j = e < IDXCAP ? sidx[e] : gidx[e];
          if (j < 0 || j >= N) {
            if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
            j = min(max(j, 0), N - 1);
          }
          const int st = c % nst;
          if (!(ok = mbar_wait(&empty[st], ((c / nst) & 1) ^ 1, abort, ctx))) break;
          mbar_arrive_expect_tx(&full[st], BLK_B);
          uint8_t* dst = ring + st * BLK_B;
          for (int h = 0; h < 2; ++h)
            for (int r = 0; r < 2; ++r)
              tma_load_2d(dst + h * 2 * TILE_B + r * TILE_B, tm, h * 64, bh * L + j * 128 + r * 64, &full[st]);
          ++c;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
      item = nxt_id;
      cur = nxt;
      if (kprod) {
        nxt_id = nn_id;
        nxt = nn;
      } else if (item >= 0) {
        nxt_id = next_id();
        nxt = row_of(nxt_id);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
    if (lane == 0 && *abort) {  // let copies still in flight land before the CTA exits
      for (int cc = max(0, c - nst); cc < c; ++cc) mbar_wait_drain(&full[cc % nst], (cc / nst) & 1, ctx.timeout_ns);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kmaj = idesc_bf16_f32(128, 128, false, false);  // S, dP: N = 128 keys
      constexpr uint32_t id_mn = idesc_bf16_f32(128, 128, false, true);     // dQ: N = 128 channels
      int kq = 0, tile = 0;  // queue entries taken, non-empty query tiles started
      int nblk = 0, blk = 0;
      int c = 0;  // blocks issued (ring positions, barrier phases)
      bool ok = true, active = true;
      while (ok && active) {
        if (blk >= nblk) {
          const int e = kq % QD;
          int it = -1;
          if (mbar_wait(&B.iqfull[e], (kq / QD) & 1, abort, ctx)) it = iq[e];
          mbar_arrive(&B.iqempty[e]);
          ++kq;
          if (it < 0) {
            active = false;
          } else {
            nblk = row_of(it).len;
            blk = 0;
            if (nblk > 0) ++tile;
          }
          continue;
        }
        // S and dP of block c; their buffers are free once dQ(c - 1) has read dS(c - 1)
        if (blk == 0 && !(ok = mbar_wait(&B.qready, (tile - 1) & 1, abort, ctx))) break;
        if (c > 0 && !(ok = mbar_wait(&B.bdone, (c - 1) & 1, abort, ctx))) break;
        const int ks = c % KST, vs = c % VST;
        if (!(ok = mbar_wait(&B.kfull[ks], (c / KST) & 1, abort, ctx))) break;
        if (!(ok = mbar_wait(&B.vfull[vs], (c / VST) & 1, abort, ctx))) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(dsm + OFF_K + ks * BLK_B);
        const uint32_t va = smem_u32(dsm + OFF_V + vs * BLK_B);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + TM_S, tmem + TM_Q + 8 * kk, sdesc_sw128(ka + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024),
                      id_kmaj, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + TM_DP, tmem + TM_DO + 8 * kk,
                      sdesc_sw128(va + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_kmaj, kk > 0);
        mma_commit(&B.vempty[vs]);
        mma_commit(&B.sfull);
        // dQ += dS K_j: dS over S in bf16 (keys 16kk..: columns 64(kk/4) + 8(kk%4)), K_j read
        // MN-major from the same stage
        if (!(ok = mbar_wait(&B.dsfull, c & 1, abort, ctx))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + TM_DQ, tmem + TM_S + 64 * (kk >> 2) + 8 * (kk & 3),
                      sdesc_sw128(ka + kk * 2048, 2 * TILE_B, 1024), id_mn, (blk > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&B.kempty[ks]);
        mma_commit(&B.bdone);
        ++c;
        ++blk;
      }
      mma_commit(&B.done);
      mbar_wait_drain(&B.done, 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ dS, warps 0-7
    const int qd = warp & 3, ch = warp >> 2;  // row quarter, key half (and channel half of Q, dO, dQ)
    const int row = 32 * qd + lane;           // query row of the tile = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const int pair_bar = 1 + qd;  // the two warps of this row quarter
    const int all_bar = 5;        // all 256 softmax threads
    float* red = reinterpret_cast<float*>(dsm + OFF_RED);  // [channel half][row]
    volatile int* cur_item = iq + QD;                      // [kq parity]
    const float2 cc = make_float2(c2, c2);
    int g = 0;  // blocks processed
    for (int kq = 0;; ++kq) {
      // warp 0 takes the next queue entry and hands it to the other seven
      if (warp == 0 && lane == 0) {
        const int e = kq % QD;
        int id = -1;
        if (mbar_wait(&B.iqfull[e], (kq / QD) & 1, abort, ctx)) id = iq[e];
        mbar_arrive(&B.iqempty[e]);
        cur_item[kq & 1] = id;
      }
      named_bar_sync(all_bar, 256);
      const int item = cur_item[kq & 1];
      if (item < 0) break;
      const int bh = item / N, qt = item - bh * N;
      const Row rw = load_row(kv_off, bh, qt, N, cap, ctx, warp == 0 && lane == 0);
      const size_t tok = (size_t)bh * L + (size_t)qt * 128 + row;
      float4* dst = reinterpret_cast<float4*>(dq_out + tok * 128 + 64 * ch);
      // this row's channel half of Q and dO into TMEM; Delta = rowsum(dO * O) over both halves
      float part = 0.f;
      {
        uint32_t qv[32], dv[32];
        const uint4* qs = reinterpret_cast<const uint4*>(qg + tok * 128 + 64 * ch);
        const uint4* ds = reinterpret_cast<const uint4*>(dog + tok * 128 + 64 * ch);
        const uint4* os = reinterpret_cast<const uint4*>(og + tok * 128 + 64 * ch);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 a = __ldg(qs + e), d = __ldg(ds + e), o = __ldg(os + e);
          const uint32_t dw[4] = {d.x, d.y, d.z, d.w}, ow[4] = {o.x, o.y, o.z, o.w};
          qv[4 * e] = a.x, qv[4 * e + 1] = a.y, qv[4 * e + 2] = a.z, qv[4 * e + 3] = a.w;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            dv[4 * e + u] = dw[u];
            part = fmaf(__uint_as_float(dw[u] << 16), __uint_as_float(ow[u] << 16), part);
            part = fmaf(__uint_as_float(dw[u] & 0xffff0000u), __uint_as_float(ow[u] & 0xffff0000u), part);
          }
        }
        if (rw.len > 0) {
          tmem_st32(tl + TM_Q + 32 * ch, qv);
          tmem_st32(tl + TM_DO + 32 * ch, dv);
          tmem_st_wait();
        }
      }
      red[ch * 128 + row] = part;
      named_bar_sync(pair_bar, 64);
      const float dlt = part + red[(ch ^ 1) * 128 + row];  // rewritten only after the next all_bar
      const float lse_t = lse[tok];
      const float nl2 = lse_t == -INFINITY ? -INFINITY : -lse_t * kLog2e;
      if (ch == 0) {  // for the dK/dV kernel
        ndelta[tok] = -dlt;
        nlse2[tok] = nl2;
      }
      if (rw.len == 0) {
#pragma unroll
        for (int e = 0; e < 16; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.qready);
      const float2 ll = make_float2(nl2, nl2), nd = make_float2(-dlt, -dlt);
      for (int n = 0; n < rw.len; ++n, ++g) {
        mbar_wait(&B.sfull, g & 1, abort, ctx);
        tc_fence_after();
        uint32_t pk[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // 32 keys at a time
          uint32_t sv[32], dp[32];
          tmem_ld32(tl + TM_S + 64 * ch + 32 * hh, sv);
          tmem_ld32(tl + TM_DP + 64 * ch + 32 * hh, dp);
          tmem_ld_wait();
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            const float2 arg =
                __ffma2_rn(make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1])), cc, ll);
            const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
            const float2 d2 = __fmul2_rn(
                p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * i2]), __uint_as_float(dp[2 * i2 + 1])), nd));
            pk[16 * hh + i2] = pack_bf16(d2.x, d2.y);
          }
        }
        tmem_st32(tl + TM_S + 64 * ch, pk);  // dS over the first 32 of this warp's S columns
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.dsfull);
      }
      // epilogue: the last dQ block is done -> scale by 1/sqrt(D), store this channel half (fp32)
      mbar_wait(&B.bdone, (g - 1) & 1, abort, ctx);
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[32];
        tmem_ld32(tl + TM_DQ + 64 * ch + 32 * hh, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[8 * hh + e] = make_float4(__uint_as_float(o[4 * e]) * scale, __uint_as_float(o[4 * e + 1]) * scale,
                                        __uint_as_float(o[4 * e + 2]) * scale, __uint_as_float(o[4 * e + 3]) * scale);
      }
      tc_fence_before();
      if (named_bar_or(all_bar, 256, *abort != 0)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                       uint32_t box_rows);

// 128-token tiles (d.Bt = 128), bf16, D = 128, grids the tile divides: dQ from the 128-token CSR,
// plus -Delta and -lse * log2(e) per token into `ndelta` and `nlse2` for the dK/dV kernel.
vsa2_status attn_bwd_dq_b128_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, const int32_t* kv_off, const int32_t* kv_idx,
                                float* dq, float* ndelta, float* nlse2, int topk, char* ws, cudaStream_t s) {
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tk, k, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tv, v, 128, rows, 64, 64))
    return tmap_fail("tensor map encoding for the backward operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(sms, items));
  const float c1 = 1.f / sqrtf(128.f);
  cudaFuncSetAttribute(attn_bwd_dq_b128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  int* ctr = reinterpret_cast<int*>(ws + kWsWorkCounter);  // the item counter, in the workspace header
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_bwd_dq_b128: item counter reset");
  attn_bwd_dq_b128_kernel<<<grid, FT, SMEM_DYN, s>>>(tk, tv, (const __nv_bfloat16*)q, (const __nv_bfloat16*)o,
                                                     (const __nv_bfloat16*)dout, lse, ndelta, nlse2, kv_off, kv_idx, dq,
                                                     d.N, (int)d.L, topk, items, kLog2e * c1, c1, ctr, ctx);
  return check_launch("attn_bwd_dq_b128");
}

}  // namespace vsa2
