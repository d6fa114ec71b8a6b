// Block-sparse attention forward for 128-token tiles on tcgen05 (bf16 in, fp32 accumulate),
// head_dim 128. Eq. 12 of "Improving Video Sparse Attention with Fine-grained Router and Sparse
// Rebasing" with the attention definition of its §2.1, for the tile of 128 tokens (4x4x8) and
// 8-token router sub-cubes that the deep-read blog infers for VSA2 (its section 07).
//
// A 128-token query tile fills the M side of a full-rate MMA, and one selected 128-token KV tile
// its N side, so every MMA here is M=128, N=128 with all of its output used:
//   S [128 q, 128 kv] = Q . K_j^T    A = Q (TMEM, written once per query tile), B = K_j (K-major)
//   O [128 q, 128 d] += P . V_j       A = P (TMEM, written by the softmax over S), B = V_j (MN-major)
// against M=64 MMAs at half that rate when the same selection is run on 64-token tiles, and half
// the K/V bytes gathered per FLOP.
//
// CTA (persistent, one query tile at a time): warps 0-7 run the softmax; warp w reads TMEM lane
// quarter w%4 (32 query rows) and key half w/4 (64 columns) of S. The two warps of a row quarter
// combine their row maxima through shared memory once per block; the running max is raised (with
// an O rescale in TMEM, each warp its half of the channels) only when a row's block maximum
// exceeds it by more than 2^8. Each warp writes P over the S columns it read itself. Warp 8 loads
// the K tiles (and draws query tiles from a global counter), warp 10 the V tiles, each into its
// own ring; warp 9 issues the MMAs in the order S0, S1, O0, S2, O1, ...
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int FT = 352;            // 11 warps
constexpr uint32_t TILE_B = 8192;  // one 64x64 bf16 box (64 rows x 128 B)
constexpr uint32_t BLK_B = 32768;  // a 128-token K or V tile: [d half][128 rows x 128 B]
constexpr int KST = 3, VST = 3;    // ring stages
constexpr int IDXCAP = 256;        // KV indices of a row kept in shared memory (per producer)
constexpr int QD = 4;              // item queue entries

constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + KST * BLK_B;
constexpr uint32_t OFF_IDX = OFF_V + VST * BLK_B;        // [producer][2 rows][IDXCAP] int32
constexpr uint32_t OFF_RMAX = OFF_IDX + 2 * 2 * IDXCAP * 4;  // [block parity][key half][128 rows] fp32
constexpr uint32_t OFF_RSUM = OFF_RMAX + 2 * 2 * 128 * 4;    // [key half][128 rows] fp32
constexpr uint32_t OFF_BAR = OFF_RSUM + 2 * 128 * 4;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr uint32_t OFF_IQ = OFF_FLAG + 64;  // [QD] items, then [2] hand-over
constexpr uint32_t SMEM_USED = OFF_IQ + (QD + 2) * 4;
constexpr uint32_t SMEM_DYN = SMEM_USED + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");

// TMEM columns (all 128 lanes). P(n) is written in bf16 over the S buffer it was read from: key
// half h at columns 64h .. 64h + 31, so each warp overwrites only columns it has read itself.
// S(n + 2) overwrites the buffer only after O(n) has read P(n): the MMA issuer issues S(n + 2)
// after O(n), and the tensor pipe runs one thread's MMAs in order.
constexpr uint32_t TM_S = 0;    // two S / P buffers of 128 fp32 columns
constexpr uint32_t TM_Q = 256;  // Q: 128 bf16 = 64 columns
constexpr uint32_t TM_O = 320;  // O: 128 fp32 columns
constexpr uint32_t TM_COLS = 512;
constexpr float kThresh = 8.0f;  // log2 headroom before the running max must move

struct Bars {
  uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  uint64_t sfull[2], pfull[2], pvdone[2];  // [block parity]
  uint64_t qready, done;
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
    attn_fwd_b128_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __nv_bfloat16* __restrict__ qg, const int32_t* __restrict__ kv_off,
                         const int32_t* __restrict__ kv_idx, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                         int N, int L, int topk, int items, float c2, int* __restrict__ work_ctr, DevCtx ctx) {
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
    for (int b = 0; b < 2; ++b) mbar_init(&B.sfull[b], 1), mbar_init(&B.pfull[b], 8), mbar_init(&B.pvdone[b], 1);
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
    // Warp 8: the K tiles, in the query tile's list order; it also draws the query tiles from the
    // global counter (two items ahead of its loads) and passes them on through the queue. Warp 10:
    // the V tiles, taking the items from the queue one ahead. Each copies the index row of the
    // next item into its own shared-memory rows (cp.async) while it loads the current one.
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
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, 128, false, true);
      int kq = 0, tile = 0;  // queue entries taken, non-empty query tiles started
      int nblk = 0, s_next = 0, o_next = 0;
      int kc = 0, vc = 0;  // S and O ops issued (also the ring positions and block parities)
      bool ok = true, active = true;
      while (ok && active) {
        int op = 0, blk = 0;
        if (s_next < nblk && s_next <= o_next + 1) {
          op = 1;
          blk = s_next++;
        } else if (o_next < nblk) {
          op = 2;
          blk = o_next++;
        } else {
          const int e = kq % QD;
          int it = -1;
          if (mbar_wait(&B.iqfull[e], (kq / QD) & 1, abort, ctx)) it = iq[e];
          mbar_arrive(&B.iqempty[e]);
          ++kq;
          if (it < 0) {
            active = false;
          } else {
            nblk = row_of(it).len;
            s_next = o_next = 0;
            if (nblk > 0) ++tile;
          }
          continue;
        }
        if (op == 1) {
          if (blk == 0 && !(ok = mbar_wait(&B.qready, (tile - 1) & 1, abort, ctx))) break;
          const int st = kc % KST;
          if (!(ok = mbar_wait(&B.kfull[st], (kc / KST) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(dsm + OFF_K + st * BLK_B);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + TM_S + (kc & 1) * 128, tmem + TM_Q + 8 * kk,
                        sdesc_sw128(ka + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
          mma_commit(&B.kempty[st]);
          mma_commit(&B.sfull[kc & 1]);
          ++kc;
        } else {
          const int st = vc % VST;
          if (!(ok = mbar_wait(&B.vfull[st], (vc / VST) & 1, abort, ctx))) break;
          if (!(ok = mbar_wait(&B.pfull[vc & 1], (vc >> 1) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t va = smem_u32(dsm + OFF_V + st * BLK_B);
          const uint32_t pa = tmem + TM_S + (vc & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // keys 16kk..: P columns 64(kk/4) + 8(kk%4)
            mma_bf16_ts(tmem + TM_O, pa + 64 * (kk >> 2) + 8 * (kk & 3), sdesc_sw128(va + kk * 2048, 2 * TILE_B, 1024),
                        id_o, (blk > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.vempty[st]);
          mma_commit(&B.pvdone[vc & 1]);
          ++vc;
        }
      }
      mma_commit(&B.done);
      mbar_wait_drain(&B.done, 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax, warps 0-7
    const int qd = warp & 3, ch = warp >> 2;  // row quarter, key half (and channel half of Q, O)
    const int row = 32 * qd + lane;           // query row of the tile = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const int pair_bar = 1 + qd;  // the two warps of this row quarter
    const int all_bar = 5;        // all 256 softmax threads
    float* rmax = reinterpret_cast<float*>(dsm + OFF_RMAX);  // [block parity][key half][row]
    float* rsum = reinterpret_cast<float*>(dsm + OFF_RSUM);  // [key half][row]
    volatile int* cur_item = iq + QD;                        // [kq parity]
    int g = 0;                                               // blocks processed
    for (int kq = 0;; ++kq) {
      // warp 0 takes the next queue entry and hands it to the other seven; the hand-over word
      // alternates with the entry's parity, so it is rewritten only after every warp passed the
      // next barrier
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
      if (rw.len == 0) {  // empty selection: o = 0, lse = -inf (each warp its channel half)
        uint4* o4 = reinterpret_cast<uint4*>(out + tok * 128 + 64 * ch);
#pragma unroll
        for (int e = 0; e < 8; ++e) o4[e] = make_uint4(0, 0, 0, 0);
        if (ch == 0) lse[tok] = -INFINITY;
        continue;
      }
      {
        // this row's channel half of Q into TMEM (A operand of S; the S MMAs of the previous
        // tile are done, the softmax has read all of their outputs)
        uint32_t qv[32];
        const uint4* src = reinterpret_cast<const uint4*>(qg + tok * 128 + 64 * ch);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 v = __ldg(src + e);
          qv[4 * e] = v.x, qv[4 * e + 1] = v.y, qv[4 * e + 2] = v.z, qv[4 * e + 3] = v.w;
        }
        tmem_st32(tl + TM_Q + 32 * ch, qv);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.qready);
      }
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < rw.len; ++n, ++g) {
        const int b = g & 1;
        const uint32_t ts = tl + TM_S + 128 * b + 64 * ch;
        mbar_wait(&B.sfull[b], (g >> 1) & 1, abort, ctx);
        tc_fence_after();
        uint32_t xa[32], xb[32];  // S[row][64ch + i], S[row][64ch + 32 + i]
        tmem_ld32(ts, xa);
        tmem_ld32(ts + 32, xb);
        tmem_ld_wait();
        float mx = __uint_as_float(xa[0]);
#pragma unroll
        for (int i = 1; i < 31; i += 2) mx = fmax3(mx, __uint_as_float(xa[i]), __uint_as_float(xa[i + 1]));
        mx = fmax3(mx, __uint_as_float(xa[31]), __uint_as_float(xb[0]));
#pragma unroll
        for (int i = 1; i < 31; i += 2) mx = fmax3(mx, __uint_as_float(xb[i]), __uint_as_float(xb[i + 1]));
        mx = fmaxf(mx, __uint_as_float(xb[31])) * c2;
        // the other key half of this row
        rmax[(2 * b + ch) * 128 + row] = mx;
        named_bar_sync(pair_bar, 64);
        mx = fmaxf(mx, rmax[(2 * b + (ch ^ 1)) * 128 + row]);
        float alpha = 1.f;
        const bool raise = mx > m + kThresh;
        if (raise) {
          alpha = (m == -INFINITY) ? 0.f : ex2(m - mx);
          m = mx;
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, raise && n > 0)) {
          // O holds blocks 0..n-1 of this tile: scale this warp's channel half of the raised rows
          // once the last O MMA is done
          mbar_wait(&B.pvdone[(g - 1) & 1], ((g - 1) >> 1) & 1, abort, ctx);
          tc_fence_after();
          uint32_t oa[32], ob[32];
          tmem_ld32(tl + TM_O + 64 * ch, oa);
          tmem_ld32(tl + TM_O + 64 * ch + 32, ob);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            oa[i] = __float_as_uint(__uint_as_float(oa[i]) * alpha);
            ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
          }
          tmem_st32(tl + TM_O + 64 * ch, oa);
          tmem_st32(tl + TM_O + 64 * ch + 32, ob);
          tmem_st_wait();
        }
        // probabilities (<= 2^8), partial row sum, bf16 pairs of adjacent keys (packed fp32 math)
        uint32_t pk[32];
        const float2 cc = make_float2(c2, c2), nm = make_float2(-m, -m);
        float2 ls = make_float2(0.f, 0.f);
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const uint32_t* x = i2 < 16 ? xa : xb;
          const int k2 = 2 * (i2 & 15);
          const float2 arg = __ffma2_rn(make_float2(__uint_as_float(x[k2]), __uint_as_float(x[k2 + 1])), cc, nm);
          const float pa = ex2(arg.x), pb = ex2(arg.y);
          ls = __fadd2_rn(ls, make_float2(pa, pb));
          pk[i2] = pack_bf16(pa, pb);
        }
        l += ls.x + ls.y;
        // P over the first 32 of this warp's 64 S columns (their S values are in registers)
        tmem_st32(ts, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.pfull[b]);
      }
      // ---- epilogue: last O block done -> row sum over both key halves, normalise, store
      mbar_wait(&B.pvdone[(g - 1) & 1], ((g - 1) >> 1) & 1, abort, ctx);
      tc_fence_after();
      rsum[ch * 128 + row] = l;
      named_bar_sync(pair_bar, 64);
      const float lt = l + rsum[(ch ^ 1) * 128 + row];
      const float inv = 1.f / lt;
      if (ch == 0) lse[tok] = (m + __log2f(lt)) * 0.6931471805599453f;
      uint32_t oa[32], ob[32];
      tmem_ld32(tl + TM_O + 64 * ch, oa);
      tmem_ld32(tl + TM_O + 64 * ch + 32, ob);
      tmem_ld_wait();
      uint4* o4 = reinterpret_cast<uint4*>(out + tok * 128 + 64 * ch);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t* o = e < 4 ? oa : ob;
        const int k = 8 * (e & 3);
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          w[u] = pack_bf16(__uint_as_float(o[k + 2 * u]) * inv, __uint_as_float(o[k + 2 * u + 1]) * inv);
        o4[e] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      tc_fence_before();
      // leave together if any wait of this CTA has expired
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

// 128-token tiles (d.Bt = 128), bf16, D = 128, grids the tile divides: kv_off / kv_idx are the
// 128-token selection itself.
vsa2_status attn_fwd_b128_tc(const Dims& d, const void* q, const void* k, const void* v, int topk,
                             const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                             cudaStream_t s) {
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tk, k, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tv, v, 128, rows, 64, 64))
    return tmap_fail("tensor map encoding for the attention operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(sms, items));
  const float c2 = 1.4426950408889634f / sqrtf(128.f);
  cudaFuncSetAttribute(attn_fwd_b128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  int* ctr = reinterpret_cast<int*>(ws + kWsWorkCounter);  // the item counter, in the workspace header
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_fwd_b128: item counter reset");
  attn_fwd_b128_kernel<<<grid, FT, SMEM_DYN, s>>>(tk, tv, (const __nv_bfloat16*)q, kv_off, kv_idx, (__nv_bfloat16*)o,
                                                  lse, d.N, (int)d.L, topk, items, c2, ctr, ctx);
  return check_launch("attn_fwd_b128");
}

}  // namespace vsa2
