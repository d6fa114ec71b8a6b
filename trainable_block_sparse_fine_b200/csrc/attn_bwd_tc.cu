// Block-sparse attention backward on tcgen05 (bf16 in, fp32 accumulate), head_dim 128.
// Gradients of Eq. 12 of "Improving Video Sparse Attention with Fine-grained Router and Sparse
// Rebasing" (the router itself receives none, §2.1). With P = exp(S/sqrt(D) - lse) recomputed
// from the forward's LSE and Delta = rowsum(dO * O):
//   dS = P * (dO V^T - Delta),  dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D),  dV = P^T dO.
//
// Two persistent kernels built like the forward (M=64 MMAs whose A operand lives in tensor
// memory, two work items per CTA on the two TMEM lane halves, gathered tiles brought in by TMA):
//  * dQ kernel, query-centric over the CSR, per block of two selected KV tiles:
//      S = Q K^T and dP = dO V^T     (A = Q, dO in TMEM; B = K, V in shared memory, K-major)
//      dS written back over S as bf16 by the softmax warps
//      dQ += dS K                    (B = the same K stage read MN-major)
//    It also computes Delta (it reads the dO rows anyway) for the second kernel.
//  * dK/dV kernel, KV-centric over the CSC, per selected query tile:
//      S^T = K Q^T and dP^T = V dO^T (A = K, V in TMEM; B = Q, dO, K-major)
//      P^T and dS^T written back as bf16
//      dV += P^T dO and dK += dS^T Q (B = dO, Q read MN-major)
// Every output row is written by one CTA (items are drawn from a global counter, but each is
// computed whole by the CTA that drew it): no atomics on the outputs, deterministic results.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int BT = 384;            // 12 warps: 0-7 softmax (two slots), 8/10 producers, 9/11 MMA issuers
constexpr uint32_t TILE_B = 8192;  // one 64 x 64 bf16 box (64 rows x 128 B, 128-byte swizzle)
constexpr float kLog2e = 1.4426950408889634f;

struct Row {
  int beg, len;
};
// Sanitised CSR/CSC row `i` of head bh; every role of a CTA reads it the same way.
__device__ __forceinline__ Row load_list(const int32_t* off, int bh, int i, int N, int cap, const DevCtx& ctx,
                                         bool report) {
  const int b = off[(size_t)bh * (N + 1) + i];
  const int e = off[(size_t)bh * (N + 1) + i + 1];
  if (b < 0 || e < b || e > cap || e - b > N) {
    if (report) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return Row{0, 0};
  }
  return Row{b, e - b};
}

// Items (b*h, tile) come from a global counter, one at a time, to the role that draws them (the
// rows of the per-sequence TopK have unequal lengths, so a fixed assignment leaves some CTAs
// finishing late); it passes each item to the other roles that walk the same stream through a
// queue of QD entries in shared memory (full / empty mbarriers, -1 ends the stream).
constexpr int QD = 4;
struct ItemQueue {
  volatile int* slot;  // [QD]
  uint64_t* full;      // [QD], one arrival (the drawing role)
  uint64_t* empty;     // [QD], one arrival per taking role
};
// The next item of a stream, as entry k of its queue: drawn from *ctr and written there (draw),
// or taken from there. -1 at the end of the items, or when a wait expired.
__device__ __forceinline__ int next_item(const ItemQueue& q, int& k, bool draw, int* ctr, int items,
                                         volatile int* abort, const DevCtx& ctx) {
  const int e = k % QD;
  int item = -1;
  if (draw) {
    item = atomicAdd(ctr, 1);
    if (item >= items) item = -1;
    if (mbar_wait(&q.empty[e], ((k / QD) & 1) ^ 1, abort, ctx)) {
      q.slot[e] = item;
      mbar_arrive(&q.full[e]);
    } else {
      item = -1;
    }
  } else {
    if (mbar_wait(&q.full[e], (k / QD) & 1, abort, ctx)) item = q.slot[e];
    mbar_arrive(&q.empty[e]);
  }
  ++k;
  return item;
}

// Op stream of one item sequence, each item's list cut into blocks of `per_blk` tiles, ops
// A(0), B(0), A(1), B(1), ... (A = the MMAs that need fresh operands, B = the MMAs that consume
// the softmax output). The producers and the MMA issuers walk it identically.
struct Seq {
  int kq;  // queue entries passed
  int bh, it, nblk, len, beg;
  int a_next, b_next;
  int tile;  // non-empty items started so far
  bool active;
  __device__ void init() {
    kq = 0;
    nblk = len = beg = bh = it = 0;
    a_next = b_next = 0;
    tile = 0;
    active = true;
  }
};
struct SeqSrc {  // where a walker's next item comes from
  ItemQueue q;
  bool draw;
  int* ctr;
  int items;
  volatile int* abort;
};

// 0 = none (slot finished), 1 = A op, 2 = B op; *blk = block index within the item. With
// ahead = 1 the A op of block n+1 comes before the B op of block n.
__device__ __forceinline__ int next_op(Seq& q, int* blk, const int32_t* off, int N, int cap, int per_blk,
                                       const DevCtx& ctx, const SeqSrc& src, int ahead = 0) {
  while (q.active) {
    if (q.a_next < q.nblk && q.a_next <= q.b_next + ahead) {
      *blk = q.a_next++;
      return 1;
    }
    if (q.b_next < q.a_next) {
      *blk = q.b_next++;
      return 2;
    }
    const int item = next_item(src.q, q.kq, src.draw, src.ctr, src.items, src.abort, ctx);
    if (item < 0) {
      q.active = false;
      return 0;
    }
    q.bh = item / N;
    q.it = item - q.bh * N;
    const Row r = load_list(off, q.bh, q.it, N, cap, ctx, false);
    q.len = r.len;
    q.beg = r.beg;
    q.nblk = (r.len + per_blk - 1) / per_blk;
    q.a_next = q.b_next = 0;
    if (q.nblk > 0) q.tile++;
  }
  return 0;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// A 128-wide bf16 row into the TMEM A-operand layout of a 16-lane slice (16x64b access):
// the thread writes packed words 2i + par_c, i < 32.
__device__ __forceinline__ void row_to_tmem(uint32_t taddr, const __nv_bfloat16* src_row, int par_c) {
  uint32_t v[32];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(src_row);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __ldg(src + 2 * i + par_c);
  tmem_st16x64b_x32(taddr, v);
}

// Store a 128-wide fp32 row held as columns 2i + par_c (i < 64) by a thread pair: one exchange
// gives each thread adjacent column pairs, written as float2.
__device__ __forceinline__ void store_row_f32(float* dst, const uint32_t (&v)[64], float scale, int par_c) {
#pragma unroll
  for (int i2 = 0; i2 < 32; ++i2) {
    const float a = __uint_as_float(v[2 * i2]) * scale, b = __uint_as_float(v[2 * i2 + 1]) * scale;
    const float recv = __shfl_xor_sync(0xffffffffu, par_c ? a : b, 2);
    reinterpret_cast<float2*>(dst)[2 * i2 + par_c] = par_c ? make_float2(recv, b) : make_float2(a, recv);
  }
}

// =========================================================================================
// dQ kernel
// =========================================================================================
namespace dqk {
constexpr int KST = 2, VST = 1;         // per slot: a K block is held until its dQ MMAs are done
constexpr uint32_t BLK_B = 4 * TILE_B;  // two KV tiles: [d half 0: tile a, tile b][d half 1: tile a, tile b]
// Each slot has its own K and V rings (one producer, one consumer each), so every barrier wait
// is for the phase in progress or the one just completed.
constexpr uint32_t OFF_K = 0;                          // [slot][KST] blocks
constexpr uint32_t OFF_V = OFF_K + 2 * KST * BLK_B;    // [slot][VST] blocks
constexpr uint32_t OFF_BAR = OFF_V + 2 * VST * BLK_B;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr uint32_t OFF_IQ = OFF_FLAG + 64;  // [slot][QD] item queue, then [slot][2] softmax hand-over
constexpr uint32_t SMEM_DYN = OFF_IQ + 64 + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");
// TMEM columns (both slots, through the lane halves)
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_Q = 256, TM_DO = 320, TM_DQ = 384;
struct Bars {
  uint64_t kfull[2][KST], kempty[2][KST], vfull[2][VST], vempty[2][VST];  // [slot][stage]
  uint64_t sfull[2], dsfull[2], bdone[2], qready[2];
  uint64_t done[2];
  uint64_t iqfull[2][QD], iqempty[2][QD];  // [slot][entry]
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// dS for 64 columns (32 per thread, columns 2j + par_c of the half), packed to 16 bf16 words.
// nl2 = -lse * log2(e), nd = -Delta; the two columns of a step go through packed fp32 math.
__device__ __forceinline__ void ds_half(const uint32_t (&sv)[32], const uint32_t (&dp)[32], float c2, float nl2,
                                        float nd, int par_c, uint32_t* pk) {
  const float2 cc = make_float2(c2, c2), ll = make_float2(nl2, nl2), dd = make_float2(nd, nd);
#pragma unroll
  for (int i2 = 0; i2 < 16; ++i2) {
    const float2 arg = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1])), cc, ll);
    const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
    const float2 ds =
        __fmul2_rn(p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * i2]), __uint_as_float(dp[2 * i2 + 1])), dd));
    pk[i2] = pair_pack_bf16(ds.x, ds.y, pair_perm(par_c));
  }
}
// Scores of the padding keys of a tile (bit u of `real` clear for padding token u; this thread
// holds columns 2i + par_c) set to -inf.
__device__ __forceinline__ void mask_keys(uint32_t (&sv)[32], uint64_t real, int par_c) {
  if (real == ~0ull) return;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (!((real >> (2 * i + par_c)) & 1ull)) sv[i] = __float_as_uint(-INFINITY);
}
}  // namespace dqk

__global__ void __launch_bounds__(BT, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __nv_bfloat16* __restrict__ qg, const __nv_bfloat16* __restrict__ og,
                          const __nv_bfloat16* __restrict__ dog, const float* __restrict__ lse,
                          float* __restrict__ ndelta, float* __restrict__ nlse2, const int32_t* __restrict__ kv_off,
                          const int32_t* __restrict__ kv_idx, float* __restrict__ dq_out, int N, int L, int topk,
                          int items, float c2, float scale, const uint64_t* __restrict__ tmask,
                          int* __restrict__ work_ctr, DevCtx ctx) {
  using namespace dqk;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);  // [0] abort, [4] tmem base
  volatile int* abort = flag_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int s = 0; s < 2; ++s) {
      for (int i = 0; i < KST; ++i) mbar_init(&B.kfull[s][i], 1), mbar_init(&B.kempty[s][i], 1);
      for (int i = 0; i < VST; ++i) mbar_init(&B.vfull[s][i], 1), mbar_init(&B.vempty[s][i], 1);
      mbar_init(&B.sfull[s], 1);
      mbar_init(&B.dsfull[s], 4);
      mbar_init(&B.bdone[s], 1);
      mbar_init(&B.qready[s], 4);
      mbar_init(&B.done[s], 1);
      for (int i = 0; i < QD; ++i) mbar_init(&B.iqfull[s][i], 1), mbar_init(&B.iqempty[s][i], 2);
    }
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(reinterpret_cast<uint32_t*>(flag_sh + 4), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(flag_sh + 4);

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------------ TMA producer of slot (warp - 8) / 2
    // the K block and the V block (two KV tiles each) of every A op of the slot, one thread
    if (lane == 0) {
      const int s = (warp - 8) >> 1;
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // the slot's items: drawn here from the counter and passed to its MMA issuer and softmax
      const SeqSrc src{ItemQueue{reinterpret_cast<volatile int*>(dsm + OFF_IQ) + s * QD, B.iqfull[s], B.iqempty[s]},
                       true, work_ctr, items, abort};
      Seq sq;
      sq.init();
      int c = 0;
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        if (next_op(sq, &blk, kv_off, N, cap, 2, ctx, src) != 1) continue;
        const int ntile = min(2, sq.len - 2 * blk);
        int j[2] = {0, 0};
        for (int tt = 0; tt < ntile; ++tt) {
          int v = kv_idx[(size_t)sq.bh * cap + sq.beg + 2 * blk + tt];
          if (v < 0 || v >= N) {
            if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
            v = min(max(v, 0), N - 1);
          }
          j[tt] = v;
        }
        const int ks = c % KST, vs = c % VST;
        if (!(ok = mbar_wait(&B.kempty[s][ks], ((c / KST) & 1) ^ 1, abort, ctx))) break;
        mbar_arrive_expect_tx(&B.kfull[s][ks], ntile * 2 * TILE_B);
        uint8_t* kd = dsm + OFF_K + (s * KST + ks) * BLK_B;
        for (int tt = 0; tt < ntile; ++tt)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(kd + h * 2 * TILE_B + tt * TILE_B, &tm_k, h * 64, sq.bh * L + j[tt] * 64, &B.kfull[s][ks]);
        if (!(ok = mbar_wait(&B.vempty[s][vs], ((c / VST) & 1) ^ 1, abort, ctx))) {
          ++c;  // the K block of position c is in flight
          break;
        }
        mbar_arrive_expect_tx(&B.vfull[s][vs], ntile * 2 * TILE_B);
        uint8_t* vd = dsm + OFF_V + (s * VST + vs) * BLK_B;
        for (int tt = 0; tt < ntile; ++tt)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(vd + h * 2 * TILE_B + tt * TILE_B, &tm_v, h * 64, sq.bh * L + j[tt] * 64, &B.vfull[s][vs]);
        ++c;
      }
      if (*abort) {  // let copies still in flight land before the CTA exits
        for (int cc = max(0, c - KST); cc < c; ++cc)
          mbar_wait_drain(&B.kfull[s][cc % KST], (cc / KST) & 1, ctx.timeout_ns);
        for (int cc = max(0, c - VST); cc < c; ++cc)
          mbar_wait_drain(&B.vfull[s][cc % VST], (cc / VST) & 1, ctx.timeout_ns);
      }
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuer of slot (warp - 9) / 2
    if (lane == 0) {
      const int s = (warp - 9) >> 1;
      constexpr uint32_t id_kmaj = idesc_bf16_f32(64, 128, false, false);  // S, dP: N = 128 keys
      constexpr uint32_t id_mn = idesc_bf16_f32(64, 128, false, true);     // dQ: N = 128 (d)
      const uint32_t lanes = (uint32_t)(16 * s) << 16;
      const SeqSrc src{ItemQueue{reinterpret_cast<volatile int*>(dsm + OFF_IQ) + s * QD, B.iqfull[s], B.iqempty[s]},
                       false, work_ctr, items, abort};
      Seq sq;
      sq.init();
      int ga = 0, gb = 0;  // A and B ops issued
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        const int op = next_op(sq, &blk, kv_off, N, cap, 2, ctx, src);
        if (op == 1) {
          if (blk == 0 && !(ok = mbar_wait(&B.qready[s], (sq.tile - 1) & 1, abort, ctx))) break;
          // S / dP of this slot are free once the previous dQ MMAs (which read dS) are done
          if (ga > 0 && !(ok = mbar_wait(&B.bdone[s], (ga - 1) & 1, abort, ctx))) break;
          const int ks = ga % KST, vs = ga % VST;
          if (!(ok = mbar_wait(&B.kfull[s][ks], (ga / KST) & 1, abort, ctx))) break;
          if (!(ok = mbar_wait(&B.vfull[s][vs], (ga / VST) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(dsm + OFF_K + (s * KST + ks) * BLK_B);
          const uint32_t va = smem_u32(dsm + OFF_V + (s * VST + vs) * BLK_B);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + lanes + TM_S, tmem + lanes + TM_Q + 8 * kk,
                        sdesc_sw128(ka + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_kmaj, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + lanes + TM_DP, tmem + lanes + TM_DO + 8 * kk,
                        sdesc_sw128(va + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_kmaj, kk > 0);
          mma_commit(&B.vempty[s][vs]);
          mma_commit(&B.sfull[s]);
          ++ga;
        } else if (op == 2) {
          // dQ += dS K, dS in the S region (bf16), K read MN-major from the A op's stage
          if (!(ok = mbar_wait(&B.dsfull[s], gb & 1, abort, ctx))) break;
          tc_fence_after();
          const int ks = gb % KST;
          const uint32_t ka = smem_u32(dsm + OFF_K + (s * KST + ks) * BLK_B);
          const int ksteps = (2 * blk + 1 == sq.len) ? 4 : 8;
          for (int kk = 0; kk < ksteps; ++kk)
            mma_bf16_ts(tmem + lanes + TM_DQ, tmem + lanes + TM_S + 8 * kk,
                        sdesc_sw128(ka + kk * 2048, 2 * TILE_B, 1024), id_mn, (blk > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.kempty[s][ks]);
          mma_commit(&B.bdone[s]);
          ++gb;
        }
      }
      mma_commit(&B.done[s]);
      mbar_wait_drain(&B.done[s], 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax, one slot per warpgroup
    const int s = warp >> 2, w = warp & 3;
    const int bar_id = 1 + s;
    const int par_c = (lane >> 1) & 1;
    const int row = 16 * w + 8 * (lane & 1) + (lane >> 2);
    const uint32_t tl = tmem + ((uint32_t)(32 * w + 16 * s) << 16);
    int g = 0;  // blocks processed by this slot
    const ItemQueue iq{reinterpret_cast<volatile int*>(dsm + OFF_IQ) + s * QD, B.iqfull[s], B.iqempty[s]};
    volatile int* handover = reinterpret_cast<volatile int*>(dsm + OFF_IQ) + 2 * QD + 2 * s;  // [kq parity]
    for (int kq = 0;;) {
      // the slot's first warp takes the next item and hands it to the other three (the hand-over
      // word alternates with the entry's parity, so it is rewritten only after every warp passed
      // the next barrier)
      const int par = kq & 1;
      if (w == 0 && lane == 0) handover[par] = next_item(iq, kq, false, nullptr, items, abort, ctx);
      else ++kq;
      named_bar_sync(bar_id, 128);
      const int item = handover[par];
      if (item < 0) break;
      const int bh = item / N, qt = item - bh * N;
      const Row rw = load_list(kv_off, bh, qt, N, cap, ctx, w == 0 && lane == 0);
      const int nblk = (rw.len + 1) >> 1;
      const size_t tok = (size_t)bh * L + (size_t)qt * 64 + row;
      float* dst = dq_out + tok * 128;
      if (nblk == 0) {
        float4* d4 = reinterpret_cast<float4*>(dst + par_c * 64);
#pragma unroll
        for (int e = 0; e < 16; ++e) d4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      // Q and dO rows into TMEM; Delta = rowsum(dO * O) from the same words of dO
      row_to_tmem(tl + TM_Q, qg + tok * 128, par_c);
      float dlt;
      {
        uint32_t v[32];
        const uint32_t* dsrc = reinterpret_cast<const uint32_t*>(dog + tok * 128);
        const uint32_t* osrc = reinterpret_cast<const uint32_t*>(og + tok * 128);
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = __ldg(dsrc + 2 * i + par_c);
          const uint32_t ow = __ldg(osrc + 2 * i + par_c);
          part = fmaf(bf_lo(v[i]), bf_lo(ow), part);
          part = fmaf(bf_hi(v[i]), bf_hi(ow), part);
        }
        tmem_st16x64b_x32(tl + TM_DO, v);
        dlt = part + __shfl_xor_sync(0xffffffffu, part, 2);
      }
      // a row with lse = -inf (a padding query row of a padded grid) has P = 0: -lse * log2(e)
      // is taken as -inf here and in the dK/dV kernel, which reads it from the workspace
      const float lse_t = lse[tok];
      const float nl2 = lse_t == -INFINITY ? -INFINITY : -lse_t * kLog2e;
      if (par_c == 0) {  // for the dK/dV kernel
        ndelta[tok] = -dlt;
        nlse2[tok] = nl2;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.qready[s]);
      for (int n = 0; n < nblk; ++n, ++g) {
        const bool half = (2 * n + 1 == rw.len);
        mbar_wait(&B.sfull[s], g & 1, abort, ctx);
        tc_fence_after();
        uint32_t pk[32];
        // padding keys of a padded grid (tmask): S = -inf, so P = dS = 0
        uint64_t km[2] = {~0ull, ~0ull};
        if (tmask) {
          const int32_t* ix = kv_idx + (size_t)bh * cap + rw.beg + 2 * n;
          km[0] = __ldg(tmask + min(max(__ldg(ix), 0), N - 1));
          if (!half) km[1] = __ldg(tmask + min(max(__ldg(ix + 1), 0), N - 1));
        }
        {
          uint32_t sv[32], dp[32];
          tmem_ld16x64b_x32(tl + TM_S, sv);
          tmem_ld16x64b_x32(tl + TM_DP, dp);
          tmem_ld_wait();
          mask_keys(sv, km[0], par_c);
          ds_half(sv, dp, c2, nl2, -dlt, par_c, pk);
        }
        if (!half) {
          uint32_t sv[32], dp[32];
          tmem_ld16x64b_x32(tl + TM_S + 64, sv);
          tmem_ld16x64b_x32(tl + TM_DP + 64, dp);
          tmem_ld_wait();
          mask_keys(sv, km[1], par_c);
          ds_half(sv, dp, c2, nl2, -dlt, par_c, pk + 16);
        } else {
#pragma unroll
          for (int i = 16; i < 32; ++i) pk[i] = 0u;
        }
        tmem_st16x64b_x32(tl + TM_S, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.dsfull[s]);
      }
      // epilogue: the last dQ block is done -> scale by 1/sqrt(D) and store fp32
      mbar_wait(&B.bdone[s], (g - 1) & 1, abort, ctx);
      tc_fence_after();
      uint32_t o[64];
      tmem_ld16x64b_x64(tl + TM_DQ, o);
      tmem_ld_wait();
      store_row_f32(dst, o, scale, par_c);
      if (named_bar_or(bar_id, 128, *abort != 0)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================================
// dK / dV kernel
// =========================================================================================
// One KV tile per CTA at a time, M=128 MMAs over all TMEM lanes. Lane 2j holds key j's K row and
// lane 2j+1 its V row, so with B = [Q; dO] of one selected query tile (N = 128) a single MMA per
// K-step gives S^T = K Q^T on the even lanes (columns 0-63) and dP^T = V dO^T on the odd lanes
// (columns 64-127); the two other quadrants are not used. The softmax writes P^T (even lanes)
// and dS^T (odd lanes) back as one bf16 A operand, and with B = [Q | dO] (N = 256) the second MMA
// accumulates dV = P^T dO on the even lanes and dK = dS^T Q on the odd lanes. Per query tile the
// tensor pipe does two M=128 K-loops instead of the four M=64, N=64 ones of a per-key-half split.
namespace dkv {
constexpr int KT = 384;               // 12 warps: 0-7 softmax, 8/10 producers, 9 and 11 MMA issuers
constexpr int RST = 6;                // ring stages; warp 8 fills the even ring positions, warp 10 the odd
constexpr uint32_t STAGE_B = 33792;   // [d half 0: Q, dO][d half 1: Q, dO], then 64 -lse*log2e, 64 -Delta
constexpr uint32_t OFF_BAR = RST * STAGE_B;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr uint32_t OFF_IQ = OFF_FLAG + 64;  // [QD] item queue, then [2] softmax hand-over
constexpr uint32_t SMEM_DYN = OFF_IQ + 64 + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");
static_assert(RST % 2 == 0, "each ring stage must have a single producer");
// TMEM columns (all 128 lanes)
constexpr uint32_t TM_KV = 0;     // A of the first MMA: K row (even lanes) / V row (odd lanes), 64 columns
constexpr uint32_t TM_SP = 64;    // D of the first MMA: S^T (even lanes, 0-63), dP^T (odd lanes, 64-127)
constexpr uint32_t TM_PDS = 192;  // A of the second MMA: P^T (even) / dS^T (odd) in bf16, 2 buffers x 32
constexpr uint32_t TM_G = 256;    // D of the second MMA: dV (even lanes) / dK (odd lanes), 256 columns
struct Bars {
  uint64_t full[RST], empty[RST];
  uint64_t spfull, spfree, pdsfull[2], pdsfree[2], itemdone, kvready;
  uint64_t done[2];
  uint64_t iqfull[QD], iqempty[QD];
};
static_assert(sizeof(Bars) <= 512, "barrier area");
}  // namespace dkv

__global__ void __launch_bounds__(dkv::KT, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                            const __nv_bfloat16* __restrict__ kg, const __nv_bfloat16* __restrict__ vg,
                            const float* __restrict__ nlse2, const float* __restrict__ ndelta,
                            const int32_t* __restrict__ q_off, const int32_t* __restrict__ q_idx,
                            float* __restrict__ dk_out, float* __restrict__ dv_out, int N, int L, int topk, int items,
                            float c2, float scale, const uint64_t* __restrict__ tmask, int* __restrict__ work_ctr,
                            DevCtx ctx) {
  using namespace dkv;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);
  volatile int* abort = flag_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int i = 0; i < RST; ++i) mbar_init(&B.full[i], 1), mbar_init(&B.empty[i], 1);
    mbar_init(&B.spfull, 1);
    mbar_init(&B.spfree, 8);
    for (int b = 0; b < 2; ++b) mbar_init(&B.pdsfull[b], 8), mbar_init(&B.pdsfree[b], 1);
    mbar_init(&B.itemdone, 1);
    mbar_init(&B.kvready, 8);
    mbar_init(&B.done[0], 1);
    mbar_init(&B.done[1], 1);
    // the KV tiles: drawn from the counter by warp 8, taken by warp 10, both MMA issuers and
    // the softmax
    for (int i = 0; i < QD; ++i) mbar_init(&B.iqfull[i], 1), mbar_init(&B.iqempty[i], 4);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(reinterpret_cast<uint32_t*>(flag_sh + 4), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(flag_sh + 4);
  const ItemQueue iq{reinterpret_cast<volatile int*>(dsm + OFF_IQ), B.iqfull, B.iqempty};

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------------ producers (lane 0)
    // ring position c holds the c-th selecting query tile of this CTA: its Q and dO tiles (two
    // boxes each) and its 64 -lse*log2(e) and -Delta values; warp 8 fills even positions and
    // warp 10 odd ones, so every stage has one producer
    if (lane == 0) {
      const int par = (warp - 8) >> 1;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      const SeqSrc src{iq, par == 0, work_ctr, items, abort};
      Seq sq;
      sq.init();
      int c = 0, last = -1;
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        if (next_op(sq, &blk, q_off, N, cap, 1, ctx, src) != 1) continue;
        const int pos = c++;
        if ((pos & 1) != par) continue;
        int i = q_idx[(size_t)sq.bh * cap + sq.beg + blk];
        if (i < 0 || i >= N) {
          if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
          i = min(max(i, 0), N - 1);
        }
        const int st = pos % RST;
        if (!(ok = mbar_wait(&B.empty[st], ((pos / RST) & 1) ^ 1, abort, ctx))) break;
        uint8_t* stage = dsm + st * STAGE_B;
        const int row0 = sq.bh * L + i * 64;
        mbar_arrive_expect_tx(&B.full[st], 4 * TILE_B + 512);
        tma_load_2d(stage, &tm_q, 0, row0, &B.full[st]);
        tma_load_2d(stage + TILE_B, &tm_do, 0, row0, &B.full[st]);
        tma_load_2d(stage + 2 * TILE_B, &tm_q, 64, row0, &B.full[st]);
        tma_load_2d(stage + 3 * TILE_B, &tm_do, 64, row0, &B.full[st]);
        bulk_load(stage + 4 * TILE_B, nlse2 + row0, 256, &B.full[st]);
        bulk_load(stage + 4 * TILE_B + 256, ndelta + row0, 256, &B.full[st]);
        last = pos;
      }
      if (*abort)  // let copies still in flight land before the CTA exits
        for (int pos = last; pos >= 0 && pos > last - RST; pos -= 2)
          mbar_wait_drain(&B.full[pos % RST], (pos / RST) & 1, ctx.timeout_ns);
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuers (lane 0)
    // warp 9 issues the S^T / dP^T MMAs, warp 11 the dV / dK MMAs, so the next query tile's first
    // MMAs are never held behind the previous tile's second ones in one issue order. The stage
    // of tile n is released after its second MMAs, which start only after its first ones are
    // done (through the softmax), and each commit covers the MMAs of its own thread.
    if (lane == 0) {
      const bool first = warp == 9;
      constexpr uint32_t id_a = idesc_bf16_f32(128, 128, false, false);  // [K;V] x [Q;dO]^T
      constexpr uint32_t id_b = idesc_bf16_f32(128, 256, false, true);   // [P;dS] x [Q | dO]
      const SeqSrc src{iq, false, work_ctr, items, abort};
      Seq sq;
      sq.init();
      int cnt = 0;  // MMAs groups issued by this thread
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        const int op = next_op(sq, &blk, q_off, N, cap, 1, ctx, src);
        if (op == 1 && first) {
          if (blk == 0 && !(ok = mbar_wait(&B.kvready, (sq.tile - 1) & 1, abort, ctx))) break;
          // S^T / dP^T of the previous query tile must have been read by the softmax
          if (cnt > 0 && !(ok = mbar_wait(&B.spfree, (cnt - 1) & 1, abort, ctx))) break;
          const int st = cnt % RST;
          if (!(ok = mbar_wait(&B.full[st], (cnt / RST) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(dsm + st * STAGE_B);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + TM_SP, tmem + TM_KV + 8 * kk,
                        sdesc_sw128(qa + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_a, kk > 0);
          mma_commit(&B.spfull);
          ++cnt;
        } else if (op == 2 && !first) {
          const int b = cnt & 1;
          if (!(ok = mbar_wait(&B.pdsfull[b], (cnt >> 1) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(dsm + (cnt % RST) * STAGE_B);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + TM_G, tmem + TM_PDS + 32 * b + 8 * kk, sdesc_sw128(qa + kk * 2048, TILE_B, 1024), id_b,
                        (blk > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.empty[cnt % RST]);
          mma_commit(&B.pdsfree[b]);
          if (blk == sq.len - 1) mma_commit(&B.itemdone);
          ++cnt;
        }
      }
      mma_commit(&B.done[first ? 0 : 1]);
      mbar_wait_drain(&B.done[first ? 0 : 1], 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax (8 warps)
    // warp w reads TMEM lane quarter w % 4 and handles query half c = w / 4 of each tile
    const int c = warp >> 2;
    const int lrow = 32 * (warp & 3) + lane;
    const int j = lrow >> 1, kind = lrow & 1;  // key row of the tile; 0: K side, 1: V side
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const float2 cc = make_float2(c2, c2);
    int n = 0, it = 0;  // query tiles processed, non-empty items processed
    volatile int* handover = reinterpret_cast<volatile int*>(dsm + OFF_IQ) + QD;  // [kq parity]
    for (int kq = 0;;) {
      // warp 0 takes the next KV tile and hands it to the other seven (the hand-over word
      // alternates with the entry's parity, so it is rewritten only after every warp passed the
      // next barrier)
      const int par = kq & 1;
      if (warp == 0 && lane == 0) handover[par] = next_item(iq, kq, false, nullptr, items, abort, ctx);
      else ++kq;
      named_bar_sync(1, 256);
      const int item = handover[par];
      if (item < 0) break;
      const int bh = item / N, kt = item - bh * N;
      const Row rw = load_list(q_off, bh, kt, N, cap, ctx, warp == 0 && lane == 0);
      const size_t tok = (size_t)bh * L + (size_t)kt * 64 + j;
      float* gout = (kind ? dk_out : dv_out) + tok * 128 + 64 * c;
      // a padding key of a padded grid takes no part: S = -inf, so its P, dS, dK and dV are 0
      const bool key_real = !tmask || ((__ldg(tmask + kt) >> j) & 1ull);
      if (rw.len == 0) {
        float4* z = reinterpret_cast<float4*>(gout);
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      {
        // this lane's K or V row into the first MMA's A operand (d in [64c, 64c + 64))
        uint32_t v[32];
        const uint32_t* src = reinterpret_cast<const uint32_t*>((kind ? vg : kg) + tok * 128) + 32 * c;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __ldg(src + i);
        tmem_st32(tl + TM_KV + 32 * c, v);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.kvready);
      for (int t = 0; t < rw.len; ++t, ++n) {
        const int st = n % RST, b = n & 1;
        mbar_wait(&B.spfull, n & 1, abort, ctx);
        mbar_wait(&B.full[st], (n / RST) & 1, abort, ctx);  // the stage's per-query vectors
        tc_fence_after();
        uint32_t sa[32], da[32];
        tmem_ld32(tl + TM_SP + 32 * c, sa);       // even lanes: S^T[j][32c + i]
        tmem_ld32(tl + TM_SP + 64 + 32 * c, da);  // odd lanes: dP^T[j][32c + i]
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.spfree);
        // this thread takes queries 32c + 16*kind + i (i < 16): the lane pair swaps S and dP
        float sv[16], dv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t recv = __shfl_xor_sync(0xffffffffu, kind ? da[i] : sa[16 + i], 1);
          sv[i] = key_real ? __uint_as_float(kind ? recv : sa[i]) : -INFINITY;
          dv[i] = __uint_as_float(kind ? da[16 + i] : recv);
        }
        const float2* nl = reinterpret_cast<const float2*>(dsm + st * STAGE_B + 4 * TILE_B) + 16 * c + 8 * kind;
        const float2* nd = nl + 32;
        uint32_t own[8], other[8];  // packed bf16 pairs: even lanes own P, odd lanes own dS
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          const float2 arg = __ffma2_rn(make_float2(sv[2 * i2], sv[2 * i2 + 1]), cc, nl[i2]);
          const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
          const float2 ds = __fmul2_rn(p, __fadd2_rn(make_float2(dv[2 * i2], dv[2 * i2 + 1]), nd[i2]));
          const uint32_t wp = pack_bf16(p.x, p.y), wd = pack_bf16(ds.x, ds.y);
          own[i2] = kind ? wd : wp;
          other[i2] = kind ? wp : wd;
        }
        // even lanes' row is P^T, odd lanes' dS^T: swap the halves the other lane needs
        uint32_t row16[16];
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          const uint32_t r = __shfl_xor_sync(0xffffffffu, other[i2], 1);
          row16[i2] = kind ? r : own[i2];
          row16[8 + i2] = kind ? own[i2] : r;
        }
        if (n >= 2) mbar_wait(&B.pdsfree[b], ((n >> 1) - 1) & 1, abort, ctx);  // second MMA of n - 2
        tmem_st32x16(tl + TM_PDS + 32 * b + 16 * c, row16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.pdsfull[b]);
      }
      // epilogue: the item's MMAs are done; this lane's half row of dV (even) or dK (odd)
      mbar_wait(&B.itemdone, it & 1, abort, ctx);
      ++it;
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t gk[32], gv[32];
        tmem_ld32(tl + TM_G + 128 * c + 32 * h2, gk);       // dK columns of d half c (odd lanes)
        tmem_ld32(tl + TM_G + 128 * c + 64 + 32 * h2, gv);  // dV columns of d half c (even lanes)
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(gout + 32 * h2);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t* src = kind ? gk + 4 * e : gv + 4 * e;
          const float f = kind ? scale : 1.f;
          dst[e] = make_float4(__uint_as_float(src[0]) * f, __uint_as_float(src[1]) * f, __uint_as_float(src[2]) * f,
                               __uint_as_float(src[3]) * f);
        }
      }
      if (named_bar_or(1, 256, *abort != 0)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                       uint32_t box_rows);

vsa2_status attn_bwd_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, const int32_t* kv_off, const int32_t* kv_idx, const int32_t* q_off,
                        const int32_t* q_idx, float* dq, float* dk, float* dv, int topk, char* ws,
                        const uint64_t* tmask, cudaStream_t s) {
  CUtensorMap tk, tv, tq, tdo;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tk, k, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tv, v, 128, rows, 64, 64) ||
      !make_tmap_2d_bf16(&tq, q, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tdo, dout, 128, rows, 64, 64))
    return tmap_fail("tensor map encoding for the backward operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  float* ndelta = reinterpret_cast<float*>(ws + ws_layout(d).delta);
  float* nlse2 = reinterpret_cast<float*>(ws + ws_layout(d).nlse2);
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(sms, (items + 1) / 2));
  const float c1 = 1.f / sqrtf(128.f);
  const float c2 = kLog2e * c1;
  // the item counter the kernels draw from (workspace header), reset before each of them
  int* ctr = reinterpret_cast<int*>(ws + kWsWorkCounter);
  cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::SMEM_DYN);
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_bwd_tc: item counter reset");
  attn_bwd_dq_tc_kernel<<<grid, BT, dqk::SMEM_DYN, s>>>(
      tk, tv, (const __nv_bfloat16*)q, (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, lse, ndelta, nlse2, kv_off,
      kv_idx, dq, d.N, (int)d.L, topk, items, c2, c1, tmask, ctr, ctx);
  if (check_launch("attn_bwd_dq_tc_kernel") != VSA2_OK) return VSA2_ERR_CUDA;
  cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM_DYN);
  const int grid_kv = std::max(1, std::min(sms, items));
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_bwd_tc: item counter reset");
  attn_bwd_dkdv_tc_kernel<<<grid_kv, dkv::KT, dkv::SMEM_DYN, s>>>(tq, tdo, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                                          nlse2, ndelta, q_off, q_idx, dk, dv, d.N, (int)d.L, topk,
                                                          items, c2, c1, tmask, ctr, ctx);
  return check_launch("attn_bwd_dkdv_tc_kernel");
}

// The dK/dV kernel alone, on the CSC of 64-token tiles, with -Delta and -lse * log2(e) already in
// the workspace (written by a dQ kernel of 128-token tiles).
vsa2_status attn_bwd_dkdv_only_tc(const Dims& d, const void* q, const void* k, const void* v, const void* dout,
                                  const int32_t* q_off, const int32_t* q_idx, float* dk, float* dv, int topk, char* ws,
                                  cudaStream_t s) {
  CUtensorMap tq, tdo;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tq, q, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tdo, dout, 128, rows, 64, 64))
    return tmap_fail("tensor map encoding for the backward operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const float* ndelta = reinterpret_cast<const float*>(ws + ws_layout(d).delta);
  const float* nlse2 = reinterpret_cast<const float*>(ws + ws_layout(d).nlse2);
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float c1 = 1.f / sqrtf(128.f);
  int* ctr = reinterpret_cast<int*>(ws + kWsWorkCounter);
  cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM_DYN);
  const int grid_kv = std::max(1, std::min(sms, items));
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_bwd_dkdv: item counter reset");
  attn_bwd_dkdv_tc_kernel<<<grid_kv, dkv::KT, dkv::SMEM_DYN, s>>>(tq, tdo, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                                          nlse2, ndelta, q_off, q_idx, dk, dv, d.N, (int)d.L, topk,
                                                          items, kLog2e * c1, c1, nullptr, ctr, ctx);
  return check_launch("attn_bwd_dkdv_tc_kernel");
}

}  // namespace vsa2
