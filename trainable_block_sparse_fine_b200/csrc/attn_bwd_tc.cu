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
// Every output row is owned by one CTA: no atomics, deterministic results.
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

// Op stream of one slot: items r*2G + 2c + s of CTA c, each item's list cut into blocks of
// `per_blk` tiles, ops A(0), B(0), A(1), B(1), ... (A = the MMAs that need fresh operands,
// B = the MMAs that consume the softmax output). The producers and the MMA issuer walk the
// merged stream slot 0, slot 1, slot 0, ... identically.
struct Seq {
  int item, stride, items;
  int bh, it, nblk, len, beg;
  int a_next, b_next;
  int tile;  // non-empty items started so far
  bool active;
  __device__ void init(int first, int step, int total) {
    item = first - step;
    stride = step;
    items = total;
    nblk = len = beg = bh = it = 0;
    a_next = b_next = 0;
    tile = 0;
    active = true;
  }
};

// 0 = none (slot finished), 1 = A op, 2 = B op; *blk = block index within the item
__device__ __forceinline__ int next_op(Seq& q, int* blk, const int32_t* off, int N, int cap, int per_blk,
                                       const DevCtx& ctx) {
  while (q.active) {
    if (q.a_next < q.nblk && q.a_next == q.b_next) {
      *blk = q.a_next++;
      return 1;
    }
    if (q.b_next < q.a_next) {
      *blk = q.b_next++;
      return 2;
    }
    q.item += q.stride;
    if (q.item >= q.items) {
      q.active = false;
      return 0;
    }
    q.bh = q.item / N;
    q.it = q.item - q.bh * N;
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
constexpr uint32_t SMEM_DYN = OFF_FLAG + 64 + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");
// TMEM columns (both slots, through the lane halves)
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_Q = 256, TM_DO = 320, TM_DQ = 384;
struct Bars {
  uint64_t kfull[2][KST], kempty[2][KST], vfull[2][VST], vempty[2][VST];  // [slot][stage]
  uint64_t sfull[2], dsfull[2], bdone[2], qready[2];
  uint64_t done[2];
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
}  // namespace dqk

__global__ void __launch_bounds__(BT, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __nv_bfloat16* __restrict__ qg, const __nv_bfloat16* __restrict__ og,
                          const __nv_bfloat16* __restrict__ dog, const float* __restrict__ lse,
                          float* __restrict__ ndelta, float* __restrict__ nlse2, const int32_t* __restrict__ kv_off,
                          const int32_t* __restrict__ kv_idx, float* __restrict__ dq_out, int N, int L, int topk,
                          int items, float c2, float scale, DevCtx ctx) {
  using namespace dqk;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);  // [0] abort, [4] tmem base
  volatile int* abort = flag_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;
  const int step = 2 * gridDim.x;

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
      Seq sq;
      sq.init(2 * blockIdx.x + s, step, items);
      int c = 0;
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        if (next_op(sq, &blk, kv_off, N, cap, 2, ctx) != 1) continue;
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
      Seq sq;
      sq.init(2 * blockIdx.x + s, step, items);
      int ga = 0, gb = 0;  // A and B ops issued
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        const int op = next_op(sq, &blk, kv_off, N, cap, 2, ctx);
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
    for (int item = 2 * blockIdx.x + s; item < items; item += step) {
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
      const float nl2 = -lse[tok] * kLog2e;
      if (par_c == 0) {
        // for the dK/dV kernel: each tile's 64 values ordered even rows, then odd rows
        const size_t perm = (size_t)bh * L + (size_t)qt * 64 + (row & 1) * 32 + (row >> 1);
        ndelta[perm] = -dlt;
        nlse2[perm] = nl2;
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
        {
          uint32_t sv[32], dp[32];
          tmem_ld16x64b_x32(tl + TM_S, sv);
          tmem_ld16x64b_x32(tl + TM_DP, dp);
          tmem_ld_wait();
          ds_half(sv, dp, c2, nl2, -dlt, par_c, pk);
        }
        if (!half) {
          uint32_t sv[32], dp[32];
          tmem_ld16x64b_x32(tl + TM_S + 64, sv);
          tmem_ld16x64b_x32(tl + TM_DP + 64, dp);
          tmem_ld_wait();
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
namespace dkv {
constexpr int RST = 3;                        // ring stages per slot
constexpr uint32_t STAGE_B = 33792;           // Q tile 16 KB, dO tile 16 KB, lse 256 B, Delta 256 B (1 KB aligned)
constexpr uint32_t OFF_BAR = 2 * RST * STAGE_B;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr uint32_t SMEM_DYN = OFF_FLAG + 64 + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");
// TMEM columns: K and V (A operands, 64 each), S^T and dP^T (64 fp32 columns each; P^T and
// dS^T are written back as bf16 over their first 32), dV and dK accumulators (128 each)
constexpr uint32_t TM_K = 0, TM_V = 64, TM_S = 128, TM_DP = 192, TM_DV = 256, TM_DK = 384;
struct Bars {
  uint64_t full[2 * RST], empty[2 * RST];
  uint64_t sfull[2], pfull[2], bdone[2], kvready[2];
  uint64_t done[2];
};
static_assert(sizeof(Bars) <= 512, "barrier area");
}  // namespace dkv

// The two slots are independent pipelines that share only the tensor pipe: slot s has its own
// producer warp (8 + 2s) and its own MMA-issuing warp (9 + 2s), so neither waits on the other.
__global__ void __launch_bounds__(BT, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                            const __nv_bfloat16* __restrict__ kg, const __nv_bfloat16* __restrict__ vg,
                            const float* __restrict__ nlse2, const float* __restrict__ ndelta,
                            const int32_t* __restrict__ q_off, const int32_t* __restrict__ q_idx,
                            float* __restrict__ dk_out, float* __restrict__ dv_out, int N, int L, int topk, int items,
                            float c2, float scale, DevCtx ctx) {
  using namespace dkv;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);
  volatile int* abort = flag_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;
  const int step = 2 * gridDim.x;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int i = 0; i < 2 * RST; ++i) mbar_init(&B.full[i], 1), mbar_init(&B.empty[i], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.sfull[s], 1);
      mbar_init(&B.pfull[s], 4);
      mbar_init(&B.bdone[s], 1);
      mbar_init(&B.kvready[s], 4);
      mbar_init(&B.done[s], 1);
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
    // ------------------------------------------------------------------ producer of slot (warp - 8) / 2
    // per selected query tile: its Q and dO tiles (two boxes each) and its 64 -lse*log2(e) and
    // -Delta values (written by the dQ kernel), into the slot's ring (stage = the slot's tile count mod RST)
    if (lane == 0) {
      const int s = (warp - 8) >> 1;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      Seq sq;
      sq.init(2 * blockIdx.x + s, step, items);
      int cnt = 0;
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        if (next_op(sq, &blk, q_off, N, cap, 1, ctx) != 1) continue;
        int i = q_idx[(size_t)sq.bh * cap + sq.beg + blk];
        if (i < 0 || i >= N) {
          if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
          i = min(max(i, 0), N - 1);
        }
        const int r = s * RST + cnt % RST;
        if (!(ok = mbar_wait(&B.empty[r], ((cnt / RST) & 1) ^ 1, abort, ctx))) break;
        uint8_t* stage = dsm + r * STAGE_B;
        const int row0 = sq.bh * L + i * 64;
        mbar_arrive_expect_tx(&B.full[r], 4 * TILE_B + 512);
        tma_load_2d(stage, &tm_q, 0, row0, &B.full[r]);
        tma_load_2d(stage + TILE_B, &tm_q, 64, row0, &B.full[r]);
        tma_load_2d(stage + 2 * TILE_B, &tm_do, 0, row0, &B.full[r]);
        tma_load_2d(stage + 3 * TILE_B, &tm_do, 64, row0, &B.full[r]);
        bulk_load(stage + 4 * TILE_B, nlse2 + row0, 256, &B.full[r]);
        bulk_load(stage + 4 * TILE_B + 256, ndelta + row0, 256, &B.full[r]);
        ++cnt;
      }
      if (*abort)  // let copies still in flight land before the CTA exits
        for (int cc = max(0, cnt - RST); cc < cnt; ++cc)
          mbar_wait_drain(&B.full[s * RST + cc % RST], (cc / RST) & 1, ctx.timeout_ns);
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuer of slot (warp - 9) / 2
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(64, 64, false, false);  // S^T, dP^T: N = 64 queries
      constexpr uint32_t id_g = idesc_bf16_f32(64, 128, false, true);  // dV, dK: N = 128 (d)
      const int s = (warp - 9) >> 1;
      const uint32_t lanes = (uint32_t)(16 * s) << 16;
      Seq sq;
      sq.init(2 * blockIdx.x + s, step, items);
      int ga = 0, gb = 0;
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        const int op = next_op(sq, &blk, q_off, N, cap, 1, ctx);
        if (op == 1) {
          if (blk == 0 && !(ok = mbar_wait(&B.kvready[s], (sq.tile - 1) & 1, abort, ctx))) break;
          // S^T / dP^T are free once the previous dV / dK MMAs (which read P^T / dS^T) are done
          if (ga > 0 && !(ok = mbar_wait(&B.bdone[s], (ga - 1) & 1, abort, ctx))) break;
          const int r = s * RST + ga % RST;
          if (!(ok = mbar_wait(&B.full[r], (ga / RST) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(dsm + r * STAGE_B), da = qa + 2 * TILE_B;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + lanes + TM_S, tmem + lanes + TM_K + 8 * kk,
                        sdesc_sw128(qa + (kk >> 2) * TILE_B + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + lanes + TM_DP, tmem + lanes + TM_V + 8 * kk,
                        sdesc_sw128(da + (kk >> 2) * TILE_B + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
          mma_commit(&B.sfull[s]);
          ++ga;
        } else if (op == 2) {
          // dV += P^T dO, dK += dS^T Q; P^T / dS^T in TMEM (bf16), dO / Q read MN-major
          if (!(ok = mbar_wait(&B.pfull[s], gb & 1, abort, ctx))) break;
          tc_fence_after();
          const int r = s * RST + gb % RST;
          const uint32_t qa = smem_u32(dsm + r * STAGE_B), da = qa + 2 * TILE_B;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + lanes + TM_DV, tmem + lanes + TM_S + 8 * kk, sdesc_sw128(da + kk * 2048, TILE_B, 1024),
                        id_g, (blk > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + lanes + TM_DK, tmem + lanes + TM_DP + 8 * kk, sdesc_sw128(qa + kk * 2048, TILE_B, 1024),
                        id_g, (blk > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.empty[r]);
          mma_commit(&B.bdone[s]);
          ++gb;
        }
      }
      mma_commit(&B.done[s]);
      mbar_wait_drain(&B.done[s], 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax, one slot per warpgroup
    // rows are keys of the KV tile, columns are queries of the selected query tile
    const int s = warp >> 2, w = warp & 3;
    const int bar_id = 1 + s;
    const int par_c = (lane >> 1) & 1;
    const int row = 16 * w + 8 * (lane & 1) + (lane >> 2);
    const uint32_t tl = tmem + ((uint32_t)(32 * w + 16 * s) << 16);
    int g = 0;  // query tiles processed by this slot
    for (int item = 2 * blockIdx.x + s; item < items; item += step) {
      const int bh = item / N, kt = item - bh * N;
      const Row rw = load_list(q_off, bh, kt, N, cap, ctx, w == 0 && lane == 0);
      const size_t tok = (size_t)bh * L + (size_t)kt * 64 + row;
      float* dkd = dk_out + tok * 128;
      float* dvd = dv_out + tok * 128;
      if (rw.len == 0) {
        float4* a4 = reinterpret_cast<float4*>(dkd + par_c * 64);
        float4* b4 = reinterpret_cast<float4*>(dvd + par_c * 64);
#pragma unroll
        for (int e = 0; e < 16; ++e) a4[e] = b4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      row_to_tmem(tl + TM_K, kg + tok * 128, par_c);
      row_to_tmem(tl + TM_V, vg + tok * 128, par_c);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.kvready[s]);
      for (int n = 0; n < rw.len; ++n, ++g) {
        const int r = s * RST + g % RST;
        mbar_wait(&B.sfull[s], g & 1, abort, ctx);
        // the stage's lse / Delta were written by the bulk copy: observe its barrier too
        mbar_wait(&B.full[r], (g / RST) & 1, abort, ctx);
        tc_fence_after();
        // this thread's query columns are 4*i2 + par_c and 4*i2 + 2 + par_c: in the even/odd
        // order of the stage they are one aligned float2
        const float2* nl2 = reinterpret_cast<const float2*>(dsm + r * STAGE_B + 4 * TILE_B) + par_c * 16;
        const float2* nd2 = nl2 + 32;
        uint32_t sv[32], dp[32];
        tmem_ld16x64b_x32(tl + TM_S, sv);
        tmem_ld16x64b_x32(tl + TM_DP, dp);
        tmem_ld_wait();
        const float2 cc = make_float2(c2, c2);
        const uint32_t perm = pair_perm(par_c);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          const float2 arg =
              __ffma2_rn(make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1])), cc, nl2[i2]);
          const float2 p = make_float2(ex2(arg.x), ex2(arg.y));
          const float2 ds = __fmul2_rn(
              p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * i2]), __uint_as_float(dp[2 * i2 + 1])), nd2[i2]));
          pk[i2] = pair_pack_bf16(p.x, p.y, perm);
          dk[i2] = pair_pack_bf16(ds.x, ds.y, perm);
        }
        tmem_st16x64b_x16(tl + TM_S, pk);
        tmem_st16x64b_x16(tl + TM_DP, dk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.pfull[s]);
      }
      mbar_wait(&B.bdone[s], (g - 1) & 1, abort, ctx);
      tc_fence_after();
      uint32_t o[64];
      tmem_ld16x64b_x64(tl + TM_DV, o);
      tmem_ld_wait();
      store_row_f32(dvd, o, 1.f, par_c);
      tmem_ld16x64b_x64(tl + TM_DK, o);
      tmem_ld_wait();
      store_row_f32(dkd, o, scale, par_c);
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

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                       uint32_t box_rows);

vsa2_status attn_bwd_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, const int32_t* kv_off, const int32_t* kv_idx, const int32_t* q_off,
                        const int32_t* q_idx, float* dq, float* dk, float* dv, int topk, char* ws, cudaStream_t s) {
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
  cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::SMEM_DYN);
  attn_bwd_dq_tc_kernel<<<grid, BT, dqk::SMEM_DYN, s>>>(
      tk, tv, (const __nv_bfloat16*)q, (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, lse, ndelta, nlse2, kv_off,
      kv_idx, dq, d.N, (int)d.L, topk, items, c2, c1, ctx);
  if (check_launch("attn_bwd_dq_tc_kernel") != VSA2_OK) return VSA2_ERR_CUDA;
  cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM_DYN);
  attn_bwd_dkdv_tc_kernel<<<grid, BT, dkv::SMEM_DYN, s>>>(tq, tdo, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                                          nlse2, ndelta, q_off, q_idx, dk, dv, d.N, (int)d.L, topk,
                                                          items, c2, c1, ctx);
  return check_launch("attn_bwd_dkdv_tc_kernel");
}

}  // namespace vsa2
