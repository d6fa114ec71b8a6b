// Block-sparse attention forward on tcgen05 (bf16 in, fp32 accumulate), head_dim 128.
// Eq. 12 of "Improving Video Sparse Attention with Fine-grained Router and Sparse Rebasing",
// with the attention definition of its §2.1: per query tile, softmax over the tokens of the
// KV tiles its router selected.
//
// Shape choice for sm_100a: a query tile has only 64 rows, and tcgen05 runs M=64 at half
// rate, so both GEMMs are issued transposed with M=128:
//   S^T[128 kv, 64 q]  = [K_j1; K_j2] . Q_i^T     (two selected KV tiles per block)
//   O^T[128 d, 64 q]  += [V_j1; V_j2]^T . P^T      (V^T read MN-major straight from the TMA tile)
// The softmax runs down the columns of S^T: each thread owns one KV row and keeps 64 partial
// row sums; the running max per query column is shared through shared memory and is only
// raised (with an O^T rescale) when a new score exceeds it by more than 2^8.
//
// CTA: two query-tile slots in flight. Warps 0-3 = softmax of slot 0, warps 4-7 = slot 1,
// warp 8 = TMA producer, warp 9 = MMA issuer. TMEM: per slot two S^T buffers (64 columns
// each) and one O^T accumulator (64 columns).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int FT = 320;            // threads per CTA
constexpr int KST = 2, VST = 2;    // K and V ring stages (one block = 2 tiles = 32 KB each)
constexpr uint32_t TILE_B = 8192;  // one 64x64 bf16 box (64 rows x 128 B)
constexpr uint32_t Q_B = 16384;    // Q tile: 2 column halves
constexpr uint32_t BLK_B = 32768;  // K or V block: [half0: tile A, tile B][half1: tile A, tile B]
constexpr uint32_t PT_B = 16384;   // P^T: 128 kv rows x 64 q (bf16), MN-major 128B swizzle

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + 2 * Q_B;
constexpr uint32_t OFF_V = OFF_K + KST * BLK_B;
constexpr uint32_t OFF_P = OFF_V + VST * BLK_B;
constexpr uint32_t OFF_BAR = OFF_P + 2 * PT_B;  // mbarriers
constexpr int NBAR = 2 * KST + 2 * VST + 4 /*q*/ + 8 /*s*/ + 6 /*p,o*/ + 1;
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 32;
// misc: m[2][64], red[2][4][64], alpha[2][64], inv_l[2][64], flags
constexpr uint32_t OFF_M = OFF_MISC;
constexpr uint32_t OFF_RED = OFF_M + 2 * 64 * 4;
constexpr uint32_t OFF_ALPHA = OFF_RED + 2 * 4 * 64 * 4;
constexpr uint32_t OFF_FLAG = OFF_ALPHA + 2 * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_FLAG + 64;
constexpr uint32_t SMEM_DYN = SMEM_USED + 1024;

constexpr float kThresh = 8.0f;  // log2 headroom before the running max must move

struct Bars {
  uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  uint64_t qfull[2], qempty[2];
  uint64_t sfull[2][2], sfree[2][2];
  uint64_t pfull[2], odone[2], ofree[2];
  uint64_t done;
};
static_assert(sizeof(Bars) <= 8 * 32, "barrier area");

// Sanitised CSR row of query tile i of head bh; both producer and consumers read it the same way.
struct Row {
  int beg, len;
};
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

// Deterministic per-slot op stream: for a tile with n blocks, S0, S1, O0, S2, O1, ..., O(n-1).
// Items are (bh, query tile) in head-major order; CTA c slot s takes items r*2G + 2c + s.
struct SlotSeq {
  int item, items_total, stride;
  int bh, qt, nblk, len, beg;
  int s_next, o_next;
  int tiles_done;    // non-empty tiles started before the current one
  bool active;

  __device__ void init(int first, int total, int step) {
    item = first - step;
    items_total = total;
    stride = step;
    tiles_done = -1;
    nblk = 0;
    s_next = o_next = 0;
    active = true;
  }
};

__device__ __forceinline__ uint32_t u32(float f) { return __float_as_uint(f); }

// 64-column reduce-scatter across a warp: afterwards lane l holds columns 2l and 2l+1.
template <bool MAX>
__device__ __forceinline__ void warp_rs64(float (&v)[64], const int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 32 >> step;  // values kept after this step
    const int mask = 16 >> step;
    const bool hi = lane & mask;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = hi ? v[j] : v[half + j];
      const float keep = hi ? v[half + j] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, mask);
      v[j] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

__global__ void __launch_bounds__(FT, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ kv_off,
                       const int32_t* __restrict__ kv_idx, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                       int N, int L, int topk, int items, float c2, DevCtx ctx) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  float* m_sh = reinterpret_cast<float*>(dsm + OFF_M);         // [2][64]
  float* red_sh = reinterpret_cast<float*>(dsm + OFF_RED);     // [2][4][64]
  float* alpha_sh = reinterpret_cast<float*>(dsm + OFF_ALPHA); // [2][64]
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);       // [0] abort, [1..2] wg fail, [4] tmem base
  volatile int* abort = flag_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;
  const int step = 2 * gridDim.x;

  if (threadIdx.x == 0) {
    flag_sh[0] = flag_sh[1] = flag_sh[2] = 0;
    for (int i = 0; i < KST; ++i) mbar_init(&B.kfull[i], 1), mbar_init(&B.kempty[i], 1);
    for (int i = 0; i < VST; ++i) mbar_init(&B.vfull[i], 1), mbar_init(&B.vempty[i], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.qfull[s], 1);
      mbar_init(&B.qempty[s], 1);
      for (int b = 0; b < 2; ++b) mbar_init(&B.sfull[s][b], 1), mbar_init(&B.sfree[s][b], 4);
      mbar_init(&B.pfull[s], 4);
      mbar_init(&B.odone[s], 1);
      mbar_init(&B.ofree[s], 4);
    }
    mbar_init(&B.done, 1);
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

  // next op of a slot's stream; returns 0 = none, 1 = S, 2 = O; *blk = block index in the tile
  auto next_op = [&](SlotSeq& q, int* blk, bool* tile_start, bool report) -> int {
    while (true) {
      if (!q.active) return 0;
      if (q.s_next < q.nblk && q.s_next <= q.o_next + 1) {
        *blk = q.s_next++;
        *tile_start = (*blk == 0);
        return 1;
      }
      if (q.o_next < q.nblk) {
        *blk = q.o_next++;
        *tile_start = false;
        return 2;
      }
      // advance to the next non-empty tile
      q.item += q.stride;
      if (q.item >= q.items_total) {
        q.active = false;
        return 0;
      }
      q.bh = q.item / N;
      q.qt = q.item - q.bh * N;
      Row r = load_row(kv_off, q.bh, q.qt, N, cap, ctx, report);
      q.len = r.len;
      q.beg = r.beg;
      q.nblk = (r.len + 1) >> 1;
      q.s_next = q.o_next = 0;
      if (q.nblk > 0) q.tiles_done++;
    }
  };

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      SlotSeq sq[2];
      sq[0].init(2 * blockIdx.x, items, step);
      sq[1].init(2 * blockIdx.x + 1, items, step);
      int kc = 0, vc = 0, qc[2] = {0, 0};
      int last_k[KST], last_v[VST];
      for (int i = 0; i < KST; ++i) last_k[i] = -1;
      for (int i = 0; i < VST; ++i) last_v[i] = -1;
      bool ok = true;
      while (ok && (sq[0].active || sq[1].active)) {
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (!ok) break;
          int blk;
          bool start;
          const int op = next_op(sq[s], &blk, &start, false);
          if (op == 0) continue;
          SlotSeq& q = sq[s];
          const int row0 = q.bh * L;  // first row of this head in the [BH*L, D] view
          const int ntile = min(2, q.len - 2 * blk);
          int jt[2] = {0, 0};
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (t >= ntile) break;
            int j = kv_idx[(size_t)q.bh * cap + q.beg + 2 * blk + t];
            if (j < 0 || j >= N) {
              if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
              j = j < 0 ? 0 : N - 1;
            }
            jt[t] = j;
          }
          if (op == 1) {
            if (start) {
              if (!(ok = mbar_wait(&B.qempty[s], (qc[s] & 1) ^ 1, abort, ctx))) break;
              mbar_arrive_expect_tx(&B.qfull[s], Q_B);
              for (int h = 0; h < 2; ++h)
                tma_load_2d(dsm + OFF_Q + s * Q_B + h * TILE_B, &tm_q, h * 64, row0 + q.qt * 64, &B.qfull[s]);
              qc[s]++;
            }
            const int st = kc % KST;
            if (!(ok = mbar_wait(&B.kempty[st], ((kc / KST) & 1) ^ 1, abort, ctx))) break;
            mbar_arrive_expect_tx(&B.kfull[st], ntile * 2 * TILE_B);
#pragma unroll
            for (int t = 0; t < 2; ++t)
              for (int h = 0; h < 2 && t < ntile; ++h)
                tma_load_2d(dsm + OFF_K + st * BLK_B + h * 2 * TILE_B + t * TILE_B, &tm_k, h * 64,
                            row0 + jt[t] * 64, &B.kfull[st]);
            last_k[st] = kc++;
          } else {
            const int st = vc % VST;
            if (!(ok = mbar_wait(&B.vempty[st], ((vc / VST) & 1) ^ 1, abort, ctx))) break;
            mbar_arrive_expect_tx(&B.vfull[st], ntile * 2 * TILE_B);
#pragma unroll
            for (int t = 0; t < 2; ++t)
              for (int h = 0; h < 2 && t < ntile; ++h)
                tma_load_2d(dsm + OFF_V + st * BLK_B + h * 2 * TILE_B + t * TILE_B, &tm_v, h * 64,
                            row0 + jt[t] * 64, &B.vfull[st]);
            last_v[st] = vc++;
          }
        }
      }
      if (*abort) {  // let copies still in flight land before the CTA exits
        for (int i = 0; i < KST; ++i)
          if (last_k[i] >= 0) mbar_wait_drain(&B.kfull[i], (last_k[i] / KST) & 1, ctx.timeout_ns);
        for (int i = 0; i < VST; ++i)
          if (last_v[i] >= 0) mbar_wait_drain(&B.vfull[i], (last_v[i] / VST) & 1, ctx.timeout_ns);
        for (int s = 0; s < 2; ++s)
          if (qc[s] > 0) mbar_wait_drain(&B.qfull[s], (qc[s] - 1) & 1, ctx.timeout_ns);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, 64, true, true);
      SlotSeq sq[2];
      sq[0].init(2 * blockIdx.x, items, step);
      sq[1].init(2 * blockIdx.x + 1, items, step);
      int kc = 0, vc = 0, qc[2] = {0, 0}, sb[2] = {0, 0}, ob[2] = {0, 0};
      bool ok = true;
      while (ok && (sq[0].active || sq[1].active)) {
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (!ok) break;
          int blk;
          bool start;
          const int op = next_op(sq[s], &blk, &start, false);
          if (op == 0) continue;
          SlotSeq& q = sq[s];
          const bool half = (2 * blk + 1 == q.len);
          const uint32_t tslot = tmem + s * 192;
          if (op == 1) {
            if (start) {
              if (!(ok = mbar_wait(&B.qfull[s], qc[s] & 1, abort, ctx))) break;
              qc[s]++;
            }
            const int st = kc % KST;
            if (!(ok = mbar_wait(&B.kfull[st], (kc / KST) & 1, abort, ctx))) break;
            const int buf = sb[s] & 1;
            if (!(ok = mbar_wait(&B.sfree[s][buf], ((sb[s] >> 1) & 1) ^ 1, abort, ctx))) break;
            tc_fence_after();
            const uint32_t ka = smem_u32(dsm + OFF_K + st * BLK_B);
            const uint32_t qa = smem_u32(dsm + OFF_Q + s * Q_B);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t h = kk >> 2, sub = (kk & 3) * 32;
              mma_bf16_ss(tslot + buf * 64, sdesc_sw128(ka + h * 2 * TILE_B + sub, 16, 1024),
                          sdesc_sw128(qa + h * TILE_B + sub, 16, 1024), id_s, kk > 0);
            }
            mma_commit(&B.kempty[st]);
            mma_commit(&B.sfull[s][buf]);
            if (blk == q.nblk - 1) mma_commit(&B.qempty[s]);
            kc++;
            sb[s]++;
          } else {
            if (blk == 0 && q.tiles_done > 0) {
              if (!(ok = mbar_wait(&B.ofree[s], (q.tiles_done - 1) & 1, abort, ctx))) break;
            }
            const int st = vc % VST;
            if (!(ok = mbar_wait(&B.vfull[st], (vc / VST) & 1, abort, ctx))) break;
            if (!(ok = mbar_wait(&B.pfull[s], ob[s] & 1, abort, ctx))) break;
            tc_fence_after();
            const uint32_t va = smem_u32(dsm + OFF_V + st * BLK_B);
            const uint32_t pa = smem_u32(dsm + OFF_P + s * PT_B);
            const int ksteps = half ? 4 : 8;
            for (int kk = 0; kk < ksteps; ++kk) {
              mma_bf16_ss(tslot + 128, sdesc_sw128(va + kk * 2048, 2 * TILE_B, 1024),
                          sdesc_sw128(pa + kk * 2048, PT_B, 1024), id_o, (blk > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&B.vempty[st]);
            mma_commit(&B.odone[s]);
            vc++;
            ob[s]++;
          }
        }
      }
      mma_commit(&B.done);
      mbar_wait_drain(&B.done, 0, ctx.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------------ softmax, slot s
    const int s = warp >> 2;
    const int wq = warp & 3;
    const int tid = threadIdx.x & 127;
    const int bar_id = 1 + s;
    float* m_s = m_sh + s * 64;
    float* red = red_sh + s * 256;
    float* alpha = alpha_sh + s * 64;
    volatile int* wfail = flag_sh + 1 + s;
    const uint32_t tslot = tmem + s * 192 + ((uint32_t)(32 * wq) << 16);
    const uint32_t pt = smem_u32(dsm + OFF_P + s * PT_B);
    uint8_t* pt_ptr = dsm + OFF_P + s * PT_B;
    int gb = 0;  // blocks processed by this slot (S buffer / phase counter)
    // wait by one thread, decision shared by the whole warpgroup
    auto wg_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (tid == 0) *wfail = mbar_wait(bar, parity, abort, ctx) ? 0 : 1;
      named_bar_sync(bar_id, 128);
      const bool ok = *wfail == 0;
      named_bar_sync(bar_id, 128);
      return ok;
    };
    bool ok = true;
    for (int item = 2 * blockIdx.x + s; ok && item < items; item += step) {
      const int bh = item / N, qt = item - bh * N;
      const Row row = load_row(kv_off, bh, qt, N, cap, ctx, tid == 0);
      const int nblk = (row.len + 1) >> 1;
      const size_t tok0 = (size_t)bh * L + (size_t)qt * 64;
      if (nblk == 0) {
        uint4* o4 = reinterpret_cast<uint4*>(out + tok0 * 128);
        for (int e = tid; e < 64 * 128 / 8; e += 128) o4[e] = make_uint4(0, 0, 0, 0);
        if (tid < 64) lse[tok0 + tid] = -INFINITY;
        continue;
      }
      if (tid < 64) m_s[tid] = -INFINITY;
      float lpart[64];
#pragma unroll
      for (int q = 0; q < 64; ++q) lpart[q] = 0.f;
      named_bar_sync(bar_id, 128);
      for (int n = 0; n < nblk; ++n, ++gb) {
        const bool valid_row = !(2 * n + 1 == row.len && tid >= 64);
        const int buf = gb & 1;
        if (!(ok = wg_wait(&B.sfull[s][buf], (gb >> 1) & 1))) break;
        tc_fence_after();
        uint32_t ra[32], rb[32];
        float tmax = -INFINITY;
        tmem_ld32(tslot + buf * 64, ra);
        tmem_ld32(tslot + buf * 64 + 32, rb);
        tmem_ld_wait();
#define RV(q) __uint_as_float((q) < 32 ? ra[(q) & 31] : rb[(q) & 31])
        if (valid_row) {
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 mv = reinterpret_cast<const float4*>(m_s)[q4];
            tmax = fmaxf(tmax, fmaf(RV(4 * q4 + 0), c2, -mv.x));
            tmax = fmaxf(tmax, fmaf(RV(4 * q4 + 1), c2, -mv.y));
            tmax = fmaxf(tmax, fmaf(RV(4 * q4 + 2), c2, -mv.z));
            tmax = fmaxf(tmax, fmaf(RV(4 * q4 + 3), c2, -mv.w));
          }
        }
        const bool rescale = named_bar_or(bar_id, 128, tmax > kThresh);
        if (rescale) {
          // column max of this block over all 128 kv rows, then raise the running max
          float v[64];
#pragma unroll
          for (int q = 0; q < 64; ++q) v[q] = valid_row ? RV(q) * c2 : -INFINITY;
          warp_rs64<true>(v, lane);
          red[wq * 64 + 2 * lane] = v[0];
          red[wq * 64 + 2 * lane + 1] = v[1];
          named_bar_sync(bar_id, 128);
          if (tid < 64) {
            const float cm = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
            const float mo = m_s[tid];
            const float mn = fmaxf(mo, cm);
            alpha[tid] = mo == -INFINITY ? 0.f : ex2(mo - mn);
            m_s[tid] = mn;
          }
          named_bar_sync(bar_id, 128);
#pragma unroll
          for (int q = 0; q < 64; ++q) lpart[q] *= alpha[q];
          if (n > 0) {
            // O^T holds blocks 0..n-1: wait for the last one, then scale its columns
            if (!(ok = wg_wait(&B.odone[s], (gb - 1) & 1))) break;
            tc_fence_after();
            uint32_t o[32];
#pragma unroll
            for (int hcol = 0; hcol < 2; ++hcol) {
              tmem_ld32(tslot + 128 + hcol * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] = u32(__uint_as_float(o[q]) * alpha[hcol * 32 + q]);
              tmem_st32(tslot + 128 + hcol * 32, o);
            }
            tmem_st_wait();
          }
          // the S values were consumed by the reduction above; read them again
          tmem_ld32(tslot + buf * 64, ra);
          tmem_ld32(tslot + buf * 64 + 32, rb);
          tmem_ld_wait();
        }
        // probabilities (log2 domain, <= 2^8), partial row sums, bf16 pack
        uint32_t pk[32];
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 mv = reinterpret_cast<const float4*>(m_s)[q4];
          float p0 = ex2(fmaf(RV(4 * q4 + 0), c2, -mv.x));
          float p1 = ex2(fmaf(RV(4 * q4 + 1), c2, -mv.y));
          float p2 = ex2(fmaf(RV(4 * q4 + 2), c2, -mv.z));
          float p3 = ex2(fmaf(RV(4 * q4 + 3), c2, -mv.w));
          if (!valid_row) p0 = p1 = p2 = p3 = 0.f;
          lpart[4 * q4 + 0] += p0;
          lpart[4 * q4 + 1] += p1;
          lpart[4 * q4 + 2] += p2;
          lpart[4 * q4 + 3] += p3;
          pk[2 * q4] = pack_bf16(p0, p1);
          pk[2 * q4 + 1] = pack_bf16(p2, p3);
        }
        // P^T buffer is free once O of the previous block has finished
        if (n > 0) {
          if (!(ok = wg_wait(&B.odone[s], (gb - 1) & 1))) break;
        }
        if (valid_row) {
          const uint32_t rowaddr = pt + tid * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(rowaddr + ((c ^ (tid & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
#undef RV
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.sfree[s][buf]);
          mbar_arrive(&B.pfull[s]);
        }
      }
      if (!ok) break;
      // ---- epilogue: wait for the last O block, finish the row sums, normalise, store
      if (!(ok = wg_wait(&B.odone[s], (gb - 1) & 1))) break;
      tc_fence_after();
      warp_rs64<false>(lpart, lane);
      red[wq * 64 + 2 * lane] = lpart[0];
      red[wq * 64 + 2 * lane + 1] = lpart[1];
      named_bar_sync(bar_id, 128);
      if (tid < 64) {
        const float l = (red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]);
        alpha[tid] = 1.f / l;
        lse[tok0 + tid] = (m_s[tid] + __log2f(l)) * 0.6931471805599453f;
      }
      named_bar_sync(bar_id, 128);
      {
        // thread tid owns O^T row d = tid; write O[q][d] into the (now free) P^T buffer
        uint32_t o[32];
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(pt_ptr);
#pragma unroll
        for (int hcol = 0; hcol < 2; ++hcol) {
          tmem_ld32(tslot + 128 + hcol * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q)
            stage[(hcol * 32 + q) * 128 + tid] = __float2bfloat16_rn(__uint_as_float(o[q]) * alpha[hcol * 32 + q]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.ofree[s]);
      fence_proxy_async_smem();
      named_bar_sync(bar_id, 128);
      if (tid == 0) {
        bulk_store(out + tok0 * 128, pt_ptr, 64 * 128 * 2);
        bulk_commit();
        bulk_wait_read0();
      }
      named_bar_sync(bar_id, 128);
    }
    if (tid == 0) bulk_wait0();
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

vsa2_status attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v, int topk, const int32_t* kv_off,
                        const int32_t* kv_idx, void* o, float* lse, char* ws, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tq, q, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tk, k, 128, rows, 64, 64) ||
      !make_tmap_2d_bf16(&tv, v, 128, rows, 64, 64))
    return cuda_fail("tensor map encoding for the attention operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(sms, (items + 1) / 2);
  const float c2 = 1.4426950408889634f / sqrtf(128.f);
  cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  attn_fwd_tc_kernel<<<grid, FT, SMEM_DYN, s>>>(tq, tk, tv, kv_off, kv_idx, (__nv_bfloat16*)o, lse, d.N, (int)d.L,
                                                topk, items, c2, ctx);
  return check_launch(__func__);
}

}  // namespace vsa2
