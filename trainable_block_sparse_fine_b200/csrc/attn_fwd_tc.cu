// Block-sparse attention forward on tcgen05 (bf16 in, fp32 accumulate), head_dim 128.
// Eq. 12 of "Improving Video Sparse Attention with Fine-grained Router and Sparse Rebasing",
// with the attention definition of its §2.1: per query tile, softmax over the tokens of the
// KV tiles its router selected.
//
// Shape choice for sm_100a: a query tile has only 64 rows, and tcgen05 runs M=64 at half
// rate, so both GEMMs are issued transposed with M=128:
//   S^T[128 kv, 64 q]  = [K_j1; K_j2] . Q_i^T     (two selected KV tiles per block)
//   O^T[128 d, 64 q]  += [V_j1; V_j2]^T . P^T      (V^T read MN-major straight from the TMA tile)
// The softmax runs down the columns of S^T: each thread owns one KV row; the running max per
// query column lives in shared memory and is only raised (with an O^T rescale) when a new score
// exceeds it by more than 2^8, so the common block needs a single warpgroup barrier.
//
// CTA (persistent, one query tile at a time): warps 0-3 and 4-7 are two softmax warpgroups that
// split the 64 query columns (32 each); warp 8 loads Q and K, warp 10 loads V (two TMA issuing
// threads keep more copies in flight than one), warp 9 issues the MMAs.
// Double buffers: Q (per tile), S^T and P^T (per block), O^T (per tile, so the epilogue of one
// tile overlaps the first MMAs of the next). K and V rings of two blocks each.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int FT = 352;            // 11 warps
constexpr uint32_t TILE_B = 8192;  // one 64x64 bf16 box (64 rows x 128 B)
constexpr uint32_t Q_B = 16384;    // Q tile: 2 column halves of 64 rows
constexpr uint32_t BLK_B = 32768;  // K or V block: [half0: tile A, tile B][half1: tile A, tile B]
constexpr uint32_t PT_B = 16384;   // P^T: 128 kv rows x 64 q (bf16), MN-major 128B swizzle
constexpr uint32_t ST_B = 8192;    // output staging per warpgroup: 32 rows x 128 bf16

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + 2 * Q_B;
constexpr uint32_t OFF_V = OFF_K + 2 * BLK_B;
constexpr uint32_t OFF_P = OFF_V + 2 * BLK_B;
constexpr uint32_t OFF_ST = OFF_P + 2 * PT_B;
constexpr uint32_t OFF_BAR = OFF_ST + 2 * ST_B;
constexpr uint32_t OFF_M = OFF_BAR + 256;                 // [2 wg][32] running max (log2 units)
constexpr uint32_t OFF_RED = OFF_M + 2 * 32 * 4;          // [2 wg][4 warps][32]
constexpr uint32_t OFF_ALPHA = OFF_RED + 2 * 4 * 32 * 4;  // [2 wg][32]
constexpr uint32_t OFF_FLAG = OFF_ALPHA + 2 * 32 * 4;
constexpr uint32_t SMEM_USED = OFF_FLAG + 64;
constexpr uint32_t SMEM_DYN = SMEM_USED + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");

constexpr uint32_t TM_COLS = 256;  // S^T at columns 0 / 64, O^T at 128 / 192
constexpr float kThresh = 8.0f;    // log2 headroom before the running max must move

struct Bars {
  uint64_t kfull[2], kempty[2], vfull[2], vempty[2];
  uint64_t qfull[2], qempty[2];
  uint64_t sfull[2], sfree[2], pfull[2], odone[2], ofree[2];
  uint64_t done;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

// Sanitised CSR row of query tile i of head bh; every role reads it the same way.
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

__device__ __forceinline__ uint32_t u32(float f) { return __float_as_uint(f); }

// 32-column reduce-scatter across a warp: afterwards lane l holds column l.
template <bool MAX>
__device__ __forceinline__ float warp_rs32(float (&v)[32], const int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step;
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
  return v[0];
}

// Phase parity of the n-th completion of a barrier used by every other block (double buffers).
__device__ __forceinline__ uint32_t par(int n) { return (uint32_t)((n >> 1) & 1); }

__global__ void __launch_bounds__(FT, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ kv_off,
                       const int32_t* __restrict__ kv_idx, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                       int N, int L, int topk, int items, float c2, DevCtx ctx) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);  // [0] abort, [4] tmem base
  volatile int* abort = flag_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.kfull[i], 1), mbar_init(&B.kempty[i], 1);
      mbar_init(&B.vfull[i], 1), mbar_init(&B.vempty[i], 1);
      mbar_init(&B.qfull[i], 1), mbar_init(&B.qempty[i], 1);
      mbar_init(&B.sfull[i], 1), mbar_init(&B.sfree[i], 8);
      mbar_init(&B.pfull[i], 8), mbar_init(&B.odone[i], 1);
      mbar_init(&B.ofree[i], 8);
    }
    mbar_init(&B.done, 1);
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

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------------ TMA producers
    const bool k_role = warp == 8;
    if (lane == 0) {
      tma_prefetch_desc(k_role ? &tm_k : &tm_v);
      if (k_role) tma_prefetch_desc(&tm_q);
      int t = 0, g = 0;
      int last = -1, last_q = -1;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const int bh = item / N, qt = item - bh * N;
        const Row row = load_row(kv_off, bh, qt, N, cap, ctx, false);
        const int nblk = (row.len + 1) >> 1;
        if (nblk == 0) continue;
        const int row0 = bh * L;
        if (k_role) {
          const int qb = t & 1;
          if (!(ok = mbar_wait(&B.qempty[qb], par(t) ^ 1, abort, ctx))) break;
          mbar_arrive_expect_tx(&B.qfull[qb], Q_B);
          for (int h = 0; h < 2; ++h)
            tma_load_2d(dsm + OFF_Q + qb * Q_B + h * TILE_B, &tm_q, h * 64, row0 + qt * 64, &B.qfull[qb]);
          last_q = t;
        }
        const int32_t* idx = kv_idx + (size_t)bh * cap + row.beg;
        for (int n = 0; n < nblk; ++n, ++g) {
          const int st = g & 1;
          const int ntile = min(2, row.len - 2 * n);
          uint64_t* empty = k_role ? &B.kempty[st] : &B.vempty[st];
          uint64_t* full = k_role ? &B.kfull[st] : &B.vfull[st];
          const CUtensorMap* map = k_role ? &tm_k : &tm_v;
          uint8_t* dst = dsm + (k_role ? OFF_K : OFF_V) + st * BLK_B;
          if (!(ok = mbar_wait(empty, par(g) ^ 1, abort, ctx))) break;
          mbar_arrive_expect_tx(full, ntile * 2 * TILE_B);
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            if (tt >= ntile) break;
            int j = idx[2 * n + tt];
            if (j < 0 || j >= N) {
              if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
              j = j < 0 ? 0 : N - 1;
            }
            tma_load_2d(dst + tt * TILE_B, map, 0, row0 + j * 64, full);
            tma_load_2d(dst + 2 * TILE_B + tt * TILE_B, map, 64, row0 + j * 64, full);
          }
          last = g;
        }
        ++t;
      }
      if (*abort) {  // let copies still in flight land before the CTA exits
        for (int gg = max(0, last - 1); gg <= last; ++gg)
          mbar_wait_drain(k_role ? &B.kfull[gg & 1] : &B.vfull[gg & 1], par(gg), ctx.timeout_ns);
        if (last_q >= 0) mbar_wait_drain(&B.qfull[last_q & 1], par(last_q), ctx.timeout_ns);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, 64, true, true);
      int t = 0, g0 = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const int bh = item / N, qt = item - bh * N;
        const Row row = load_row(kv_off, bh, qt, N, cap, ctx, false);
        const int nblk = (row.len + 1) >> 1;
        if (nblk == 0) continue;
        const int qb = t & 1;
        const uint32_t qa = smem_u32(dsm + OFF_Q + qb * Q_B);
        const uint32_t o_acc = tmem + 128 + (t & 1) * 64;
        if (!(ok = mbar_wait(&B.qfull[qb], par(t), abort, ctx))) break;
        int s_next = 0, o_next = 0;
        while (ok && o_next < nblk) {
          if (s_next < nblk && s_next <= o_next + 1) {
            const int g = g0 + s_next;
            if (!(ok = mbar_wait(&B.kfull[g & 1], par(g), abort, ctx))) break;
            if (!(ok = mbar_wait(&B.sfree[g & 1], par(g) ^ 1, abort, ctx))) break;
            tc_fence_after();
            const uint32_t ka = smem_u32(dsm + OFF_K + (g & 1) * BLK_B);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t h = kk >> 2, sub = (kk & 3) * 32;
              mma_bf16_ss(tmem + (g & 1) * 64, sdesc_sw128(ka + h * 2 * TILE_B + sub, 16, 1024),
                          sdesc_sw128(qa + h * TILE_B + sub, 16, 1024), id_s, kk > 0);
            }
            mma_commit(&B.kempty[g & 1]);
            mma_commit(&B.sfull[g & 1]);
            if (s_next == nblk - 1) mma_commit(&B.qempty[qb]);
            ++s_next;
          } else {
            const int n = o_next, g = g0 + n;
            if (n == 0 && !(ok = mbar_wait(&B.ofree[t & 1], par(t) ^ 1, abort, ctx))) break;
            if (!(ok = mbar_wait(&B.vfull[g & 1], par(g), abort, ctx))) break;
            if (!(ok = mbar_wait(&B.pfull[g & 1], par(g), abort, ctx))) break;
            tc_fence_after();
            const uint32_t va = smem_u32(dsm + OFF_V + (g & 1) * BLK_B);
            const uint32_t pa = smem_u32(dsm + OFF_P + (g & 1) * PT_B);
            const int ksteps = (2 * n + 1 == row.len) ? 4 : 8;
            for (int kk = 0; kk < ksteps; ++kk)
              mma_bf16_ss(o_acc, sdesc_sw128(va + kk * 2048, 2 * TILE_B, 1024), sdesc_sw128(pa + kk * 2048, PT_B, 1024),
                          id_o, (n > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&B.vempty[g & 1]);
            mma_commit(&B.odone[g & 1]);
            ++o_next;
          }
        }
        g0 += nblk;
        ++t;
      }
      mma_commit(&B.done);
      mbar_wait_drain(&B.done, 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = warp >> 2;   // warpgroup: query columns 32w .. 32w+31
    const int wq = warp & 3;   // TMEM lane quarter
    const int tid = threadIdx.x & 127;
    const int bar_id = 1 + w;
    float* m_s = reinterpret_cast<float*>(dsm + OFF_M) + w * 32;
    float* red = reinterpret_cast<float*>(dsm + OFF_RED) + w * 128;
    float* alpha = reinterpret_cast<float*>(dsm + OFF_ALPHA) + w * 32;
    uint8_t* stage = dsm + OFF_ST + w * ST_B;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    int t = 0, g = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int bh = item / N, qt = item - bh * N;
      const Row row = load_row(kv_off, bh, qt, N, cap, ctx, tid == 0 && w == 0);
      const int nblk = (row.len + 1) >> 1;
      const size_t tok0 = (size_t)bh * L + (size_t)qt * 64 + 32 * w;  // this warpgroup's 32 query rows
      if (nblk == 0) {
        uint4* o4 = reinterpret_cast<uint4*>(out + tok0 * 128);
        for (int e = tid; e < 32 * 128 / 8; e += 128) o4[e] = make_uint4(0, 0, 0, 0);
        if (tid < 32) lse[tok0 + tid] = -INFINITY;
        continue;
      }
      const uint32_t o_acc = tmem + lane_off + 128 + (t & 1) * 64 + 32 * w;
      if (tid < 32) m_s[tid] = -INFINITY;
      float lpart[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) lpart[q] = 0.f;
      named_bar_sync(bar_id, 128);
      for (int n = 0; n < nblk; ++n, ++g) {
        const bool valid_row = !(2 * n + 1 == row.len && tid >= 64);
        const uint32_t s_addr = tmem + lane_off + (g & 1) * 64 + 32 * w;
        mbar_wait(&B.sfull[g & 1], par(g), abort, ctx);
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(s_addr, r);
        tmem_ld_wait();
        float tmax = -INFINITY;
        if (valid_row) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 mv = reinterpret_cast<const float4*>(m_s)[q4];
            tmax = fmaxf(tmax, fmaf(__uint_as_float(r[4 * q4 + 0]), c2, -mv.x));
            tmax = fmaxf(tmax, fmaf(__uint_as_float(r[4 * q4 + 1]), c2, -mv.y));
            tmax = fmaxf(tmax, fmaf(__uint_as_float(r[4 * q4 + 2]), c2, -mv.z));
            tmax = fmaxf(tmax, fmaf(__uint_as_float(r[4 * q4 + 3]), c2, -mv.w));
          }
        }
        if (named_bar_or(bar_id, 128, tmax > kThresh)) {
          // raise the running max of these 32 columns to the block's column max
          float v[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = valid_row ? __uint_as_float(r[q]) * c2 : -INFINITY;
          red[wq * 32 + lane] = warp_rs32<true>(v, lane);
          named_bar_sync(bar_id, 128);
          if (tid < 32) {
            const float cm = fmaxf(fmaxf(red[tid], red[32 + tid]), fmaxf(red[64 + tid], red[96 + tid]));
            const float mo = m_s[tid];
            const float mn = fmaxf(mo, cm);
            alpha[tid] = mo == -INFINITY ? 0.f : ex2(mo - mn);
            m_s[tid] = mn;
          }
          named_bar_sync(bar_id, 128);
#pragma unroll
          for (int q = 0; q < 32; ++q) lpart[q] *= alpha[q];
          if (n > 0) {
            // O^T holds blocks 0..n-1 of this tile: wait for the last, then scale our columns
            mbar_wait(&B.odone[(g - 1) & 1], par(g - 1), abort, ctx);
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(o_acc, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = u32(__uint_as_float(o[q]) * alpha[q]);
            tmem_st32(o_acc, o);
            tmem_st_wait();
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 mv = reinterpret_cast<const float4*>(m_s)[q4];
          float p0 = ex2(fmaf(__uint_as_float(r[4 * q4 + 0]), c2, -mv.x));
          float p1 = ex2(fmaf(__uint_as_float(r[4 * q4 + 1]), c2, -mv.y));
          float p2 = ex2(fmaf(__uint_as_float(r[4 * q4 + 2]), c2, -mv.z));
          float p3 = ex2(fmaf(__uint_as_float(r[4 * q4 + 3]), c2, -mv.w));
          if (!valid_row) p0 = p1 = p2 = p3 = 0.f;
          lpart[4 * q4 + 0] += p0;
          lpart[4 * q4 + 1] += p1;
          lpart[4 * q4 + 2] += p2;
          lpart[4 * q4 + 3] += p3;
          pk[2 * q4] = pack_bf16(p0, p1);
          pk[2 * q4 + 1] = pack_bf16(p2, p3);
        }
        // P^T buffer g&1 was last read by the O MMA of block g-2
        mbar_wait(&B.odone[g & 1], par(g) ^ 1, abort, ctx);
        if (valid_row) {
          const uint32_t rowaddr = smem_u32(dsm + OFF_P + (g & 1) * PT_B) + tid * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(rowaddr + (((4 * w + c) ^ (tid & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                         pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.sfree[g & 1]);
          mbar_arrive(&B.pfull[g & 1]);
        }
      }
      // ---- epilogue: wait for the last O block, finish the row sums, normalise, store
      mbar_wait(&B.odone[(g - 1) & 1], par(g - 1), abort, ctx);
      tc_fence_after();
      red[wq * 32 + lane] = warp_rs32<false>(lpart, lane);
      named_bar_sync(bar_id, 128);
      if (tid < 32) {
        const float l = (red[tid] + red[32 + tid]) + (red[64 + tid] + red[96 + tid]);
        alpha[tid] = 1.f / l;
        lse[tok0 + tid] = (m_s[tid] + __log2f(l)) * 0.6931471805599453f;
      }
      named_bar_sync(bar_id, 128);
      {
        // thread tid owns O^T row d = tid; O[q][d] for this warpgroup's 32 query rows
        uint32_t o[32];
        tmem_ld32(o_acc, o);
        tmem_ld_wait();
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(stage);
#pragma unroll
        for (int q = 0; q < 32; ++q) st[q * 128 + tid] = __float2bfloat16_rn(__uint_as_float(o[q]) * alpha[q]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.ofree[t & 1]);
      fence_proxy_async_smem();
      named_bar_sync(bar_id, 128);
      if (tid == 0) {
        bulk_store(out + tok0 * 128, stage, ST_B);
        bulk_commit();
        bulk_wait_read0();
      }
      ++t;
      // leave together if any wait of this CTA has expired
      if (named_bar_or(bar_id, 128, *abort != 0)) break;
    }
    if (tid == 0) bulk_wait0();
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
  const int grid = std::min(sms, items);
  const float c2 = 1.4426950408889634f / sqrtf(128.f);
  cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  attn_fwd_tc_kernel<<<grid, FT, SMEM_DYN, s>>>(tq, tk, tv, kv_off, kv_idx, (__nv_bfloat16*)o, lse, d.N, (int)d.L,
                                                topk, items, c2, ctx);
  return check_launch(__func__);
}

}  // namespace vsa2
