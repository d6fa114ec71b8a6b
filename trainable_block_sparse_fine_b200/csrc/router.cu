// Fine-grained router of VSA2 ("Improving Video Sparse Attention with Fine-grained Router and
// Sparse Rebasing", §2.2 Eq. 5-7 and Fig. 5): MeanPool_R of Q and K, then a fused two-pass
// kernel - pass 1 accumulates the log-sum-exp of every pooled query row over all pooled keys,
// pass 2 recomputes the logits, applies the softmax and pools G x G on chip, writing only the
// N x N tile scores.
#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

// ------------------------------------------------------------------------------------------
// MeanPool_R (Eq. 5): each pooled row is the mean of R consecutive cube-major rows (R = 16, or 8
// with 128-token tiles).
// One thread per (pooled row, 16-byte column chunk); 16 independent 16-byte loads per thread.
// ------------------------------------------------------------------------------------------
// With kMask (a padded grid), each mean runs over the sub-cube's real tokens only (tmask, the
// per-tile real-token masks); a sub-cube without one is written as zeros.
// With kCoarse (bf16, D = 128, R = 16: a tile's four sub-cubes are the 64 consecutive threads of
// a warp pair) the same read also gives the coarse branch's tile means (Eq. 1) over the tile's
// real tokens, written as row (b*h) * Lc + tile of qc / kc.
template <typename T, bool kMask, int R, bool kCoarse = false>
__global__ void __launch_bounds__(256) router_pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          T* __restrict__ qr, T* __restrict__ kr,
                                                          int64_t pooled_rows, int chunks_per_row,
                                                          const uint64_t* __restrict__ tmask, int Lr,
                                                          T* __restrict__ qc, T* __restrict__ kc, int Lc) {
  static_assert(!kCoarse || (sizeof(T) == 2 && R == 16), "tile means need 16 chunks per row and 4 sub-cubes");
  constexpr int EPC = 16 / sizeof(T);  // elements per 16-byte chunk
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per_tensor = pooled_rows * chunks_per_row;
  if (tid >= 2 * per_tensor) return;
  const bool is_k = tid >= per_tensor;
  const int64_t t = is_k ? tid - per_tensor : tid;
  const int64_t prow = t / chunks_per_row;
  const int chunk = (int)(t % chunks_per_row);
  const T* src = (is_k ? k : q) + (prow * R) * (int64_t)chunks_per_row * EPC + chunk * EPC;
  const int64_t stride = (int64_t)chunks_per_row * EPC;
  float acc[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
  uint32_t valid = 0xffffu;
  float inv = 1.f / R;
  if constexpr (kMask) {
    const int a = (int)(prow % Lr);
    valid = (uint32_t)(__ldg(tmask + (a >> 2)) >> (16 * (a & 3))) & 0xffffu;
    inv = valid ? 1.f / __popc(valid) : 0.f;
  }
  uint4 buf[R];
#pragma unroll
  for (int r = 0; r < R; ++r) buf[r] = __ldg(reinterpret_cast<const uint4*>(src + r * stride));
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (kMask && !((valid >> r) & 1u)) continue;
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&buf[r]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    } else {
      const float* f = reinterpret_cast<const float*>(&buf[r]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] += f[e];
    }
  }
  T* dst = (is_k ? kr : qr) + prow * stride + chunk * EPC;
  uint4 out;
  if constexpr (sizeof(T) == 2) {
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = pack_bf16(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  } else {
    float* o = reinterpret_cast<float*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = acc[e] * inv;
  }
  *reinterpret_cast<uint4*>(dst) = out;
  if constexpr (kCoarse) {
    // rows 4T .. 4T+3 of tile T are threads 64T + 16g + chunk (g < 4): lanes 0-15 / 16-31 of the
    // pair's two warps. (Each 64-thread group is active or inactive as a whole: pooled_rows is a
    // multiple of 4 and the block holds 256 threads.)
    __shared__ float part[4][16][EPC + 1];
    float cnt = kMask ? (float)__popc(valid) : (float)R;
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 16);
    const int pair = threadIdx.x >> 6;
    const bool upper = threadIdx.x & 32;
    const int lane = threadIdx.x & 31;
    if (upper && lane < 16) {
#pragma unroll
      for (int e = 0; e < EPC; ++e) part[pair][lane][e] = acc[e];
      part[pair][lane][EPC] = cnt;
    }
    named_bar_sync(1 + pair, 64);
    if (!upper && lane < 16) {
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] += part[pair][lane][e];
      cnt += part[pair][lane][EPC];
      const float ti = cnt > 0.f ? 1.f / cnt : 0.f;
      const int64_t bh = prow / Lr;
      const int tile = (int)(prow % Lr) >> 2;
      T* cdst = (is_k ? kc : qc) + ((bh * Lc + tile) * chunks_per_row + chunk) * EPC;
      uint4 co;
      uint32_t* o = reinterpret_cast<uint32_t*>(&co);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = pack_bf16(acc[2 * e] * ti, acc[2 * e + 1] * ti);
      *reinterpret_cast<uint4*>(cdst) = co;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Fused two-pass router scores on tcgen05 (bf16 Qr/Kr, fp32 accumulate in TMEM).
// CTA = 128 pooled query rows (32 query tiles) of one (b, h). Key chunks of 256 pooled keys
// (64 key tiles) stream through a 2-stage TMA ring; S = Qr Kr^T lands in one of two TMEM
// buffers (256 fp32 columns each).
// Warp roles: 0 = TMA producer, 1 = MMA issuer (+ TMEM owner), 2..9 = softmax/pool epilogue
// (warp w reads TMEM lanes 32*(w%4).., columns half (w-2)/4 of the chunk).
// ------------------------------------------------------------------------------------------
constexpr int RS_M = 128;
constexpr int RS_N = 256;
constexpr int RS_THREADS = 320;

template <int ND>  // ND = head_dim / 64
struct RouterSmem {
  static constexpr uint32_t kQBytes = 16384u * ND;   // 128 rows x 128 B per 64-column half
  static constexpr uint32_t kKBytes = 32768u * ND;   // 256 rows x 128 B per half
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQBytes;
  static constexpr uint32_t kTotal = kQBytes + 2 * kKBytes;
  // slack to align the base to 1024 B; at least 117 KB so that one CTA (and its 512 TMEM
  // columns) owns the SM
  static constexpr uint32_t kDyn = (kTotal + 1024 > 119808u) ? kTotal + 1024 : 119808u;
};

// Pooled key b is valid unless it lies past Lr or (kMask) its sub-cube holds no real token.
// Returns the validity of keys key0 .. key0+31 as a bit mask (the same in every lane).
template <bool kMask>
__device__ __forceinline__ uint32_t piece_keys(int key0, int Lr, const uint64_t* tmask) {
  const int lane = threadIdx.x & 31;
  const int b = key0 + lane;
  bool ok = b < Lr;
  if (kMask && ok) ok = ((__ldg(tmask + (b >> 2)) >> (16 * (b & 3))) & 0xffffu) != 0;
  return __ballot_sync(0xffffffffu, ok);
}

// kMask (a padded grid): pooled keys without a real token are masked in the softmax of Eq. 6,
// pooled query rows without one add nothing, and Eq. 7 averages over the tile's real query
// sub-cubes (rows still sum to 1).
// G is the number of sub-cubes per tile: 4 (64-token tiles, 16-token sub-cubes) or 16 (128-token
// tiles, 8-token sub-cubes, no padded grids).
template <int ND, bool kMask, int G>
__global__ void __launch_bounds__(RS_THREADS, 1)
    router_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            float* __restrict__ scores, int Lr, int N, float c2, const uint64_t* __restrict__ tmask,
                            DevCtx ctx) {
  using SL = RouterSmem<ND>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[2], bar_kempty[2], bar_sfull[2], bar_sfree[2], bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float m_half[2][RS_M], l_half[2][RS_M], lse_sh[RS_M];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int m0 = blockIdx.x * RS_M;
  const int nchunk = (Lr + RS_N - 1) / RS_N;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bar_q, 1);
    mbar_init(&bar_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_kfull[i], 1);
      mbar_init(&bar_kempty[i], 1);
      mbar_init(&bar_sfull[i], 1);
      mbar_init(&bar_sfree[i], 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort = &abort_sh;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(&bar_q, SL::kQBytes);
      for (int h = 0; h < ND; ++h) tma_load_3d(dsm + SL::kQOff + h * 16384, &tm_q, h * 64, m0, bh, &bar_q);
      int issued[2] = {-1, -1};
      for (int it = 0; it < 2 * nchunk; ++it) {
        const int st = it & 1, c = it % nchunk;
        if (!mbar_wait(&bar_kempty[st], ((it >> 1) & 1) ^ 1, abort, ctx)) break;
        mbar_arrive_expect_tx(&bar_kfull[st], SL::kKBytes);
        for (int h = 0; h < ND; ++h)
          tma_load_3d(dsm + SL::kKOff + st * SL::kKBytes + h * 32768, &tm_k, h * 64, c * RS_N, bh, &bar_kfull[st]);
        issued[st] = it;
      }
      if (*abort) {  // drain the copies still in flight before the CTA exits
        mbar_wait_drain(&bar_q, 0, ctx.timeout_ns);
        for (int st = 0; st < 2; ++st)
          if (issued[st] >= 0) mbar_wait_drain(&bar_kfull[st], (issued[st] >> 1) & 1, ctx.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(RS_M, RS_N, false, false);
      const uint32_t qa = smem_u32(dsm + SL::kQOff);
      bool ok = mbar_wait(&bar_q, 0, abort, ctx);
      for (int it = 0; ok && it < 2 * nchunk; ++it) {
        const int st = it & 1;
        if (!mbar_wait(&bar_kfull[st], (it >> 1) & 1, abort, ctx)) break;
        if (!mbar_wait(&bar_sfree[st], ((it >> 1) & 1) ^ 1, abort, ctx)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(dsm + SL::kKOff + st * SL::kKBytes);
#pragma unroll
        for (int kk = 0; kk < 4 * ND; ++kk) {
          const uint32_t h = kk >> 2, sub = (kk & 3) * 32;
          mma_bf16_ss(tmem + st * RS_N, sdesc_sw128(qa + h * 16384 + sub, 16, 1024),
                      sdesc_sw128(ka + h * 32768 + sub, 16, 1024), idesc, kk > 0);
        }
        mma_commit(&bar_kempty[st]);
        mma_commit(&bar_sfull[st]);
      }
      // every MMA issued above has finished once this barrier completes (also on abort)
      mma_commit(&bar_done);
      mbar_wait_drain(&bar_done, 0, ctx.timeout_ns);
    }
  } else {
    // epilogue warps
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const int row = 32 * quarter + lane;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    float m = -INFINITY, l = 0.f;
    for (int it = 0; it < nchunk; ++it) {
      const int st = it & 1;
      if (!mbar_wait(&bar_sfull[st], (it >> 1) & 1, abort, ctx)) break;
      tc_fence_after();
#pragma unroll 1
      for (int piece = 0; piece < 4; ++piece) {
        const int col0 = half * 128 + piece * 32;
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + st * RS_N + col0, r);
        tmem_ld_wait();
        const int key0 = it * RS_N + col0;
        const uint32_t kv = kMask ? piece_keys<true>(key0, Lr, tmask) : (key0 + 32 <= Lr ? 0xffffffffu : 0u);
        if (kv == 0xffffffffu) {
          // full piece: max on the raw scores (c2 > 0), then one packed FMA per column pair
          float pm = __uint_as_float(r[0]);
#pragma unroll
          for (int j = 1; j < 31; j += 2) pm = fmax3(pm, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
          pm = fmaxf(pm, __uint_as_float(r[31]));
          const float mn = fmaxf(m, pm * c2);
          const float2 cc = make_float2(c2, c2), nm = make_float2(-mn, -mn);
          float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 a = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), cc, nm);
            s2 = __fadd2_rn(s2, make_float2(ex2(a.x), ex2(a.y)));
          }
          l = l * ex2(m - mn) + (s2.x + s2.y);
          m = mn;
          continue;
        }
        float x[32];
        float pm = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const bool ok = kMask ? ((kv >> j) & 1u) : key0 + j < Lr;
          x[j] = ok ? __uint_as_float(r[j]) * c2 : -INFINITY;
          pm = fmaxf(pm, x[j]);
        }
        const float mn = fmaxf(m, pm);
        if (mn == -INFINITY) continue;
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) s += ex2(x[j] - mn);
        l = l * ex2(m - mn) + s;
        m = mn;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sfree[st]);
    }
    m_half[half][row] = m;
    l_half[half][row] = l;
    named_bar_sync(1, 256);
    if (half == 0) {
      const float m1 = m_half[0][row], m2 = m_half[1][row];
      const float mm = fmaxf(m1, m2);
      const float ll = l_half[0][row] * ex2(m1 - mm) + l_half[1][row] * ex2(m2 - mm);
      lse_sh[row] = mm + __log2f(ll);
    }
    named_bar_sync(1, 256);
    const float lse2 = lse_sh[row];
    const int qtile = (m0 + row) / G;  // G pooled rows per tile
    const bool row_ok = qtile < N;
    // kMask: this pooled query row counts only if its sub-cube holds a real token; the tile's
    // score row is the mean over its real query sub-cubes (lanes 4g .. 4g+3 are tile g's rows)
    float qw = 1.f, tile_inv = 1.f / G;
    if constexpr (kMask) {
      const int a = m0 + row;
      qw = (a < Lr && ((__ldg(tmask + (a >> 2)) >> (16 * (a & 3))) & 0xffffu)) ? 1.f : 0.f;
      float gsum = qw + __shfl_xor_sync(0xffffffffu, qw, 1);
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
      tile_inv = gsum > 0.f ? 1.f / gsum : 0.f;
    }
    float* out_row = scores + ((size_t)bh * N + (row_ok ? qtile : 0)) * N;
    for (int it = nchunk; it < 2 * nchunk; ++it) {
      const int st = it & 1, c = it - nchunk;
      if (!mbar_wait(&bar_sfull[st], (it >> 1) & 1, abort, ctx)) break;
      tc_fence_after();
      float t[32];
#pragma unroll
      for (int piece = 0; piece < 4; ++piece) {
        const int col0 = half * 128 + piece * 32;
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + st * RS_N + col0, r);
        tmem_ld_wait();
        const int key0 = c * RS_N + col0;
        const uint32_t kv = kMask ? piece_keys<true>(key0, Lr, tmask) : (key0 + 32 <= Lr ? 0xffffffffu : 0u);
        constexpr int TPP = 32 / G;  // key tiles per 32-key piece
        if (kv == 0xffffffffu) {
          // full piece: packed FMA for the exponent arguments and packed sums per key tile
          const float2 cc = make_float2(c2, c2), nl = make_float2(-lse2, -lse2);
#pragma unroll
          for (int jj = 0; jj < TPP; ++jj) {
            float2 sum = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < G; e += 2) {
              const float2 a = __ffma2_rn(
                  make_float2(__uint_as_float(r[G * jj + e]), __uint_as_float(r[G * jj + e + 1])), cc, nl);
              sum = __fadd2_rn(sum, make_float2(ex2(a.x), ex2(a.y)));
            }
            t[piece * TPP + jj] = sum.x + sum.y;
          }
          continue;
        }
#pragma unroll
        for (int jj = 0; jj < TPP; ++jj) {
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < G; ++e) {
            const int j = G * jj + e;
            const bool ok = kMask ? ((kv >> j) & 1u) : key0 + j < Lr;
            acc += ok ? ex2(__uint_as_float(r[j]) * c2 - lse2) : 0.f;
          }
          t[piece * TPP + jj] = acc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sfree[st]);
      // sum over the G = 4 query sub-rows (lanes 4g..4g+3), reduce-scatter: lane keeps 8 tiles
      if constexpr (kMask) {
#pragma unroll
        for (int j = 0; j < 32; ++j) t[j] *= qw;
      }
      if constexpr (G == 16) {
        // t[0..7]: this pooled query row's sums over the 8 key tiles of the chunk half. Sum the
        // 16 query rows of the tile (lanes 16g .. 16g+15); lane 16g writes the 8 tile scores.
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) t[j] += __shfl_xor_sync(0xffffffffu, t[j], o);
          t[j] *= tile_inv;
        }
        const int j0 = (c * RS_N + half * 128) / G;
        if (row_ok && (lane & 15) == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j0 + j < N) out_row[j0 + j] = t[j];
        }
        continue;
      }
      float u[16];
      const bool hi2 = lane & 2;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float send = hi2 ? t[j] : t[16 + j];
        const float keep = hi2 ? t[16 + j] : t[j];
        u[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
      float w[8];
      const bool hi1 = lane & 1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float send = hi1 ? u[j] : u[8 + j];
        const float keep = hi1 ? u[8 + j] : u[j];
        w[j] = (keep + __shfl_xor_sync(0xffffffffu, send, 1)) * tile_inv;
      }
      const int j0 = (c * RS_N + half * 128) / 4 + (hi2 ? 16 : 0) + (hi1 ? 8 : 0);
      if (row_ok) {
        if (j0 + 8 <= N) {
          float4* dst = reinterpret_cast<float4*>(out_row + j0);
          if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
            dst[0] = make_float4(w[0], w[1], w[2], w[3]);
            dst[1] = make_float4(w[4], w[5], w[6], w[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) out_row[j0 + j] = w[j];
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j0 + j < N) out_row[j0 + j] = w[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// CUDA-core router scores for fp32 inputs (and head_dim 64): CTA = one query tile of one
// (b, h). Step 1: LSE of its G pooled query rows over all pooled keys. Step 2: one thread per
// key tile sums exp(s - lse) over the G x G pooled pairs.
// ------------------------------------------------------------------------------------------
// tmask != nullptr (a padded grid): keys and query rows of sub-cubes without a real token are
// left out, and the tile's score row is the mean over its real query sub-cubes.
template <typename T, int D, int kG>
__global__ void __launch_bounds__(128) router_scores_simt_kernel(const T* __restrict__ qr, const T* __restrict__ kr,
                                                                 float* __restrict__ scores, int Lr, int N,
                                                                 const uint64_t* __restrict__ tmask) {
  __shared__ float qs[kG][D];
  __shared__ float red_m[kG][128], red_l[kG][128];
  __shared__ float lse_s[kG];
  const int i = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const T* qb = qr + ((size_t)bh * Lr + (size_t)i * kG) * D;
  const T* kb = kr + (size_t)bh * Lr * D;
  for (int e = t; e < kG * D; e += 128) qs[e / D][e % D] = (float)qb[e];
  __syncthreads();
  const float scale = rsqrtf((float)D);
  float m[kG], l[kG];
#pragma unroll
  for (int a = 0; a < kG; ++a) m[a] = -INFINITY, l[a] = 0.f;
  auto key_ok = [&](int b) { return !tmask || ((tmask[b / kG] >> (16 * (b % kG))) & 0xffffu) != 0; };
  for (int b = t; b < Lr; b += 128) {
    if (!key_ok(b)) continue;
    float s[kG] = {};
    for (int d = 0; d < D; ++d) {
      const float kv = (float)kb[(size_t)b * D + d];
#pragma unroll
      for (int a = 0; a < kG; ++a) s[a] += qs[a][d] * kv;
    }
#pragma unroll
    for (int a = 0; a < kG; ++a) {
      const float x = s[a] * scale;
      const float mn = fmaxf(m[a], x);
      l[a] = l[a] * __expf(m[a] - mn) + __expf(x - mn);
      m[a] = mn;
    }
  }
#pragma unroll
  for (int a = 0; a < kG; ++a) red_m[a][t] = m[a], red_l[a][t] = l[a];
  __syncthreads();
  if (t < kG) {
    float mm = -INFINITY;
    for (int u = 0; u < 128; ++u) mm = fmaxf(mm, red_m[t][u]);
    float ll = 0.f;
    for (int u = 0; u < 128; ++u)
      if (red_m[t][u] != -INFINITY) ll += red_l[t][u] * __expf(red_m[t][u] - mm);
    lse_s[t] = mm + __logf(ll);
  }
  __syncthreads();
  const uint64_t qm = tmask ? tmask[i] : ~0ull;
  float qw[kG], g = 0.f;
#pragma unroll
  for (int a = 0; a < kG; ++a) {
    qw[a] = (!tmask || ((qm >> (16 * a)) & 0xffffu)) ? 1.f : 0.f;
    g += qw[a];
  }
  for (int j = t; j < N; j += 128) {
    float acc = 0.f;
    for (int b = kG * j; b < kG * j + kG; ++b) {
      if (!key_ok(b)) continue;
      float s[kG] = {};
      for (int d = 0; d < D; ++d) {
        const float kv = (float)kb[(size_t)b * D + d];
#pragma unroll
        for (int a = 0; a < kG; ++a) s[a] += qs[a][d] * kv;
      }
#pragma unroll
      for (int a = 0; a < kG; ++a) acc += qw[a] * __expf(s[a] * scale - lse_s[a]);
    }
    scores[((size_t)bh * N + i) * N + j] = acc / g;
  }
}

}  // namespace

vsa2_status launch_router(const Dims& d, const void* q, const void* k, float* scores, char* ws, cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  void* qr = ws + w.qr;
  void* kr = ws + w.kr;
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const int64_t pooled = (int64_t)d.BH * d.Lr;
  const int cpr = d.D * d.esize / 16;
  const int64_t threads = 2 * pooled * cpr;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  const uint64_t* tmask = nullptr;
  if (d.padded) {
    tmask = reinterpret_cast<const uint64_t*>(ws + w.tmask);
    if (launch_tile_masks(d, reinterpret_cast<uint64_t*>(ws + w.tmask), s) != VSA2_OK) return VSA2_ERR_CUDA;
  }
  if (d.dtype == VSA2_BF16) {
    using bf = __nv_bfloat16;
    const bool fold = coarse_pool_in_router(d);
    auto kern = d.R == 8 ? router_pool_kernel<bf, false, 8>
                         : (d.padded ? (fold ? router_pool_kernel<bf, true, 16, true> : router_pool_kernel<bf, true, 16>)
                                     : (fold ? router_pool_kernel<bf, false, 16, true> : router_pool_kernel<bf, false, 16>));
    kern<<<blocks, 256, 0, s>>>((const bf*)q, (const bf*)k, (bf*)qr, (bf*)kr, pooled, cpr, tmask, d.Lr,
                                fold ? (bf*)(ws + w.qc) : nullptr, fold ? (bf*)(ws + w.kc) : nullptr,
                                kTile * w.Nc_tiles);
  } else {
    auto kern = d.R == 8 ? router_pool_kernel<float, false, 8>
                         : (d.padded ? router_pool_kernel<float, true, 16> : router_pool_kernel<float, false, 16>);
    kern<<<blocks, 256, 0, s>>>((const float*)q, (const float*)k, (float*)qr, (float*)kr, pooled, cpr, tmask, d.Lr,
                                nullptr, nullptr, 0);
  }
  if (check_launch(__func__) != VSA2_OK) return VSA2_ERR_CUDA;

  if (d.dtype == VSA2_BF16) {
    CUtensorMap tq, tk;
    if (!make_tmap_3d_bf16(&tq, qr, d.D, d.Lr, d.BH, 64, RS_M)) return tmap_fail("tensor map encoding (Qr) failed");
    if (!make_tmap_3d_bf16(&tk, kr, d.D, d.Lr, d.BH, 64, RS_N)) return tmap_fail("tensor map encoding (Kr) failed");
    const float c2 = 1.4426950408889634f / sqrtf((float)d.D);
    dim3 grid((d.Lr + RS_M - 1) / RS_M, d.BH);
    if (d.D == 128) {
      auto kern = d.G == 16 ? router_scores_tc_kernel<2, false, 16>
                            : (d.padded ? router_scores_tc_kernel<2, true, 4> : router_scores_tc_kernel<2, false, 4>);
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RouterSmem<2>::kDyn);
      kern<<<grid, RS_THREADS, RouterSmem<2>::kDyn, s>>>(tq, tk, scores, d.Lr, d.N, c2, tmask, ctx);
    } else {
      auto kern = d.G == 16 ? router_scores_tc_kernel<1, false, 16>
                            : (d.padded ? router_scores_tc_kernel<1, true, 4> : router_scores_tc_kernel<1, false, 4>);
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RouterSmem<1>::kDyn);
      kern<<<grid, RS_THREADS, RouterSmem<1>::kDyn, s>>>(tq, tk, scores, d.Lr, d.N, c2, tmask, ctx);
    }
  } else {
    dim3 grid(d.N, d.BH);
    const float* fq = (const float*)qr;
    const float* fk = (const float*)kr;
    if (d.G == 16) {
      if (d.D == 128)
        router_scores_simt_kernel<float, 128, 16><<<grid, 128, 0, s>>>(fq, fk, scores, d.Lr, d.N, tmask);
      else
        router_scores_simt_kernel<float, 64, 16><<<grid, 128, 0, s>>>(fq, fk, scores, d.Lr, d.N, tmask);
    } else if (d.D == 128) {
      router_scores_simt_kernel<float, 128, 4><<<grid, 128, 0, s>>>(fq, fk, scores, d.Lr, d.N, tmask);
    } else {
      router_scores_simt_kernel<float, 64, 4><<<grid, 128, 0, s>>>(fq, fk, scores, d.Lr, d.N, tmask);
    }
  }
  if (check_launch(__func__) != VSA2_OK) return VSA2_ERR_CUDA;
  return VSA2_OK;
}

}  // namespace vsa2
