// CUDA-core block-sparse attention (Eq. 12 of "Improving Video Sparse Attention with
// Fine-grained Router and Sparse Rebasing"; §2.1 definition) for the shapes the tensor-core
// kernels do not take: fp32 inputs and head_dim 64, plus the backward pass.
// Arithmetic is fp32 throughout. The forward treats keys at or beyond `kv_valid` tokens of a
// head as padding (the coarse branch's pooled sequence, Eq. 1-3, ends in a partial tile).
#include "common.cuh"
#include "internal.h"

namespace vsa2 {

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
  if constexpr (sizeof(T) == 2)
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  else
    return *p;
}
template <typename T>
__device__ __forceinline__ void stf(T* p, float v) {
  if constexpr (sizeof(T) == 2)
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
  else
    *p = v;
}

// Checks one CSR/CSC row in validate mode; returns false (and records the error) if broken.
__device__ __forceinline__ bool row_ok(int beg, int end, int cap, const DevCtx& ctx) {
  if (!(ctx.flags & VSA2_FLAG_VALIDATE)) return true;
  if (beg < 0 || end < beg || end > cap) {
    set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return false;
  }
  return true;
}
__device__ __forceinline__ bool idx_ok(int j, int N, const DevCtx& ctx) {
  if (!(ctx.flags & VSA2_FLAG_VALIDATE)) return true;
  if (j < 0 || j >= N) {
    set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return false;
  }
  return true;
}

namespace {

// Forward: CTA = one query tile of one (b, h), four threads per query row t (lanes 4t .. 4t+3 of
// the row's warp). Thread (t, g) scores the keys u = 4k + g and accumulates the output columns
// d = 4e + g; the row's maximum and sum combine over the four lanes, and its probabilities pass
// through shared memory inside the warp. K and V rows are stored with a stride of D + 1 floats
// and the probability rows with 65, so the four threads of a row read different banks.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, const int32_t* __restrict__ kv_off,
                                                            const int32_t* __restrict__ kv_idx, T* __restrict__ o,
                                                            float* __restrict__ lse, int N, int64_t L, int topk,
                                                            int64_t kv_valid, const uint64_t* __restrict__ tmask,
                                                            const float* __restrict__ gate, const T* __restrict__ oc,
                                                            T* __restrict__ of, DevCtx ctx) {
  constexpr int KS = D + 1;    // K / V row stride
  constexpr int PS = 65;       // probability row stride
  constexpr int DQ = D / 4;    // output columns per thread
  extern __shared__ float sm[];
  float* qT = sm;              // [D][64]
  float* ks = qT + D * 64;     // [64][KS]
  float* vs = ks + 64 * KS;    // [64][KS]
  float* ps = vs + 64 * KS;    // [64][PS]
  const int i = blockIdx.x, bh = blockIdx.y;
  const int t = threadIdx.x >> 2, g = threadIdx.x & 3;
  const size_t tok0 = (size_t)bh * L + (size_t)i * kTile;
  for (int e = threadIdx.x; e < 64 * D; e += 256) {
    const int r = e / D, c = e % D;
    qT[c * 64 + r] = ldf(q + (tok0 + r) * D + c);
  }
  const int beg = kv_off[(size_t)bh * (N + 1) + i], end = kv_off[(size_t)bh * (N + 1) + i + 1];
  const bool ok = row_ok(beg, end, N * topk, ctx);
  const int32_t* idx = kv_idx + (size_t)bh * N * topk;
  const float scale = rsqrtf((float)D);
  float m = -INFINITY, l = 0.f;
  float acc[DQ];
#pragma unroll
  for (int e = 0; e < DQ; ++e) acc[e] = 0.f;
  float* prow = ps + t * PS;
  for (int p = beg; ok && p < end; ++p) {
    const int j = idx[p];
    if (!idx_ok(j, N, ctx)) break;
    const size_t kt0 = (size_t)bh * L + (size_t)j * kTile;
    const uint64_t km = tmask ? tmask[j] : ~0ull;  // real tokens of a padded grid's tile
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * D; e += 256) {
      const int r = e / D, c = e % D;
      ks[r * KS + c] = ldf(k + kt0 * D + e);
      vs[r * KS + c] = ldf(v + kt0 * D + e);
    }
    __syncthreads();
    float s[16];
    float mx = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const int u = 4 * kk + g;
      float a = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) a = fmaf(qT[d * 64 + t], ks[u * KS + d], a);
      // keys past kv_valid, and padding tokens of a padded grid, are masked
      s[kk] = ((int64_t)j * kTile + u < kv_valid && ((km >> u) & 1ull)) ? a * scale : -INFINITY;
      mx = fmaxf(mx, s[kk]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(m, mx);
    const float alpha = __expf(m - mn);
    float sum = 0.f;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float pr = __expf(s[kk] - mn);
      sum += pr;
      prow[4 * kk + g] = pr;
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    l = l * alpha + sum;
    m = mn;
    __syncwarp();  // the row's 64 probabilities are written by its four lanes
#pragma unroll
    for (int e = 0; e < DQ; ++e) acc[e] *= alpha;
#pragma unroll 4
    for (int u = 0; u < 64; ++u) {
      const float pr = prow[u];
      const float* vr = vs + u * KS + g;
#pragma unroll
      for (int e = 0; e < DQ; ++e) acc[e] = fmaf(pr, vr[4 * e], acc[e]);
    }
    __syncwarp();  // before the next tile's probabilities overwrite the row
  }
  const bool q_real = !tmask || ((tmask[i] >> t) & 1ull);  // a padding query row gets o = 0, lse = -inf
  const float inv = (l > 0.f && q_real) ? 1.f / l : 0.f;
  T* orow = o + (tok0 + t) * D + g;
  if (gate) {  // Eq. 13-14 on the fp32 fine output: o = tanh(g) * oc[tile] + O_f
    const float gt = tanhf(gate[tok0 + t]);
    const T* crow = oc + ((size_t)bh * N + i) * D + g;
#pragma unroll
    for (int e = 0; e < DQ; ++e) {
      const float f = inv != 0.f ? acc[e] * inv : 0.f;
      stf(orow + 4 * e, fmaf(gt, ldf(crow + 4 * e), f));
      if (of) stf(of + (tok0 + t) * D + g + 4 * e, f);
    }
  } else {
#pragma unroll
    for (int e = 0; e < DQ; ++e) stf(orow + 4 * e, inv != 0.f ? acc[e] * inv : 0.f);
  }
  if (g == 0) lse[tok0 + t] = (l > 0.f && q_real) ? m + __logf(l) : -INFINITY;
}

// delta = rowsum(dO * O), warp per row.
template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                                                             float* __restrict__ delta, int64_t rows, int D) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int d = lane; d < D; d += 32) acc += ldf(o + row * D + d) * ldf(dout + row * D + d);
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
}

// dQ: CTA = one query tile, 128 threads = (query row t, half h). Over the tile's CSR list.
template <typename T, int D>
__global__ void __launch_bounds__(128) attn_bwd_dq_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                               const T* __restrict__ v, const T* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ delta,
                                                               const int32_t* __restrict__ kv_off,
                                                               const int32_t* __restrict__ kv_idx,
                                                               float* __restrict__ dq, int N, int64_t L, int topk,
                                                               const uint64_t* __restrict__ tmask, DevCtx ctx) {
  extern __shared__ float sm[];
  float* qT = sm;             // [D][64]
  float* doT = qT + D * 64;   // [D][64]
  float* ks = doT + D * 64;   // [64][D]
  float* vs = ks + 64 * D;    // [64][D]
  float* dsT = vs + 64 * D;   // [64 (u)][64 (t)]
  const int i = blockIdx.x, bh = blockIdx.y;
  const int t = threadIdx.x & 63, h = threadIdx.x >> 6;
  const size_t tok0 = (size_t)bh * L + (size_t)i * kTile;
  for (int e = threadIdx.x; e < 64 * D; e += 128) {
    const int r = e / D, c = e % D;
    qT[c * 64 + r] = ldf(q + (tok0 + r) * D + c);
    doT[c * 64 + r] = ldf(dout + (tok0 + r) * D + c);
  }
  const float my_lse = lse[tok0 + t], my_delta = delta[tok0 + t];
  const float scale = rsqrtf((float)D);
  float acc[D / 2];
#pragma unroll
  for (int d = 0; d < D / 2; ++d) acc[d] = 0.f;
  const int beg = kv_off[(size_t)bh * (N + 1) + i], end = kv_off[(size_t)bh * (N + 1) + i + 1];
  const bool ok = row_ok(beg, end, N * topk, ctx);
  const int32_t* idx = kv_idx + (size_t)bh * N * topk;
  for (int p = beg; ok && p < end; ++p) {
    const int j = idx[p];
    if (!idx_ok(j, N, ctx)) break;
    const size_t kt0 = (size_t)bh * L + (size_t)j * kTile;
    const uint64_t km = tmask ? tmask[j] : ~0ull;  // padding keys of a padded grid take no part
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * D; e += 128) {
      ks[e] = ldf(k + kt0 * D + e);
      vs[e] = ldf(v + kt0 * D + e);
    }
    __syncthreads();
    for (int u = 32 * h; u < 32 * h + 32; ++u) {
      float s = 0.f, dp = 0.f;
      for (int d = 0; d < D; ++d) {
        s += qT[d * 64 + t] * ks[u * D + d];
        dp += doT[d * 64 + t] * vs[u * D + d];
      }
      // a row with lse = -inf (no selection, or a padding query row) has P = 0
      const float pr = (my_lse == -INFINITY || !((km >> u) & 1ull)) ? 0.f : __expf(s * scale - my_lse);
      dsT[u * 64 + t] = pr * (dp - my_delta);
    }
    __syncthreads();
#pragma unroll 1
    for (int u = 0; u < 64; ++u) {
      const float ds = dsT[u * 64 + t];
#pragma unroll
      for (int d = 0; d < D / 2; ++d) acc[d] += ds * ks[u * D + h * (D / 2) + d];
    }
  }
#pragma unroll
  for (int d = 0; d < D / 2; ++d) dq[(tok0 + t) * D + h * (D / 2) + d] = acc[d] * scale;
}

// dK, dV: CTA = one KV tile, 128 threads = (key row u, half h). Over the tile's CSC list.
template <typename T, int D>
__global__ void __launch_bounds__(128) attn_bwd_dkdv_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                 const T* __restrict__ v, const T* __restrict__ dout,
                                                                 const float* __restrict__ lse,
                                                                 const float* __restrict__ delta,
                                                                 const int32_t* __restrict__ q_off,
                                                                 const int32_t* __restrict__ q_idx,
                                                                 float* __restrict__ dk, float* __restrict__ dv, int N,
                                                                 int64_t L, int topk, const uint64_t* __restrict__ tmask,
                                                                 DevCtx ctx) {
  extern __shared__ float sm[];
  float* kT = sm;             // [D][64]
  float* vT = kT + D * 64;    // [D][64]
  float* qs = vT + D * 64;    // [64][D]
  float* dos = qs + 64 * D;   // [64][D]
  float* ps = dos + 64 * D;   // [64 (t)][64 (u)]
  float* dss = ps + 64 * 64;  // [64 (t)][64 (u)]
  __shared__ float lse_s[64], delta_s[64];
  const int j = blockIdx.x, bh = blockIdx.y;
  const int u = threadIdx.x & 63, h = threadIdx.x >> 6;
  const size_t kt0 = (size_t)bh * L + (size_t)j * kTile;
  for (int e = threadIdx.x; e < 64 * D; e += 128) {
    const int r = e / D, c = e % D;
    kT[c * 64 + r] = ldf(k + (kt0 + r) * D + c);
    vT[c * 64 + r] = ldf(v + (kt0 + r) * D + c);
  }
  const float scale = rsqrtf((float)D);
  const bool key_real = !tmask || ((tmask[j] >> u) & 1ull);  // a padding key gets dK = dV = 0
  float adk[D / 2], adv[D / 2];
#pragma unroll
  for (int d = 0; d < D / 2; ++d) adk[d] = 0.f, adv[d] = 0.f;
  const int beg = q_off[(size_t)bh * (N + 1) + j], end = q_off[(size_t)bh * (N + 1) + j + 1];
  const bool ok = row_ok(beg, end, N * topk, ctx);
  const int32_t* idx = q_idx + (size_t)bh * N * topk;
  for (int p = beg; ok && p < end; ++p) {
    const int i = idx[p];
    if (!idx_ok(i, N, ctx)) break;
    const size_t tok0 = (size_t)bh * L + (size_t)i * kTile;
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * D; e += 128) {
      qs[e] = ldf(q + tok0 * D + e);
      dos[e] = ldf(dout + tok0 * D + e);
    }
    if (threadIdx.x < 64) {
      lse_s[threadIdx.x] = lse[tok0 + threadIdx.x];
      delta_s[threadIdx.x] = delta[tok0 + threadIdx.x];
    }
    __syncthreads();
    for (int t = 32 * h; t < 32 * h + 32; ++t) {
      float s = 0.f, dp = 0.f;
      for (int d = 0; d < D; ++d) {
        s += qs[t * D + d] * kT[d * 64 + u];
        dp += dos[t * D + d] * vT[d * 64 + u];
      }
      const float pr = (lse_s[t] == -INFINITY || !key_real) ? 0.f : __expf(s * scale - lse_s[t]);
      ps[t * 64 + u] = pr;
      dss[t * 64 + u] = pr * (dp - delta_s[t]);
    }
    __syncthreads();
#pragma unroll 1
    for (int t = 0; t < 64; ++t) {
      const float pr = ps[t * 64 + u], ds = dss[t * 64 + u];
#pragma unroll
      for (int d = 0; d < D / 2; ++d) {
        adv[d] += pr * dos[t * D + h * (D / 2) + d];
        adk[d] += ds * qs[t * D + h * (D / 2) + d];
      }
    }
  }
#pragma unroll
  for (int d = 0; d < D / 2; ++d) {
    dk[(kt0 + u) * D + h * (D / 2) + d] = adk[d] * scale;
    dv[(kt0 + u) * D + h * (D / 2) + d] = adv[d];
  }
}

template <typename T, int D>
vsa2_status fwd_simt(const Dims& d, const void* q, const void* k, const void* v, const int32_t* kv_off,
                     const int32_t* kv_idx, void* o, float* lse, const DevCtx& ctx, int topk, int64_t kv_valid,
                     const uint64_t* tmask, const float* gate, const void* oc, void* of, cudaStream_t s) {
  const size_t smem = ((size_t)64 * D + 2 * 64 * (D + 1) + 64 * 65) * sizeof(float);
  auto kern = attn_fwd_simt_kernel<T, D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<dim3(d.N, d.BH), 256, smem, s>>>((const T*)q, (const T*)k, (const T*)v, kv_off, kv_idx, (T*)o, lse, d.N,
                                         d.L, topk, kv_valid, tmask, gate, (const T*)oc, (T*)of, ctx);
  return check_launch(__func__);
}

template <typename T, int D>
vsa2_status bwd_simt(const Dims& d, const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, const int32_t* kv_off, const int32_t* kv_idx, const int32_t* q_off,
                     const int32_t* q_idx, float* dq, float* dk, float* dv, float* delta, int topk,
                     const uint64_t* tmask, const DevCtx& ctx, cudaStream_t s) {
  const int64_t rows = (int64_t)d.BH * d.L;
  attn_bwd_delta_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const T*)o, (const T*)dout, delta, rows, d.D);
  const size_t smem_dq = ((size_t)4 * 64 * D + 64 * 64) * sizeof(float);
  auto kq = attn_bwd_dq_simt_kernel<T, D>;
  cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
  kq<<<dim3(d.N, d.BH), 128, smem_dq, s>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta,
                                           kv_off, kv_idx, dq, d.N, d.L, topk, tmask, ctx);
  const size_t smem_kv = ((size_t)4 * 64 * D + 2 * 64 * 64) * sizeof(float);
  auto kk = attn_bwd_dkdv_simt_kernel<T, D>;
  cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv);
  kk<<<dim3(d.N, d.BH), 128, smem_kv, s>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, q_off,
                                           q_idx, dk, dv, d.N, d.L, topk, tmask, ctx);
  return check_launch(__func__);
}

}  // namespace

vsa2_status attn_fwd_simt(const Dims& d, const void* q, const void* k, const void* v, int topk,
                          const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                          int64_t kv_valid, const uint64_t* tmask, cudaStream_t s, const float* gate,
                          const void* oc, void* of) {
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  if (d.dtype == VSA2_BF16) {
    if (d.D == 128)
      return fwd_simt<__nv_bfloat16, 128>(d, q, k, v, kv_off, kv_idx, o, lse, ctx, topk, kv_valid, tmask, gate, oc,
                                          of, s);
    return fwd_simt<__nv_bfloat16, 64>(d, q, k, v, kv_off, kv_idx, o, lse, ctx, topk, kv_valid, tmask, gate, oc, of,
                                       s);
  }
  if (d.D == 128)
    return fwd_simt<float, 128>(d, q, k, v, kv_off, kv_idx, o, lse, ctx, topk, kv_valid, tmask, gate, oc, of, s);
  return fwd_simt<float, 64>(d, q, k, v, kv_off, kv_idx, o, lse, ctx, topk, kv_valid, tmask, gate, oc, of, s);
}

vsa2_status attn_bwd_simt(const Dims& d, const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, const int32_t* kv_off, const int32_t* kv_idx, const int32_t* q_off,
                          const int32_t* q_idx, float* dq, float* dk, float* dv, int topk, char* ws,
                          const uint64_t* tmask, cudaStream_t s) {
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  float* delta = reinterpret_cast<float*>(ws + ws_layout(d).delta);
  if (d.dtype == VSA2_BF16) {
    if (d.D == 128)
      return bwd_simt<__nv_bfloat16, 128>(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, delta,
                                          topk, tmask, ctx, s);
    return bwd_simt<__nv_bfloat16, 64>(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, delta,
                                       topk, tmask, ctx, s);
  }
  if (d.D == 128)
    return bwd_simt<float, 128>(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, delta, topk, tmask,
                                ctx, s);
  return bwd_simt<float, 64>(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, delta, topk, tmask, ctx, s);
}

}  // namespace vsa2
