// Coarse branch and gated merge of "Improving Video Sparse Attention with Fine-grained Router and
// Sparse Rebasing", §2.2:
//   Qc, Kc, Vc = MeanPool_B(Q, K, V)                 Eq. 1 (one row per 64-token tile)
//   O_c_hat    = softmax(Qc Kc^T / sqrt(D)) Vc       Eq. 2-3 (dense over the N pooled rows)
//   O          = tanh(X W_g) * Repeat_B(O_c_hat) + O_f   Eq. 4, 13-14 (X W_g given per token)
// and their gradients.
//
// The pooled rows of a head form a sequence of N "tokens", padded to Nc = ceil(N / 64) tiles.
// Dense attention over it is the block-sparse forward with every tile listed and the padded
// keys masked, so it runs on the same kernels as the fine branch (tcgen05 for bf16 with
// D = 128). Pooling and the merge read each input once and are HBM-bound.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

// the two bf16 halves of a packed word, as fp32
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// V consecutive elements of a row as fp32 (V * sizeof(T) bytes in one load)
template <typename T, int V>
__device__ __forceinline__ void load_vec(const T* p, float* f) {
  if constexpr (std::is_same<T, float>::value) {
    if constexpr (V == 4) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(p));
      f[0] = x.x, f[1] = x.y, f[2] = x.z, f[3] = x.w;
    } else {
      const float2 x = __ldg(reinterpret_cast<const float2*>(p));
      f[0] = x.x, f[1] = x.y;
    }
  } else {
    if constexpr (V == 4) {
      const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
      f[0] = bf_lo(x.x), f[1] = bf_hi(x.x), f[2] = bf_lo(x.y), f[3] = bf_hi(x.y);
    } else {
      const uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(p));
      f[0] = bf_lo(x), f[1] = bf_hi(x);
    }
  }
}

template <typename T, int V>
__device__ __forceinline__ void store_vec(T* p, const float* f) {
  if constexpr (std::is_same<T, float>::value) {
    if constexpr (V == 4)
      *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    else
      *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
  } else {
    if constexpr (V == 4)
      *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
    else
      *reinterpret_cast<uint32_t*>(p) = pack_bf16(f[0], f[1]);
  }
}

// Eq. 1: warp per pooled row r of head bh; lane owns D/32 consecutive channels. Rows r >= N
// (padding of the last tile) are written as zeros. With tmask (a padded grid) each mean runs
// over the tile's real tokens only. With v_only the rows r < N of Qc and Kc are left as they are
// (the router's pooling pass wrote them) and only V is read.
template <typename T, int D>
__global__ void __launch_bounds__(256) coarse_pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, T* __restrict__ qc,
                                                          T* __restrict__ kc, T* __restrict__ vc, int N, int Lc,
                                                          int64_t L, const uint64_t* __restrict__ tmask,
                                                          bool v_only) {
  constexpr int V = D / 32;
  const int bh = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= Lc) return;
  const size_t dst = ((size_t)bh * Lc + r) * D + lane * V;
  const T* src[3] = {q, k, v};
  T* out[3] = {qc, kc, vc};
#pragma unroll
  for (int x = 0; x < 3; ++x) {
    if (v_only && x < 2 && r < N) continue;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    if (r < N) {
      const T* p = src[x] + ((size_t)bh * L + (size_t)r * kTile) * D + lane * V;
      const uint64_t real = tmask ? __ldg(tmask + r) : ~0ull;
#pragma unroll 8
      for (int t = 0; t < kTile; ++t) {
        if (!((real >> t) & 1ull)) continue;
        float f[V];
        load_vec<T, V>(p + (size_t)t * D, f);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += f[e];
      }
      const float inv = 1.f / __popcll(real);  // every tile holds a real token
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] *= inv;
    }
    store_vec<T, V>(out[x] + dst, acc);
  }
}

// Every query tile of the pooled sequence lists all Nc tiles: offsets i * Nc, indices 0..Nc-1.
__global__ void __launch_bounds__(256) coarse_csr_kernel(int Nc, int32_t* __restrict__ off, int32_t* __restrict__ idx) {
  const int bh = blockIdx.x;
  for (int i = threadIdx.x; i <= Nc; i += blockDim.x) off[(size_t)bh * (Nc + 1) + i] = i * Nc;
  for (int e = threadIdx.x; e < Nc * Nc; e += blockDim.x) idx[(size_t)bh * Nc * Nc + e] = e % Nc;
}

// Eq. 4, 13-14: one 16-byte chunk of an output row per iteration. o may alias o_f (each element
// is read before it is written, by the same thread).
template <typename T>
__global__ void __launch_bounds__(256) gated_merge_kernel(const T* o_f, const float* __restrict__ gate_logits,
                                                          const T* __restrict__ oc, T* o, int64_t rows, int64_t L,
                                                          int N, int D) {
  constexpr int VW = 16 / sizeof(T);
  const int cpr = D / VW;
  const int64_t total = rows * cpr;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total; c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = c / cpr;
    const int col = (int)(c - row * cpr) * VW;
    const int64_t bh = row / L;
    const int tile = (int)((row - bh * L) / kTile);
    const float gate = tanhf(__ldg(gate_logits + row));
    const uint4 a = *reinterpret_cast<const uint4*>(o_f + row * D + col);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(oc + ((size_t)bh * N + tile) * D + col));
    uint4 r;
    if constexpr (std::is_same<T, float>::value) {
      r.x = __float_as_uint(fmaf(gate, __uint_as_float(b.x), __uint_as_float(a.x)));
      r.y = __float_as_uint(fmaf(gate, __uint_as_float(b.y), __uint_as_float(a.y)));
      r.z = __float_as_uint(fmaf(gate, __uint_as_float(b.z), __uint_as_float(a.z)));
      r.w = __float_as_uint(fmaf(gate, __uint_as_float(b.w), __uint_as_float(a.w)));
    } else {
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
      uint32_t rw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        rw[e] = pack_bf16(fmaf(gate, bf_lo(bw[e]), bf_lo(aw[e])), fmaf(gate, bf_hi(bw[e]), bf_hi(aw[e])));
      r = make_uint4(rw[0], rw[1], rw[2], rw[3]);
    }
    *reinterpret_cast<uint4*>(o + row * D + col) = r;
  }
}

// Gradients of Eq. 4, 13-14, warp per tile i of head bh (64 tokens t):
//   d_logits[t] = (1 - G[t]^2) * (dout[t] . oc[i]),   d_oc[i] = sum_t G[t] * dout[t],   G = tanh(logits)
// On a grid the tile does not divide (padded), the outputs of padding rows are dropped, so their
// dout reaches nothing: d_logits is 0 there and d_oc sums the real tokens only.
template <typename T, int D>
__global__ void __launch_bounds__(256) gated_merge_bwd_kernel(const T* __restrict__ dout,
                                                              const float* __restrict__ gate_logits,
                                                              const T* __restrict__ oc, float* __restrict__ d_logits,
                                                              float* __restrict__ d_oc, int N, int64_t L,
                                                              GridGeom geom, bool padded) {
  constexpr int V = D / 32;
  const int bh = blockIdx.y;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= N) return;
  const bool real0 = !padded || token_real(geom, i, lane), real1 = !padded || token_real(geom, i, 32 + lane);
  const size_t row0 = (size_t)bh * L + (size_t)i * kTile;
  float c[V], acc[V];
  load_vec<T, V>(oc + ((size_t)bh * N + i) * D + lane * V, c);
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  const float g0 = tanhf(__ldg(gate_logits + row0 + lane)), g1 = tanhf(__ldg(gate_logits + row0 + 32 + lane));
  float r0 = 0.f, r1 = 0.f;
#pragma unroll 4
  for (int t = 0; t < kTile; ++t) {
    if (!__shfl_sync(0xffffffffu, t < 32 ? real0 : real1, t & 31)) continue;  // warp-uniform
    float x[V];
    load_vec<T, V>(dout + (row0 + t) * D + lane * V, x);
    const float G = __shfl_sync(0xffffffffu, t < 32 ? g0 : g1, t & 31);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < V; ++e) {
      dot = fmaf(x[e], c[e], dot);
      acc[e] = fmaf(G, x[e], acc[e]);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (lane == (t & 31)) (t < 32 ? r0 : r1) = (1.f - G * G) * dot;
  }
  d_logits[row0 + lane] = r0;
  d_logits[row0 + 32 + lane] = r1;
  float* dst = d_oc + ((size_t)bh * N + i) * D + lane * V;
#pragma unroll
  for (int e = 0; e < V; ++e) dst[e] = acc[e];
}

// Inputs of the pooled sequence's backward, padded to Lc rows per head: O_c_hat and its
// gradient in the input dtype with zero rows past N, and the LSE with 0 past N. With zero K, V,
// O and dO rows there, the padded rows add nothing to the gradients of the real rows.
template <typename T, int D>
__global__ void __launch_bounds__(256) coarse_pad_bwd_kernel(const T* __restrict__ oc, const float* __restrict__ lse_c,
                                                             const float* __restrict__ d_oc, T* __restrict__ oc_pad,
                                                             float* __restrict__ lse_pad, T* __restrict__ doc_pad,
                                                             int N, int Lc) {
  constexpr int V = D / 32;
  const int bh = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= Lc) return;
  float o[V], g[V];
#pragma unroll
  for (int e = 0; e < V; ++e) o[e] = g[e] = 0.f;
  if (r < N) {
    load_vec<T, V>(oc + ((size_t)bh * N + r) * D + lane * V, o);
#pragma unroll
    for (int e = 0; e < V; ++e) g[e] = __ldg(d_oc + ((size_t)bh * N + r) * D + lane * V + e);
  }
  const size_t dst = ((size_t)bh * Lc + r) * D + lane * V;
  store_vec<T, V>(oc_pad + dst, o);
  store_vec<T, V>(doc_pad + dst, g);
  if (lane == 0) lse_pad[(size_t)bh * Lc + r] = r < N ? __ldg(lse_c + (size_t)bh * N + r) : 0.f;
}

// MeanPool_B's adjoint, accumulated: dx[t] += dxc[tile(t)] / 64 for Q, K and V (fp32), four
// channels per thread and iteration. With tmask (a padded grid) the mean ran over the tile's n
// real tokens: each of them gets dxc / n and the padding tokens nothing.
__global__ void __launch_bounds__(256) coarse_pool_bwd_kernel(const float* __restrict__ dqc,
                                                              const float* __restrict__ dkc,
                                                              const float* __restrict__ dvc, float* __restrict__ dq,
                                                              float* __restrict__ dk, float* __restrict__ dv,
                                                              int64_t rows, int64_t L, int Lc, int D,
                                                              const uint64_t* __restrict__ tmask) {
  const int cpr = D / 4;
  const int64_t total = rows * cpr;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total; c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = c / cpr;
    const int col = (int)(c - row * cpr) * 4;
    const int64_t bh = row / L;
    const int64_t tile = (row - bh * L) / kTile;
    const int64_t src = ((size_t)bh * Lc + tile) * D + col;
    float w = 1.f / kTile;
    if (tmask) {
      const uint64_t real = __ldg(tmask + tile);
      if (!((real >> ((row - bh * L) % kTile)) & 1ull)) continue;
      w = 1.f / __popcll(real);  // every tile holds a real token
    }
    const float* in[3] = {dqc, dkc, dvc};
    float* out[3] = {dq, dk, dv};
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(in[x] + src));
      float4* o = reinterpret_cast<float4*>(out[x] + row * D + col);
      float4 b = *o;
      b.x = fmaf(a.x, w, b.x);
      b.y = fmaf(a.y, w, b.y);
      b.z = fmaf(a.z, w, b.z);
      b.w = fmaf(a.w, w, b.w);
      *o = b;
    }
  }
}

template <typename T, int D>
void launch_pool(const Dims& d, const void* q, const void* k, const void* v, char* ws, const WsLayout& w,
                 const uint64_t* tmask, cudaStream_t s, bool v_only = false) {
  const int Lc = kTile * w.Nc_tiles;
  coarse_pool_kernel<T, D><<<dim3((Lc + 7) / 8, d.BH), 256, 0, s>>>(
      (const T*)q, (const T*)k, (const T*)v, (T*)(ws + w.qc), (T*)(ws + w.kc), (T*)(ws + w.vc), d.N, Lc, d.L, tmask,
      v_only);
}

int grid_for(int64_t work, int per_block) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return (int)std::max<int64_t>(1, std::min<int64_t>((work + per_block - 1) / per_block, (int64_t)sms * 8));
}

}  // namespace

vsa2_status launch_coarse_attn(const Dims& d, const void* q, const void* k, const void* v, void* oc, float* lse_c,
                               char* ws, cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  const int Nc = w.Nc_tiles;
  const int Lc = kTile * Nc;
  // Eq. 1: pooled rows (over the real tokens of a padded grid), padded with zeros to whole tiles
  uint64_t* tmask = nullptr;
  if (d.padded) {
    tmask = reinterpret_cast<uint64_t*>(ws + w.tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
  }
  if (d.dtype == VSA2_BF16 && d.D == 128)
    launch_pool<__nv_bfloat16, 128>(d, q, k, v, ws, w, tmask, s, coarse_pool_in_router(d));
  else if (d.dtype == VSA2_BF16)
    launch_pool<__nv_bfloat16, 64>(d, q, k, v, ws, w, tmask, s);
  else if (d.D == 128)
    launch_pool<float, 128>(d, q, k, v, ws, w, tmask, s);
  else
    launch_pool<float, 64>(d, q, k, v, ws, w, tmask, s);
  int32_t* c_off = reinterpret_cast<int32_t*>(ws + w.c_off);
  int32_t* c_idx = reinterpret_cast<int32_t*>(ws + w.c_idx);
  coarse_csr_kernel<<<d.BH, 256, 0, s>>>(Nc, c_off, c_idx);
  vsa2_status st = check_launch("coarse pooling");
  if (st != VSA2_OK) return st;
  // Eq. 2-3: dense attention over the pooled sequence; keys at rows >= N are padding
  Dims dc = d;
  dc.L = Lc;
  dc.N = Nc;
  dc.Lr = Lc / kPool;
  dc.padded = false;  // the pooled sequence's own padding is the kv_valid bound below
  void* oc_pad = ws + w.oc;
  float* lse_pad = reinterpret_cast<float*>(ws + w.lse_c);
  st = (d.dtype == VSA2_BF16 && d.D == 128)
           ? attn_fwd_tc_masked(dc, ws + w.qc, ws + w.kc, ws + w.vc, Nc, c_off, c_idx, oc_pad, lse_pad, ws, d.N, s)
           : attn_fwd_simt(dc, ws + w.qc, ws + w.kc, ws + w.vc, Nc, c_off, c_idx, oc_pad, lse_pad, ws, d.N, nullptr, s);
  if (st != VSA2_OK) return st;
  // the first N rows of every head, packed
  const size_t row_b = (size_t)d.D * d.esize;
  if (cudaMemcpy2DAsync(oc, (size_t)d.N * row_b, oc_pad, (size_t)Lc * row_b, (size_t)d.N * row_b, d.BH,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return cuda_fail("coarse branch: copy of the output rows");
  if (lse_c && cudaMemcpy2DAsync(lse_c, (size_t)d.N * 4, lse_pad, (size_t)Lc * 4, (size_t)d.N * 4, d.BH,
                                 cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return cuda_fail("coarse branch: copy of the LSE rows");
  return VSA2_OK;
}

vsa2_status launch_gated_merge_bwd(const Dims& d, const void* dout, const float* gate_logits, const void* oc,
                                   float* d_logits, float* d_oc, cudaStream_t s) {
  const dim3 grid((d.N + 7) / 8, d.BH);
  const GridGeom geom = grid_geom(d);
  if (d.dtype == VSA2_BF16 && d.D == 128)
    gated_merge_bwd_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)dout, gate_logits,
                                                                    (const __nv_bfloat16*)oc, d_logits, d_oc, d.N, d.L, geom, d.padded);
  else if (d.dtype == VSA2_BF16)
    gated_merge_bwd_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)dout, gate_logits,
                                                                   (const __nv_bfloat16*)oc, d_logits, d_oc, d.N, d.L, geom, d.padded);
  else if (d.D == 128)
    gated_merge_bwd_kernel<float, 128><<<grid, 256, 0, s>>>((const float*)dout, gate_logits, (const float*)oc,
                                                            d_logits, d_oc, d.N, d.L, geom, d.padded);
  else
    gated_merge_bwd_kernel<float, 64><<<grid, 256, 0, s>>>((const float*)dout, gate_logits, (const float*)oc,
                                                           d_logits, d_oc, d.N, d.L, geom, d.padded);
  return check_launch("gated_merge_bwd_kernel");
}

namespace {
template <typename T, int D>
void launch_pad_bwd(const Dims& d, const void* oc, const float* lse_c, const float* d_oc, char* ws, const WsLayout& w,
                    cudaStream_t s) {
  const int Lc = kTile * w.Nc_tiles;
  coarse_pad_bwd_kernel<T, D><<<dim3((Lc + 7) / 8, d.BH), 256, 0, s>>>(
      (const T*)oc, lse_c, d_oc, (T*)(ws + w.oc), (float*)(ws + w.lse_c), (T*)(ws + w.doc), d.N, Lc);
}
}  // namespace

vsa2_status launch_coarse_attn_bwd(const Dims& d, const void* q, const void* k, const void* v, const void* oc,
                                   const float* lse_c, const float* d_oc, float* dq, float* dk, float* dv, char* ws,
                                   cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  const int Nc = w.Nc_tiles;
  const int Lc = kTile * Nc;
  Dims dc = d;
  dc.L = Lc;
  dc.N = Nc;
  dc.Lr = Lc / kPool;
  dc.padded = false;  // the pooled sequence is dense (its zero rows past N add nothing)
  // the backward of the pooled sequence keeps its Delta and LSE where ws_layout(dc) puts them;
  // every region of dc is at most the size of d's, so they end before the coarse regions
  if (ws_layout(dc).nlse2 + align256((size_t)dc.BH * Lc * 4) > w.qc) return VSA2_ERR_UNSUPPORTED;
  // pooled operands (Eq. 1) again (over the real tokens of a padded grid), the padded O_c_hat,
  // LSE and dO_c_hat, and the dense CSR / CSC
  uint64_t* tmask = nullptr;
  if (d.padded) {
    tmask = reinterpret_cast<uint64_t*>(ws + w.tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
  }
  if (d.dtype == VSA2_BF16 && d.D == 128) {
    launch_pool<__nv_bfloat16, 128>(d, q, k, v, ws, w, tmask, s);
    launch_pad_bwd<__nv_bfloat16, 128>(d, oc, lse_c, d_oc, ws, w, s);
  } else if (d.dtype == VSA2_BF16) {
    launch_pool<__nv_bfloat16, 64>(d, q, k, v, ws, w, tmask, s);
    launch_pad_bwd<__nv_bfloat16, 64>(d, oc, lse_c, d_oc, ws, w, s);
  } else if (d.D == 128) {
    launch_pool<float, 128>(d, q, k, v, ws, w, tmask, s);
    launch_pad_bwd<float, 128>(d, oc, lse_c, d_oc, ws, w, s);
  } else {
    launch_pool<float, 64>(d, q, k, v, ws, w, tmask, s);
    launch_pad_bwd<float, 64>(d, oc, lse_c, d_oc, ws, w, s);
  }
  int32_t* c_off = reinterpret_cast<int32_t*>(ws + w.c_off);
  int32_t* c_idx = reinterpret_cast<int32_t*>(ws + w.c_idx);
  coarse_csr_kernel<<<d.BH, 256, 0, s>>>(Nc, c_off, c_idx);
  vsa2_status st = check_launch("coarse backward: pooling and padding");
  if (st != VSA2_OK) return st;
  // gradients of Eq. 2-3 over the pooled sequence; every tile lists every tile, so the CSC
  // equals the CSR
  float* dqc = reinterpret_cast<float*>(ws + w.dqc);
  float* dkc = reinterpret_cast<float*>(ws + w.dkc);
  float* dvc = reinterpret_cast<float*>(ws + w.dvc);
  st = launch_attn_bwd(dc, ws + w.qc, ws + w.kc, ws + w.vc, ws + w.oc, reinterpret_cast<const float*>(ws + w.lse_c),
                       ws + w.doc, Nc, c_off, c_idx, c_off, c_idx, dqc, dkc, dvc, ws, s);
  if (st != VSA2_OK) return st;
  // MeanPool_B's adjoint, added to the caller's gradients
  const int64_t rows = (int64_t)d.BH * d.L;
  coarse_pool_bwd_kernel<<<grid_for(rows * (d.D / 4), 256), 256, 0, s>>>(dqc, dkc, dvc, dq, dk, dv, rows, d.L, Lc,
                                                                         d.D, tmask);
  return check_launch("coarse_pool_bwd_kernel");
}

vsa2_status launch_gated_merge(const Dims& d, const void* o_f, const float* gate_logits, const void* oc, void* o,
                               cudaStream_t s) {
  const int64_t rows = (int64_t)d.BH * d.L;
  if (d.dtype == VSA2_BF16) {
    const int64_t chunks = rows * (d.D / 8);
    gated_merge_kernel<__nv_bfloat16><<<grid_for(chunks, 256), 256, 0, s>>>(
        (const __nv_bfloat16*)o_f, gate_logits, (const __nv_bfloat16*)oc, (__nv_bfloat16*)o, rows, d.L, d.N, d.D);
  } else {
    const int64_t chunks = rows * (d.D / 4);
    gated_merge_kernel<float><<<grid_for(chunks, 256), 256, 0, s>>>((const float*)o_f, gate_logits, (const float*)oc,
                                                                    (float*)o, rows, d.L, d.N, d.D);
  }
  return check_launch("gated_merge_kernel");
}

}  // namespace vsa2
