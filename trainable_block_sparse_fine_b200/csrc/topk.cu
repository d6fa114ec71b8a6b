// Per-sequence TopK of VSA2 ("Improving Video Sparse Attention with Fine-grained Router and
// Sparse Rebasing", §2.2 Eq. 8-9): per (b, h) keep the N*K largest of the N*N tile scores.
//
// Exact radix select on the fp32 bit patterns (scores are >= 0, so unsigned order equals
// float order): three histograms over 11/11/10-bit digits find the threshold T and how many
// entries equal to T still fit the budget. Ties at T go to the lowest flat index i*N+j: a
// per-row scan assigns the tie quota row by row, then each row is compacted in ascending j
// (CSR). The CSC used by the backward pass is built from a per-column bitmap, so both lists
// are deterministic. The third histogram is formed in the same pass over the scores as the
// per-row counts: that pass counts, per row, the entries whose top 22 bits exceed the prefix
// found so far, and lists the few entries that share it (row and low 10 bits) for a small fix-up
// once T is known; when a head has more of them than the list holds (heavy ties), a full
// recount against T takes over.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

enum { ST_PREFIX = 0, ST_REMAIN = 1, ST_THRESH = 2, ST_TIES = 3 };

__device__ __forceinline__ uint32_t score_key(float s) { return __float_as_uint(s) & 0x7FFFFFFFu; }

// Exclusive scan over a 1024-thread block; returns this thread's exclusive prefix, *total the sum.
__device__ __forceinline__ uint32_t block_scan_excl_1024(uint32_t v, uint32_t* sh32, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh32[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = sh32[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh32[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t warp_base = warp ? sh32[warp - 1] : 0u;
  *total = sh32[31];
  __syncthreads();
  return warp_base + x - v;
}

template <int PASS>
__global__ void __launch_bounds__(512) topk_hist_kernel(const float* __restrict__ scores, int64_t nn,
                                                        const uint32_t* __restrict__ state, uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[2048];
  const int bh = blockIdx.y;
  for (int b = threadIdx.x; b < 2048; b += blockDim.x) h[b] = 0;
  __syncthreads();
  const uint32_t prefix = PASS == 0 ? 0u : state[bh * 8 + ST_PREFIX];
  const float* s = scores + (size_t)bh * nn;
  const int64_t per = (((nn + gridDim.x - 1) / gridDim.x) + 3) & ~int64_t(3);
  const int64_t beg = (int64_t)blockIdx.x * per;
  const int64_t end = beg + per < nn ? beg + per : nn;
  if (beg >= end) return;
  auto add = [&](float v) {
    const uint32_t key = score_key(v);
    if (PASS == 0) {
      atomicAdd(&h[key >> 21], 1u);
    } else if (PASS == 1) {
      if ((key >> 21) == prefix) atomicAdd(&h[(key >> 10) & 2047u], 1u);
    } else {
      if ((key >> 10) == prefix) atomicAdd(&h[key & 1023u], 1u);
    }
  };
  if (((reinterpret_cast<uintptr_t>(s + beg)) & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(s + beg);
    const int64_t n4 = (end - beg) >> 2;
    for (int64_t x = threadIdx.x; x < n4; x += blockDim.x) {
      const float4 v = __ldg(s4 + x);
      add(v.x), add(v.y), add(v.z), add(v.w);
    }
    for (int64_t x = beg + 4 * n4 + threadIdx.x; x < end; x += blockDim.x) add(__ldg(s + x));
  } else {
    for (int64_t x = beg + threadIdx.x; x < end; x += blockDim.x) add(__ldg(s + x));
  }
  __syncthreads();
  uint32_t* gh = hist + ((size_t)bh * 3 + PASS) * 2048;
  for (int b = threadIdx.x; b < 2048; b += blockDim.x)
    if (h[b]) atomicAdd(&gh[b], h[b]);
}

// Pick the digit whose bin holds the budget boundary; update prefix and remaining count.
template <int PASS>
__global__ void __launch_bounds__(1024) topk_select_digit_kernel(const uint32_t* __restrict__ hist,
                                                                 uint32_t* __restrict__ state, uint32_t budget) {
  __shared__ uint32_t sh32[32];
  const int bh = blockIdx.x, t = threadIdx.x;
  constexpr int NB = PASS == 2 ? 1024 : 2048;
  constexpr int BITS = PASS == 2 ? 10 : 11;
  const uint32_t* gh = hist + ((size_t)bh * 3 + PASS) * 2048;
  const uint32_t prefix = PASS == 0 ? 0u : state[bh * 8 + ST_PREFIX];
  const uint32_t remain = PASS == 0 ? budget : state[bh * 8 + ST_REMAIN];
  // descending bin order: thread t owns bins NB-1-2t and NB-2-2t (or one bin when NB == 1024)
  constexpr int PER = NB / 1024;
  uint32_t c[PER];
  uint32_t mine = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    c[e] = gh[NB - 1 - (PER * t + e)];
    mine += c[e];
  }
  uint32_t total;
  uint32_t above = block_scan_excl_1024(mine, sh32, &total);  // count in bins above this thread's
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    if (above < remain && above + c[e] >= remain) {
      const uint32_t digit = (uint32_t)(NB - 1 - (PER * t + e));
      const uint32_t np = (prefix << BITS) | digit;
      state[bh * 8 + ST_PREFIX] = np;
      state[bh * 8 + ST_REMAIN] = remain - above;
      if (PASS == 2) {
        state[bh * 8 + ST_THRESH] = np;
        state[bh * 8 + ST_TIES] = remain - above;
      }
    }
    above += c[e];
  }
}

// Warp per row: entries above the threshold and entries equal to it.
// Every row of a scores block starts on a 16-byte boundary when the block itself does and N is
// a multiple of 4; then rows are read as float4.
__device__ __forceinline__ bool rows_vec4(const float* scores, int N) {
  return (N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
}

// With cand_cnt, the recount runs only for heads whose candidate list overflowed.
__global__ void __launch_bounds__(256) topk_row_count_kernel(const float* __restrict__ scores, int N,
                                                             const uint32_t* __restrict__ state,
                                                             int32_t* __restrict__ row_gt, int32_t* __restrict__ row_eq,
                                                             const uint32_t* __restrict__ cand_cnt) {
  const int bh = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= N) return;
  if (cand_cnt && cand_cnt[bh] <= (uint32_t)kCandCap) return;
  const uint32_t T = state[bh * 8 + ST_THRESH];
  const float* s = scores + ((size_t)bh * N + row) * N;
  int gt = 0, eq = 0;
  if (rows_vec4(scores, N)) {  // four columns per lane and load
    const float4* s4 = reinterpret_cast<const float4*>(s);
#pragma unroll 4
    for (int q = lane; q < (N >> 2); q += 32) {
      const float4 v = __ldg(s4 + q);
      const uint32_t k0 = score_key(v.x), k1 = score_key(v.y), k2 = score_key(v.z), k3 = score_key(v.w);
      gt += (k0 > T) + (k1 > T) + (k2 > T) + (k3 > T);
      eq += (k0 == T) + (k1 == T) + (k2 == T) + (k3 == T);
    }
  } else {
    for (int j = lane; j < N; j += 32) {
      const uint32_t key = score_key(__ldg(s + j));
      gt += key > T;
      eq += key == T;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    row_gt[(size_t)bh * N + row] = gt;
    row_eq[(size_t)bh * N + row] = eq;
  }
}

// Warp per row, after the second digit: entries whose top 22 bits exceed the prefix P22 (row_gt),
// and the entries equal to it: their low 10 bits go to the third histogram and, with the row, to
// the head's candidate list (the count goes on past kCandCap to flag an overflow).
__global__ void __launch_bounds__(256) topk_row_count22_kernel(const float* __restrict__ scores, int N,
                                                               const uint32_t* __restrict__ state,
                                                               int32_t* __restrict__ row_gt, int32_t* __restrict__ row_eq,
                                                               uint32_t* __restrict__ hist, uint32_t* __restrict__ cand,
                                                               uint32_t* __restrict__ cand_cnt) {
  const int bh = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= N) return;
  const uint32_t P = state[bh * 8 + ST_PREFIX];
  const float* s = scores + ((size_t)bh * N + row) * N;
  uint32_t* h2 = hist + ((size_t)bh * 3 + 2) * 2048;
  int gt = 0;
  auto cand_add = [&](uint32_t key) {
    atomicAdd(&h2[key & 1023u], 1u);
    const uint32_t at = atomicAdd(&cand_cnt[bh], 1u);
    if (at < (uint32_t)kCandCap) cand[(size_t)bh * kCandCap + at] = ((uint32_t)row << 10) | (key & 1023u);
  };
  if (rows_vec4(scores, N)) {
    const float4* s4 = reinterpret_cast<const float4*>(s);
#pragma unroll 4
    for (int q = lane; q < (N >> 2); q += 32) {
      const float4 v = __ldg(s4 + q);
      const uint32_t k[4] = {score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t p = k[e] >> 10;
        gt += p > P;
        if (p == P) cand_add(k[e]);
      }
    }
  } else {
    for (int j = lane; j < N; j += 32) {
      const uint32_t key = score_key(__ldg(s + j));
      gt += (key >> 10) > P;
      if ((key >> 10) == P) cand_add(key);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  if (lane == 0) {
    row_gt[(size_t)bh * N + row] = gt;
    row_eq[(size_t)bh * N + row] = 0;
  }
}

// Per (b, h), once T is known: the listed candidates above T join their row's count, those equal
// to T its ties. Heads whose list overflowed are recounted in full instead.
__global__ void __launch_bounds__(256) topk_cand_fix_kernel(const uint32_t* __restrict__ state,
                                                            const uint32_t* __restrict__ cand,
                                                            const uint32_t* __restrict__ cand_cnt, int N,
                                                            int32_t* __restrict__ row_gt, int32_t* __restrict__ row_eq) {
  const int bh = blockIdx.x;
  const uint32_t n = cand_cnt[bh];
  if (n > (uint32_t)kCandCap) return;
  const uint32_t d = state[bh * 8 + ST_THRESH] & 1023u;
  for (uint32_t c = threadIdx.x; c < n; c += blockDim.x) {
    const uint32_t e = cand[(size_t)bh * kCandCap + c];
    const uint32_t row = e >> 10, low = e & 1023u;
    if (low > d) atomicAdd(&row_gt[(size_t)bh * N + row], 1);
    else if (low == d) atomicAdd(&row_eq[(size_t)bh * N + row], 1);
  }
}

// Per (b, h): hand the tie quota to rows in order and build the CSR row offsets.
__global__ void __launch_bounds__(1024) topk_offsets_kernel(int N, const uint32_t* __restrict__ state,
                                                            const int32_t* __restrict__ row_gt,
                                                            const int32_t* __restrict__ row_eq,
                                                            int32_t* __restrict__ row_take, int32_t* __restrict__ kv_off) {
  __shared__ uint32_t sh32[32];
  const int bh = blockIdx.x, t = threadIdx.x;
  const uint32_t ties = state[bh * 8 + ST_TIES];
  uint32_t eq_carry = 0, cnt_carry = 0;
  for (int base = 0; base < N; base += 1024) {
    const int i = base + t;
    const uint32_t gt = i < N ? (uint32_t)row_gt[(size_t)bh * N + i] : 0u;
    const uint32_t eq = i < N ? (uint32_t)row_eq[(size_t)bh * N + i] : 0u;
    uint32_t eq_tot;
    const uint32_t eq_before = eq_carry + block_scan_excl_1024(eq, sh32, &eq_tot);
    uint32_t take = 0;
    if (ties > eq_before) take = min(eq, ties - eq_before);
    const uint32_t cnt = gt + take;
    uint32_t cnt_tot;
    const uint32_t off = cnt_carry + block_scan_excl_1024(cnt, sh32, &cnt_tot);
    if (i < N) {
      row_take[(size_t)bh * N + i] = (int32_t)take;
      kv_off[(size_t)bh * (N + 1) + i] = (int32_t)off;
    }
    eq_carry += eq_tot;
    cnt_carry += cnt_tot;
  }
  if (t == 0) kv_off[(size_t)bh * (N + 1) + N] = (int32_t)cnt_carry;
}

// Warp per row: compact the selected KV tiles in ascending j; optionally mark the CSC bitmap.
__global__ void __launch_bounds__(256) topk_emit_kernel(const float* __restrict__ scores, int N, int topk,
                                                        const uint32_t* __restrict__ state,
                                                        const int32_t* __restrict__ row_take,
                                                        const int32_t* __restrict__ kv_off, int32_t* __restrict__ kv_idx,
                                                        int32_t* __restrict__ col_cnt, uint32_t* __restrict__ col_bits,
                                                        int words, DevCtx ctx) {
  const int bh = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= N) return;
  const uint32_t T = state[bh * 8 + ST_THRESH];
  const int take = row_take[(size_t)bh * N + row];
  const int base = kv_off[(size_t)bh * (N + 1) + row];
  const int next = kv_off[(size_t)bh * (N + 1) + row + 1];
  const float* s = scores + ((size_t)bh * N + row) * N;
  int32_t* out = kv_idx + (size_t)bh * N * topk;
  int written = 0, ties_seen = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  if (rows_vec4(scores, N)) {
    // four consecutive columns per lane (lane-major order is column order): per element slot one
    // ballot for ties and one for selections; positions add the lower lanes' counts to the
    // lane's own prefix
    const float4* s4 = reinterpret_cast<const float4*>(s);
#pragma unroll 2
    for (int j0 = 0; j0 < N; j0 += 128) {
      const int jl = j0 + 4 * lane;
      const bool valid = jl < N;
      const float4 v = valid ? __ldg(s4 + (jl >> 2)) : make_float4(0.f, 0.f, 0.f, 0.f);
      const uint32_t key[4] = {score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w)};
      uint32_t eqm[4];
      int ties_before = ties_seen;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        eqm[e] = __ballot_sync(0xffffffffu, valid && key[e] == T);
        ties_before += __popc(eqm[e] & lt_mask);
      }
      bool sel[4];
      int tr = ties_before;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool is_eq = valid && key[e] == T;
        sel[e] = valid && (key[e] > T || (is_eq && tr < take));
        tr += is_eq;
      }
      int pos = base + written, nsel = 0, nties = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t selm = __ballot_sync(0xffffffffu, sel[e]);
        pos += __popc(selm & lt_mask);
        nsel += __popc(selm);
        nties += __popc(eqm[e]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!sel[e]) continue;
        const int j = jl + e;
        if (pos < next) out[pos] = j;
        ++pos;
        if (col_cnt) {
          atomicAdd(&col_cnt[(size_t)bh * N + j], 1);
          atomicOr(&col_bits[((size_t)bh * N + j) * words + (row >> 5)], 1u << (row & 31));
        }
      }
      written += nsel;
      ties_seen += nties;
    }
    if ((ctx.flags & VSA2_FLAG_VALIDATE) && lane == 0 && base + written != next) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return;
  }
  for (int j0 = 0; j0 < N; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < N ? score_key(__ldg(s + j)) : 0u;
    const bool is_eq = j < N && key == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int tie_rank = ties_seen + __popc(eq_mask & lt_mask);
    const bool sel = j < N && (key > T || (is_eq && tie_rank < take));
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = base + written + __popc(sel_mask & lt_mask);
      if (pos < next) out[pos] = j;
      if (col_cnt) {
        atomicAdd(&col_cnt[(size_t)bh * N + j], 1);
        atomicOr(&col_bits[((size_t)bh * N + j) * words + (row >> 5)], 1u << (row & 31));
      }
    }
    written += __popc(sel_mask);
    ties_seen += __popc(eq_mask);
  }
  if ((ctx.flags & VSA2_FLAG_VALIDATE) && lane == 0 && base + written != next) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
}

__global__ void __launch_bounds__(1024) topk_csc_offsets_kernel(int N, const int32_t* __restrict__ col_cnt,
                                                                int32_t* __restrict__ q_off) {
  __shared__ uint32_t sh32[32];
  const int bh = blockIdx.x, t = threadIdx.x;
  uint32_t carry = 0;
  for (int base = 0; base < N; base += 1024) {
    const int j = base + t;
    const uint32_t c = j < N ? (uint32_t)col_cnt[(size_t)bh * N + j] : 0u;
    uint32_t tot;
    const uint32_t off = carry + block_scan_excl_1024(c, sh32, &tot);
    if (j < N) q_off[(size_t)bh * (N + 1) + j] = (int32_t)off;
    carry += tot;
  }
  if (t == 0) q_off[(size_t)bh * (N + 1) + N] = (int32_t)carry;
}

// Warp per KV tile j: list the query tiles of its bitmap in ascending order.
__global__ void __launch_bounds__(256) topk_csc_emit_kernel(int N, int topk, const uint32_t* __restrict__ col_bits,
                                                            int words, const int32_t* __restrict__ q_off,
                                                            int32_t* __restrict__ q_idx) {
  const int bh = blockIdx.y;
  const int col = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (col >= N) return;
  const uint32_t* bits = col_bits + ((size_t)bh * N + col) * words;
  int32_t* out = q_idx + (size_t)bh * N * topk + q_off[(size_t)bh * (N + 1) + col];
  int carry = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t b = w < words ? bits[w] : 0u;
    const int cnt = __popc(b);
    int x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int pos = carry + x - cnt;
    while (b) {
      const int bit = __ffs(b) - 1;
      out[pos++] = 32 * w + bit;
      b &= b - 1;
    }
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
}

// Exclusive scan over a 256-thread block; returns this thread's exclusive prefix, *total the sum.
__device__ __forceinline__ uint32_t block_scan_excl_256(uint32_t v, uint32_t* sh8, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh8[warp] = x;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const uint32_t c = sh8[w];
    base += w < warp ? c : 0u;
    tot += c;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

// Per-query-tile TopK (VSA's selection, the variant that Eq. 8-9 replace): one 256-thread CTA
// per row keeps the row's `topk` largest scores. Exact radix select over the row's fp32 bit
// patterns in three passes (11/11/10 bits); equal scores go to the lower KV tile. The row is
// read from global memory on every pass (it stays in L1: N*4 bytes). Writes the row's CSR
// entries in ascending j and, with col_cnt, marks the CSC bitmap like topk_emit_kernel.
__global__ void __launch_bounds__(256) topk_row_select_kernel(const float* __restrict__ scores, int N, int topk,
                                                              int32_t* __restrict__ kv_off,
                                                              int32_t* __restrict__ kv_idx,
                                                              int32_t* __restrict__ col_cnt,
                                                              uint32_t* __restrict__ col_bits, int words) {
  __shared__ uint32_t h[2048];
  __shared__ uint32_t sh8[8];
  __shared__ uint32_t s_prefix, s_remain;
  const int bh = blockIdx.y, row = blockIdx.x, t = threadIdx.x;
  const float* s = scores + ((size_t)bh * N + row) * N;
  uint32_t prefix = 0, remain = (uint32_t)topk;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    for (int b = t; b < 2048; b += 256) h[b] = 0;
    __syncthreads();
    for (int j = t; j < N; j += 256) {
      const uint32_t key = score_key(__ldg(s + j));
      if (pass == 0) atomicAdd(&h[key >> 21], 1u);
      else if (pass == 1) {
        if ((key >> 21) == prefix) atomicAdd(&h[(key >> 10) & 2047u], 1u);
      } else if ((key >> 10) == prefix) {
        atomicAdd(&h[key & 1023u], 1u);
      }
    }
    __syncthreads();
    // descending bins: thread t owns bins NB-1-PER*t-e, e < PER
    const int NB = pass == 2 ? 1024 : 2048, PER = NB / 256, BITS = pass == 2 ? 10 : 11;
    uint32_t c[8], mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = e < PER ? h[NB - 1 - (PER * t + e)] : 0u;
      mine += c[e];
    }
    uint32_t tot;
    uint32_t above = block_scan_excl_256(mine, sh8, &tot);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (e < PER && above < remain && above + c[e] >= remain) {
        s_prefix = (prefix << BITS) | (uint32_t)(NB - 1 - (PER * t + e));
        s_remain = remain - above;
      }
      above += c[e];
    }
    __syncthreads();
    prefix = s_prefix;
    remain = s_remain;
    __syncthreads();
  }
  const uint32_t T = prefix, ties = remain;  // threshold key; entries equal to it still taken
  int32_t* out = kv_idx + (size_t)bh * N * topk + (size_t)row * topk;
  uint32_t written = 0, ties_seen = 0;
  for (int j0 = 0; j0 < N; j0 += 256) {
    const int j = j0 + t;
    const uint32_t key = j < N ? score_key(__ldg(s + j)) : 0u;
    const bool is_eq = j < N && key == T;
    uint32_t eq_tot, sel_tot;
    const uint32_t rank = ties_seen + block_scan_excl_256(is_eq, sh8, &eq_tot);
    const bool sel = j < N && (key > T || (is_eq && rank < ties));
    const uint32_t pos = written + block_scan_excl_256(sel, sh8, &sel_tot);
    if (sel) {
      if (pos < (uint32_t)topk) out[pos] = j;
      if (col_cnt) {
        atomicAdd(&col_cnt[(size_t)bh * N + j], 1);
        atomicOr(&col_bits[((size_t)bh * N + j) * words + (row >> 5)], 1u << (row & 31));
      }
    }
    written += sel_tot;
    ties_seen += eq_tot;
  }
  if (t == 0) {
    kv_off[(size_t)bh * (N + 1) + row] = row * topk;
    if (row == N - 1) kv_off[(size_t)bh * (N + 1) + N] = N * topk;
  }
}

}  // namespace

vsa2_status launch_topk_per_row(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                                int32_t* q_off, int32_t* q_idx, char* ws, cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  int32_t* col_cnt = reinterpret_cast<int32_t*>(ws + w.col_cnt);
  uint32_t* col_bits = reinterpret_cast<uint32_t*>(ws + w.col_bits);
  const bool csc = q_off != nullptr;
  if (csc) {
    if (cudaMemsetAsync(col_cnt, 0, (size_t)d.BH * d.N * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
    if (cudaMemsetAsync(col_bits, 0, (size_t)d.BH * d.N * w.words * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
  }
  topk_row_select_kernel<<<dim3(d.N, d.BH), 256, 0, s>>>(scores, d.N, topk, kv_off, kv_idx, csc ? col_cnt : nullptr,
                                                         col_bits, w.words);
  if (csc) {
    dim3 rgrid((d.N + 7) / 8, d.BH);
    topk_csc_offsets_kernel<<<d.BH, 1024, 0, s>>>(d.N, col_cnt, q_off);
    topk_csc_emit_kernel<<<rgrid, 256, 0, s>>>(d.N, topk, col_bits, w.words, q_off, q_idx);
  }
  return check_launch(__func__);
}

vsa2_status launch_topk(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                        int32_t* q_off, int32_t* q_idx, char* ws, cudaStream_t s) {
  const WsLayout w = ws_layout(d);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + w.hist);
  uint32_t* state = reinterpret_cast<uint32_t*>(ws + w.state);
  int32_t* row_gt = reinterpret_cast<int32_t*>(ws + w.row_gt);
  int32_t* row_eq = reinterpret_cast<int32_t*>(ws + w.row_eq);
  int32_t* row_take = reinterpret_cast<int32_t*>(ws + w.row_take);
  int32_t* col_cnt = reinterpret_cast<int32_t*>(ws + w.col_cnt);
  uint32_t* col_bits = reinterpret_cast<uint32_t*>(ws + w.col_bits);
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const bool csc = q_off != nullptr;
  const int64_t nn = (int64_t)d.N * d.N;
  const uint32_t budget = (uint32_t)d.N * (uint32_t)topk;

  uint32_t* cand = reinterpret_cast<uint32_t*>(ws + w.cand);
  uint32_t* cand_cnt = reinterpret_cast<uint32_t*>(ws + w.cand_cnt);
  if (cudaMemsetAsync(hist, 0, (size_t)d.BH * 3 * 2048 * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
  if (cudaMemsetAsync(cand_cnt, 0, (size_t)d.BH * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
  if (csc) {
    if (cudaMemsetAsync(col_cnt, 0, (size_t)d.BH * d.N * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
    if (cudaMemsetAsync(col_bits, 0, (size_t)d.BH * d.N * w.words * 4, s) != cudaSuccess) return VSA2_ERR_CUDA;
  }
  int per_head = (int)((nn + 16383) / 16384);
  const int cap = (148 * 8 + d.BH - 1) / d.BH;
  if (per_head > cap) per_head = cap;
  if (per_head < 1) per_head = 1;
  dim3 hgrid(per_head, d.BH);
  topk_hist_kernel<0><<<hgrid, 512, 0, s>>>(scores, nn, state, hist);
  topk_select_digit_kernel<0><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  topk_hist_kernel<1><<<hgrid, 512, 0, s>>>(scores, nn, state, hist);
  topk_select_digit_kernel<1><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  dim3 rgrid((d.N + 7) / 8, d.BH);
  topk_row_count22_kernel<<<rgrid, 256, 0, s>>>(scores, d.N, state, row_gt, row_eq, hist, cand, cand_cnt);
  topk_select_digit_kernel<2><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  topk_cand_fix_kernel<<<d.BH, 256, 0, s>>>(state, cand, cand_cnt, d.N, row_gt, row_eq);
  topk_row_count_kernel<<<rgrid, 256, 0, s>>>(scores, d.N, state, row_gt, row_eq, cand_cnt);  // overflow only
  topk_offsets_kernel<<<d.BH, 1024, 0, s>>>(d.N, state, row_gt, row_eq, row_take, kv_off);
  topk_emit_kernel<<<rgrid, 256, 0, s>>>(scores, d.N, topk, state, row_take, kv_off, kv_idx,
                                         csc ? col_cnt : nullptr, col_bits, w.words, ctx);
  if (csc) {
    topk_csc_offsets_kernel<<<d.BH, 1024, 0, s>>>(d.N, col_cnt, q_off);
    topk_csc_emit_kernel<<<rgrid, 256, 0, s>>>(d.N, topk, col_bits, w.words, q_off, q_idx);
  }
  if (check_launch(__func__) != VSA2_OK) return VSA2_ERR_CUDA;
  return VSA2_OK;
}

// ------------------------------------------------------------------------------------------
// Allocation-free variant (CSR only). Its scratch is a fixed array in the library's device
// image instead of a caller workspace; see vsa2_topk_select_noalloc in vsa2.h.
// ------------------------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
__device__ __align__(256) unsigned char g_topk_scratch[kNoAllocScratchBytes];

struct NoAllocLayout {
  size_t err, hist, state, row_gt, row_eq, row_take, total;
};
NoAllocLayout noalloc_layout(const Dims& d) {
  NoAllocLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  l.err = take(sizeof(int));
  l.hist = take((size_t)d.BH * 3 * 2048 * 4);
  l.state = take((size_t)d.BH * 8 * 4);
  l.row_gt = take((size_t)d.BH * d.N * 4);
  l.row_eq = take((size_t)d.BH * d.N * 4);
  l.row_take = take((size_t)d.BH * d.N * 4);
  l.total = off;
  return l;
}

std::mutex g_scratch_mu;
struct ScratchSlot {
  unsigned long long ctx_id;  // context the address belongs to (0: unknown)
  void* ptr;                  // device address of g_topk_scratch in that context
};
ScratchSlot g_scratch[64] = {};  // per device ordinal

// Device address of the scratch array for the current device, looked up with that device
// current (cudaGetSymbolAddress; the host-side symbol is not a device address). The address is
// kept per device and per context: a context that replaced the one it was taken in (after
// cudaDeviceReset, say) gets a fresh lookup. If the context id cannot be read, every call looks
// the address up again.
vsa2_status noalloc_scratch(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess)
    return cuda_fail("cudaGetDevice failed");
  if (dev < 0 || dev >= 64) return cuda_fail("device ordinal out of range for the TopK scratch table");
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (!have_id || !slot.ptr || slot.ctx_id != id) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_topk_scratch) != cudaSuccess || !ptr)
      return cuda_fail("cudaGetSymbolAddress of the TopK scratch array failed");
    slot.ptr = ptr;
    slot.ctx_id = have_id ? id : 0;
  }
  *out = static_cast<char*>(slot.ptr);
  return VSA2_OK;
}
}  // namespace

size_t topk_noalloc_bytes(const Dims& d) { return noalloc_layout(d).total; }
size_t topk_noalloc_capacity() { return kNoAllocScratchBytes; }

vsa2_status launch_topk_noalloc(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                                cudaStream_t s) {
  const NoAllocLayout w = noalloc_layout(d);
  if (w.total > kNoAllocScratchBytes) return VSA2_ERR_UNSUPPORTED;
  char* base = nullptr;
  vsa2_status st = noalloc_scratch(&base);
  if (st != VSA2_OK) return st;
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + w.hist);
  uint32_t* state = reinterpret_cast<uint32_t*>(base + w.state);
  int32_t* row_gt = reinterpret_cast<int32_t*>(base + w.row_gt);
  int32_t* row_eq = reinterpret_cast<int32_t*>(base + w.row_eq);
  int32_t* row_take = reinterpret_cast<int32_t*>(base + w.row_take);
  // validate-mode reports have nowhere to go without a workspace: the flag is ignored here
  DevCtx ctx{reinterpret_cast<int*>(base + w.err), d.timeout_ns, 0};
  const int64_t nn = (int64_t)d.N * d.N;
  const uint32_t budget = (uint32_t)d.N * (uint32_t)topk;
  // the array keeps the previous call's contents: the histograms must start at zero
  if (cudaMemsetAsync(base, 0, w.state, s) != cudaSuccess) return cuda_fail("cudaMemsetAsync of the TopK scratch failed");
  int per_head = (int)((nn + 16383) / 16384);
  const int cap = (148 * 8 + d.BH - 1) / d.BH;
  if (per_head > cap) per_head = cap;
  if (per_head < 1) per_head = 1;
  dim3 hgrid(per_head, d.BH);
  topk_hist_kernel<0><<<hgrid, 512, 0, s>>>(scores, nn, state, hist);
  topk_select_digit_kernel<0><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  topk_hist_kernel<1><<<hgrid, 512, 0, s>>>(scores, nn, state, hist);
  topk_select_digit_kernel<1><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  topk_hist_kernel<2><<<hgrid, 512, 0, s>>>(scores, nn, state, hist);
  topk_select_digit_kernel<2><<<d.BH, 1024, 0, s>>>(hist, state, budget);
  dim3 rgrid((d.N + 7) / 8, d.BH);
  topk_row_count_kernel<<<rgrid, 256, 0, s>>>(scores, d.N, state, row_gt, row_eq, nullptr);
  topk_offsets_kernel<<<d.BH, 1024, 0, s>>>(d.N, state, row_gt, row_eq, row_take, kv_off);
  topk_emit_kernel<<<rgrid, 256, 0, s>>>(scores, d.N, topk, state, row_take, kv_off, kv_idx, nullptr, nullptr, 0, ctx);
  return check_launch(__func__);
}

}  // namespace vsa2
