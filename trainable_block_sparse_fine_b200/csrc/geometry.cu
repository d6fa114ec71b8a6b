// Token grids that the tile does not divide ("Improving Video Sparse Attention with
// Fine-grained Router and Sparse Rebasing", §2.2 "Kernel Implementation": every dimension is
// padded to a multiple of the tile and the padding is masked). The padded grid is laid out in
// cube-major order like any other; this kernel marks, for every tile, which of its 64 tokens
// belong to the real grid. The router, the forward and the coarse branch read these masks.
#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

// One thread per tile: bit u of mask[i] is set when cube-major token u of tile i lies inside
// the real grid.
__global__ void __launch_bounds__(256) tile_mask_kernel(GridGeom g, int N, uint64_t* __restrict__ mask) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  uint64_t m = 0;
  for (int u = 0; u < 64; ++u)
    if (token_real(g, i, u)) m |= 1ull << u;
  mask[i] = m;
}

// 128-token tiles: a list (CSR over query tiles, or CSC over KV tiles) at tile granularity
// becomes one over 64-token tiles. Tile I is 64-tiles 2I and 2I+1 (consecutive in cube-major
// order), so 64-tile u takes 2J, 2J+1 for every J of list u / 2, in order. One warp per 64-tile.
// Offsets of a broken list are written as -1 (the attention kernels report and skip such rows).
__global__ void __launch_bounds__(256) expand_lists_kernel(const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ idx, int N, int topk,
                                                           int rows64, int32_t* __restrict__ off64,
                                                           int32_t* __restrict__ idx64) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows64) return;
  const int n64 = 2 * N;
  const int bh = r / n64, u = r - bh * n64, I = u >> 1;
  const int cap = N * topk;
  const int b = off[(size_t)bh * (N + 1) + I], e = off[(size_t)bh * (N + 1) + I + 1];
  int32_t* o64 = off64 + (size_t)bh * (n64 + 1);
  if (b < 0 || e < b || e > cap || e - b > N) {
    if (lane == 0) {
      o64[u] = -1;
      if (u == n64 - 1) o64[n64] = -1;
    }
    return;
  }
  const int len = e - b, start = 4 * b + 2 * (u & 1) * len;
  if (lane == 0) {
    o64[u] = start;
    if (u == n64 - 1) o64[n64] = 4 * e;
  }
  const int32_t* src = idx + (size_t)bh * cap + b;
  int32_t* dst = idx64 + (size_t)bh * 4 * cap + start;
  for (int k = lane; k < len; k += 32) {
    const int J = src[k];
    dst[2 * k] = 2 * J;
    dst[2 * k + 1] = 2 * J + 1;
  }
}

}  // namespace

vsa2_status launch_expand_lists(const Dims& d, int topk, const int32_t* off, const int32_t* idx, int32_t* off64,
                                int32_t* idx64, cudaStream_t s) {
  const int rows64 = d.BH * 2 * d.N;
  expand_lists_kernel<<<(rows64 + 7) / 8, 256, 0, s>>>(off, idx, d.N, topk, rows64, off64, idx64);
  return check_launch("expand_lists_kernel");
}

vsa2_status launch_tile_masks(const Dims& d, uint64_t* mask, cudaStream_t s) {
  tile_mask_kernel<<<(d.N + 255) / 256, 256, 0, s>>>(grid_geom(d), d.N, mask);
  return check_launch("tile_mask_kernel");
}

}  // namespace vsa2
