// Token permutation of "Improving Video Sparse Attention with Fine-grained Router and Sparse
// Rebasing", §2.2 "Permutation": raster order (t, h, w) <-> cube-major order (tiles in raster
// order over the tile grid; inside a tile its pooling sub-cubes in raster order; inside a
// sub-cube its tokens in raster order). A pure gather/scatter of D-element rows, HBM-bound:
// every row is read once and written once, 16 bytes per thread and iteration, so each group
// of D*esize/16 threads moves one whole row.
//
// A grid the tile does not divide is padded to whole tiles (§2.2 "Kernel Implementation"): the
// cube-major side then holds the padded grid, raster -> cube-major writes zeros in the padding
// rows, and cube-major -> raster drops them.
//
// The row index arithmetic divides by runtime constants (grid, tile and pool extents) eight
// times per row. To keep it off the critical path it uses division by invariant integers with
// a multiply-high and a shift (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", 1994, the round-up variant): for 1 <= d < 2^31 and s = ceil(log2 d),
// m = floor(2^32 (2^s - d) / d) + 1 gives n / d = (umulhi(n, m) + n) >> s for all n < 2^31.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

struct FastDiv {
  uint32_t d, m, s;
};

FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((uint64_t(1) << s) < d) ++s;
  const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
  return FastDiv{d, (uint32_t)m, s};
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) { return (__umulhi(n, f.m) + n) >> f.s; }

struct Geom {
  FastDiv L;                 // tokens per (b, h)
  FastDiv tile, pool;        // tokens per tile, per sub-cube
  FastDiv tiles_hw, tiles_w; // tile grid: tiles per t-slab, per h-row
  FastDiv subs_hw, subs_w;   // sub-cubes of a tile: per t-slab, per h-row
  FastDiv pool_hw, pool_w;   // tokens of a sub-cube: per t-slab, per h-row
  uint32_t bt, bh, bw, rt, rh, rw, gt, gh, gw;  // tile, sub-cube, real grid
  uint32_t Lr;                                    // real tokens per (b, h)
};

// raster index (t*H + h)*W + w (in the real grid) of the token at cube-major index l of a head,
// or UINT32_MAX for a padding token
__device__ __forceinline__ uint32_t raster_of(uint32_t l, const Geom& g) {
  const uint32_t i = fdiv(l, g.tile), in_tile = l - i * g.tile.d;
  const uint32_t sidx = fdiv(in_tile, g.pool), r = in_tile - sidx * g.pool.d;
  const uint32_t a = fdiv(i, g.tiles_hw), i2 = i - a * g.tiles_hw.d;
  const uint32_t b = fdiv(i2, g.tiles_w), c = i2 - b * g.tiles_w.d;
  const uint32_t st = fdiv(sidx, g.subs_hw), s2 = sidx - st * g.subs_hw.d;
  const uint32_t sh = fdiv(s2, g.subs_w), sw = s2 - sh * g.subs_w.d;
  const uint32_t dt = fdiv(r, g.pool_hw), r2 = r - dt * g.pool_hw.d;
  const uint32_t dh = fdiv(r2, g.pool_w), dw = r2 - dh * g.pool_w.d;
  const uint32_t t = a * g.bt + st * g.rt + dt;
  const uint32_t h = b * g.bh + sh * g.rh + dh;
  const uint32_t w = c * g.bw + sw * g.rw + dw;
  if (t >= g.gt || h >= g.gh || w >= g.gw) return 0xffffffffu;
  return (t * g.gh + h) * g.gw + w;
}

__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                      uint32_t rows, int ch_shift, Geom g, int to_cube) {
  const uint64_t total = (uint64_t)rows << ch_shift;
  const uint32_t ch_mask = (1u << ch_shift) - 1;
  for (uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total; c += (uint64_t)gridDim.x * blockDim.x) {
    const uint32_t row = (uint32_t)(c >> ch_shift), part = (uint32_t)c & ch_mask;
    const uint32_t bh = fdiv(row, g.L), l = row - bh * g.L.d;
    const uint32_t r = raster_of(l, g);
    if (r == 0xffffffffu) {  // a padding token: zeros on the cube-major side, nothing in raster order
      if (to_cube) dst[((uint64_t)row << ch_shift) + part] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint64_t raster_row = (uint64_t)bh * g.Lr + r;
    const uint64_t from = ((to_cube ? raster_row : (uint64_t)row) << ch_shift) + part;
    const uint64_t to = ((to_cube ? (uint64_t)row : raster_row) << ch_shift) + part;
    dst[to] = __ldg(src + from);
  }
}

}  // namespace

vsa2_status launch_permute(const Dims& d, const vsa2_problem* p, const void* src, void* dst, int to_cube,
                           cudaStream_t s) {
  const int row_bytes = d.D * d.esize;  // 128, 256 or 512
  int ch_shift = 0;
  while ((16 << ch_shift) < row_bytes) ++ch_shift;
  Geom g;
  g.L = make_fastdiv((uint32_t)d.L);
  g.tile = make_fastdiv((uint32_t)(p->tile_t * p->tile_h * p->tile_w));
  g.pool = make_fastdiv((uint32_t)(p->pool_t * p->pool_h * p->pool_w));
  const uint32_t nh = (uint32_t)((p->grid_h + p->tile_h - 1) / p->tile_h);  // tiles of the padded grid
  const uint32_t nw = (uint32_t)((p->grid_w + p->tile_w - 1) / p->tile_w);
  g.tiles_hw = make_fastdiv(nh * nw);
  g.tiles_w = make_fastdiv(nw);
  const uint32_t sh_n = (uint32_t)(p->tile_h / p->pool_h), sw_n = (uint32_t)(p->tile_w / p->pool_w);
  g.subs_hw = make_fastdiv(sh_n * sw_n);
  g.subs_w = make_fastdiv(sw_n);
  g.pool_hw = make_fastdiv((uint32_t)(p->pool_h * p->pool_w));
  g.pool_w = make_fastdiv((uint32_t)p->pool_w);
  g.bt = p->tile_t, g.bh = p->tile_h, g.bw = p->tile_w;
  g.rt = p->pool_t, g.rh = p->pool_h, g.rw = p->pool_w;
  g.gt = (uint32_t)p->grid_t, g.gh = (uint32_t)p->grid_h, g.gw = (uint32_t)p->grid_w;
  g.Lr = (uint32_t)(p->grid_t * p->grid_h * p->grid_w);
  const uint32_t rows = (uint32_t)((int64_t)d.BH * d.L);
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t total = (uint64_t)rows << ch_shift;
  const int grid = (int)std::max<uint64_t>(1, std::min<uint64_t>((total + 255) / 256, (uint64_t)sms * 8));
  permute_kernel<<<grid, 256, 0, s>>>((const uint4*)src, (uint4*)dst, rows, ch_shift, g, to_cube);
  return check_launch("permute_kernel");
}

}  // namespace vsa2
