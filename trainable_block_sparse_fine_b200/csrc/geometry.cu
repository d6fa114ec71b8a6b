// Token grids that the tile does not divide ("Improving Video Sparse Attention with
// Fine-grained Router and Sparse Rebasing", §2.2 "Kernel Implementation": every dimension is
// padded to a multiple of the tile and the padding is masked). The padded grid is laid out in
// cube-major order like any other; this kernel marks, for every tile, which of its 64 tokens
// belong to the real grid. The router, the forward and the coarse branch read these masks.
#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

struct GridGeom {
  int gt, gh, gw;     // real grid
  int tt, th, tw;     // tile
  int rt, rh, rw;     // sub-cube
  int nth, ntw;       // tiles along h and w of the padded grid
};

// One thread per tile: bit u of mask[i] is set when cube-major token u of tile i (sub-cube
// u / R in raster order over the tile's sub-cubes, token u % R in raster order inside it) lies
// inside the real grid.
__global__ void __launch_bounds__(256) tile_mask_kernel(GridGeom g, int N, uint64_t* __restrict__ mask) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int per_t = g.nth * g.ntw;
  const int it = i / per_t, ih = (i % per_t) / g.ntw, iw = i % g.ntw;
  const int sh_n = g.th / g.rh, sw_n = g.tw / g.rw, R = g.rt * g.rh * g.rw;
  uint64_t m = 0;
  for (int u = 0; u < 64; ++u) {
    const int sub = u / R, r = u % R;
    const int st = sub / (sh_n * sw_n), s2 = sub % (sh_n * sw_n), sh = s2 / sw_n, sw = s2 % sw_n;
    const int dt = r / (g.rh * g.rw), r2 = r % (g.rh * g.rw), dh = r2 / g.rw, dw = r2 % g.rw;
    const int t = it * g.tt + st * g.rt + dt, h = ih * g.th + sh * g.rh + dh, w = iw * g.tw + sw * g.rw + dw;
    if (t < g.gt && h < g.gh && w < g.gw) m |= 1ull << u;
  }
  mask[i] = m;
}

}  // namespace

vsa2_status launch_tile_masks(const Dims& d, uint64_t* mask, cudaStream_t s) {
  GridGeom g;
  g.gt = d.gt, g.gh = d.gh, g.gw = d.gw;
  g.tt = d.tt, g.th = d.th, g.tw = d.tw;
  g.rt = d.rt, g.rh = d.rh, g.rw = d.rw;
  g.nth = (d.gh + d.th - 1) / d.th;
  g.ntw = (d.gw + d.tw - 1) / d.tw;
  tile_mask_kernel<<<(d.N + 255) / 256, 256, 0, s>>>(g, d.N, mask);
  return check_launch("tile_mask_kernel");
}

}  // namespace vsa2
