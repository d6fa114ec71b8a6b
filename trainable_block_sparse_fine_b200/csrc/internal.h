// Host-side internals of libvsa2: validated problem sizes, workspace layout, launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "vsa2.h"

namespace vsa2 {

// The attention kernels work on 64-token tiles. The router and the TopK work on the problem's
// tiles: 64 tokens with 16-token sub-cubes (G = 4), or 128 tokens with 8-token sub-cubes
// (G = 16); a 128-token tile is two consecutive 64-token tiles of the cube-major order, so its
// selection is expanded to 64-token tiles before the attention kernels run.
constexpr int kTile = 64;  // tokens per attention tile (4 x 4 x 4 cube)
constexpr int kPool = 16;  // tokens per router sub-cube of a 64-token tile (2 x 2 x 4)
constexpr int kG = kTile / kPool;

struct Dims {
  int B, H, D, BH;
  int64_t L;   // tokens per (b, h), of the padded grid when the tile does not divide the grid
  int N;       // tiles per (b, h)
  int Lr;      // pooled rows per (b, h)
  int dtype;   // vsa2_dtype
  int esize;   // bytes per element of Q/K/V/O/dO
  uint32_t flags;
  uint64_t timeout_ns;
  int gt, gh, gw;  // real token grid
  int tt, th, tw;  // tile
  int rt, rh, rw;  // router sub-cube
  bool padded;     // the tile does not divide the grid: every extent is rounded up to whole tiles
  int Bt, R, G;    // tokens per tile (64 or 128), per sub-cube (16 or 8), sub-cubes per tile
};

// The same problem seen in 64-token tiles (what the attention kernels take): d itself for
// 64-token tiles; for 128-token tiles N doubles.
inline Dims dims64(const Dims& d) {
  Dims e = d;
  e.N = (int)(d.L / kTile);
  e.Bt = kTile;
  e.R = kPool;
  e.G = kG;
  e.Lr = (int)(d.L / kPool);
  return e;
}

// VSA2_FLAG_COARSE_POOL_IN_ROUTER in effect: the router's pooling pass writes the coarse branch's
// Qc, Kc and the coarse branch pools only V (bf16, D = 128, 64-token tiles of 16-token sub-cubes).
inline bool coarse_pool_in_router(const Dims& d) {
  return (d.flags & VSA2_FLAG_COARSE_POOL_IN_ROUTER) && d.dtype == VSA2_BF16 && d.D == 128 && d.Bt == kTile &&
         d.R == kPool;
}

// Geometry of a grid the tile does not divide: which cube-major tokens of a tile are real.
struct GridGeom {
  int gt, gh, gw;  // real grid
  int tt, th, tw;  // tile
  int rt, rh, rw;  // sub-cube
  int nth, ntw;    // tiles along h and w of the padded grid
};
inline GridGeom grid_geom(const Dims& d) {
  GridGeom g;
  g.gt = d.gt, g.gh = d.gh, g.gw = d.gw;
  g.tt = d.tt, g.th = d.th, g.tw = d.tw;
  g.rt = d.rt, g.rh = d.rh, g.rw = d.rw;
  g.nth = (d.gh + d.th - 1) / d.th;
  g.ntw = (d.gw + d.tw - 1) / d.tw;
  return g;
}
// Cube-major token u of tile i (sub-cube u / R in raster order over the tile's sub-cubes, token
// u % R in raster order inside it) lies inside the real grid.
__host__ __device__ inline bool token_real(const GridGeom& g, int i, int u) {
  const int per_t = g.nth * g.ntw;
  const int it = i / per_t, ih = (i % per_t) / g.ntw, iw = i % g.ntw;
  const int sh_n = g.th / g.rh, sw_n = g.tw / g.rw, R = g.rt * g.rh * g.rw;
  const int sub = u / R, r = u % R;
  const int st = sub / (sh_n * sw_n), s2 = sub % (sh_n * sw_n), sh = s2 / sw_n, sw = s2 % sw_n;
  const int dt = r / (g.rh * g.rw), r2 = r % (g.rh * g.rw), dh = r2 / g.rw, dw = r2 % g.rw;
  const int t = it * g.tt + st * g.rt + dt, h = ih * g.th + sh * g.rh + dh, w = iw * g.tw + sw * g.rw + dw;
  return t < g.gt && h < g.gh && w < g.gw;
}

// Real-token mask of every tile of a padded grid (bit u = cube-major token u of the tile is a
// token of the real grid); the same for every (b, h). Enqueued on `s`, written to `mask` [N].
vsa2_status launch_tile_masks(const Dims& d, uint64_t* mask, cudaStream_t s);

// Validate a problem description; fills `d` on success.
vsa2_status make_dims(const vsa2_problem* p, Dims* d);

// Workspace regions (byte offsets from the workspace base, all 256-byte aligned).
constexpr int kCandCap = 8192;  // TopK candidate list per (b, h)
struct WsLayout {
  size_t qr, kr;         // pooled Q, K: [BH, Lr, D] in the input dtype
  size_t lse_r;          // router per-pooled-row LSE (log2 domain), [BH, Lr] fp32
  size_t hist;           // TopK radix histograms [BH, 3, 2048] u32
  size_t state;          // TopK per-(b,h) state [BH, 8] u32
  size_t row_gt, row_eq, row_take;  // [BH, N] i32
  size_t col_cnt;        // [BH, N] i32
  size_t col_bits;       // [BH, N, words] u32
  int words;             // ceil(N / 32)
  size_t delta;          // backward rowsum(dO * O), [BH, L] fp32 (the tcgen05 backward keeps
                         // -Delta here, in token order)
  size_t nlse2;          // tcgen05 backward: -lse * log2(e), [BH, L] fp32, token order
  int Nc_tiles;          // coarse branch: ceil(N / 64) tiles of pooled rows per (b, h)
  size_t qc, kc, vc, oc; // coarse branch: pooled Q, K, V and output, [BH, 64 * Nc_tiles, D] dtype,
                         // rows >= N zero (Q, K, V) or unused (output)
  size_t lse_c;          // coarse branch LSE, [BH, 64 * Nc_tiles] fp32
  size_t c_off, c_idx;   // coarse branch: CSR listing every tile, [BH, Nc_tiles + 1], [BH, Nc_tiles^2] i32
  size_t doc;            // coarse backward: padded gradient of O_c_hat, [BH, 64 * Nc_tiles, D] dtype
  size_t dqc, dkc, dvc;  // coarse backward: gradients of the pooled rows, [BH, 64 * Nc_tiles, D] fp32
  size_t tmask;          // padded grids: real-token mask per tile, [N] u64
  size_t cand, cand_cnt; // TopK: entries sharing the 22-bit threshold prefix, [BH, kCandCap] u32
                         // (row << 10 | low 10 bits), and their count per (b, h)
  size_t total;
};
WsLayout ws_layout(const Dims& d);

// 128-token tiles: the selection expanded to 64-token tiles (CSR, and CSC for the backward),
// after every region the kernels of d and of dims64(d) use. topk is the problem's budget.
struct ExpLayout {
  size_t off, idx, qoff, qidx, total;
};
ExpLayout exp_layout(const Dims& d, int topk);
// Workspace bytes a call with budget topk (0: calls without a selection) needs.
size_t ws_required(const Dims& d, int topk);
// Expand a tile-granularity list (CSR or CSC) of 128-token tiles into 64-token tiles: 64-tile u
// of head bh gets 2J, 2J+1 for every J in list u / 2. Enqueued on s.
vsa2_status launch_expand_lists(const Dims& d, int topk, const int32_t* off, const int32_t* idx, int32_t* off64,
                                int32_t* idx64, cudaStream_t s);

// Tensor map for a row-major [outer, rows, cols] bf16 tensor, box (box_cols x box_rows x 1),
// 128-byte swizzle. Returns false if the driver entry point is unavailable or encoding failed.
bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                       uint32_t box_cols, uint32_t box_rows);

// Launchers (enqueue only). Each returns VSA2_OK or VSA2_ERR_CUDA.
vsa2_status launch_router(const Dims& d, const void* q, const void* k, float* scores, char* ws, cudaStream_t s);
vsa2_status launch_topk(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                        int32_t* q_off, int32_t* q_idx, char* ws, cudaStream_t s);
vsa2_status launch_topk_per_row(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                                int32_t* q_off, int32_t* q_idx, char* ws, cudaStream_t s);
vsa2_status launch_attn_fwd(const Dims& d, const void* q, const void* k, const void* v, int topk,
                            const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                            cudaStream_t s);
vsa2_status launch_attn_bwd(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dout, int topk, const int32_t* kv_off,
                            const int32_t* kv_idx, const int32_t* q_off, const int32_t* q_idx, float* dq, float* dk,
                            float* dv, char* ws, cudaStream_t s);
// CUDA-core paths (fp32 inputs, head_dim 64, and the backward pass). The forward masks keys at
// or beyond kv_valid tokens of each head (d.L for the fine branch: no mask) and, with tmask (a
// padded grid's real-token masks), the padding tokens of every tile.
vsa2_status attn_fwd_simt(const Dims& d, const void* q, const void* k, const void* v, int topk,
                          const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                          int64_t kv_valid, const uint64_t* tmask, cudaStream_t s, const float* gate = nullptr,
                          const void* oc = nullptr, void* of = nullptr);
// backward on CUDA cores; tmask (a padded grid's real-token masks, or null): padding keys take
// no part and get dK = dV = 0, padding query rows (lse = -inf) add nothing
vsa2_status attn_bwd_simt(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, const int32_t* kv_off, const int32_t* kv_idx,
                          const int32_t* q_off, const int32_t* q_idx, float* dq, float* dk, float* dv, int topk,
                          char* ws, const uint64_t* tmask, cudaStream_t s);
// tensor-core forward (bf16, head_dim 128); the masked variant treats keys at or beyond
// kv_valid tokens of each head as padding (each listed tile must hold a valid key)
vsa2_status attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v, int topk,
                        const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                        cudaStream_t s);
// the fine forward with the gated merge of Eq. 13-14 in its epilogue (bf16, head_dim 128):
// o = tanh(gate_logits) * oc[tile] + O_f; O_f also written to o_f when it is not null
vsa2_status attn_fwd_tc_gated(const Dims& d, const void* q, const void* k, const void* v, int topk,
                              const int32_t* kv_off, const int32_t* kv_idx, const float* gate_logits, const void* oc,
                              void* o, float* lse, void* o_f, char* ws, cudaStream_t s);
vsa2_status attn_fwd_tc_masked(const Dims& d, const void* q, const void* k, const void* v, int topk,
                               const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                               int kv_valid, cudaStream_t s);
// tensor-core forward on 128-token tiles (d.Bt = 128, bf16, head_dim 128, grids the tile
// divides): M=128 query tiles against whole 128-token KV tiles of the selection as given
vsa2_status attn_fwd_b128_tc(const Dims& d, const void* q, const void* k, const void* v, int topk,
                             const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                             cudaStream_t s);
// dQ on 128-token tiles (d.Bt = 128, bf16, head_dim 128, grids the tile divides) from the
// 128-token CSR, with -Delta and -lse * log2(e) per token written to ndelta / nlse2 for the
// dK/dV kernel; and that dK/dV kernel alone, on a CSC of 64-token tiles (d in 64-token tiles)
vsa2_status attn_bwd_dq_b128_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, const int32_t* kv_off, const int32_t* kv_idx,
                                float* dq, float* ndelta, float* nlse2, int topk, char* ws, cudaStream_t s);
vsa2_status attn_bwd_dkdv_only_tc(const Dims& d, const void* q, const void* k, const void* v, const void* dout,
                                  const int32_t* q_off, const int32_t* q_idx, float* dk, float* dv, int topk, char* ws,
                                  cudaStream_t s);
// Coarse branch (Eq. 1-3) and gated merge (Eq. 4, 13-14)
vsa2_status launch_coarse_attn(const Dims& d, const void* q, const void* k, const void* v, void* oc, float* lse_c,
                               char* ws, cudaStream_t s);
vsa2_status launch_gated_merge(const Dims& d, const void* o_f, const float* gate_logits, const void* oc, void* o,
                               cudaStream_t s);
vsa2_status launch_gated_merge_bwd(const Dims& d, const void* dout, const float* gate_logits, const void* oc,
                                   float* d_logits, float* d_oc, cudaStream_t s);
vsa2_status launch_coarse_attn_bwd(const Dims& d, const void* q, const void* k, const void* v, const void* oc,
                                   const float* lse_c, const float* d_oc, float* dq, float* dk, float* dv, char* ws,
                                   cudaStream_t s);
// tensor-core backward (bf16, head_dim 128): dQ kernel (also writes Delta), then dK/dV kernel;
// tmask as for attn_bwd_simt
vsa2_status attn_bwd_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, const int32_t* kv_off, const int32_t* kv_idx, const int32_t* q_off,
                        const int32_t* q_idx, float* dq, float* dk, float* dv, int topk, char* ws,
                        const uint64_t* tmask, cudaStream_t s);
// Token permutation raster <-> cube-major (to_cube != 0: raster -> cube-major)
vsa2_status launch_permute(const Dims& d, const vsa2_problem* p, const void* src, void* dst, int to_cube,
                           cudaStream_t s);
vsa2_status launch_wait_timeout_probe(int* err, uint64_t timeout_ns, cudaStream_t s);
// allocation-free TopK (scratch in a fixed device array of the library)
size_t topk_noalloc_bytes(const Dims& d);
size_t topk_noalloc_capacity();
vsa2_status launch_topk_noalloc(const Dims& d, const float* scores, int topk, int32_t* kv_off, int32_t* kv_idx,
                                cudaStream_t s);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Unique id of the CUDA context current on this thread; false if it cannot be read. Call after
// a runtime call that binds the device's primary context (cudaGetDevice + cudaSetDevice).
bool current_context_id(unsigned long long* id);

// Records the message of a failed CUDA call (see vsa2_last_cuda_error) and returns VSA2_ERR_CUDA.
vsa2_status cuda_fail(const char* what);
// Records a failed tensor-map encoding (with the driver's result code) and returns VSA2_ERR_CUDA.
vsa2_status tmap_fail(const char* what);
// VSA2_OK if the last launch succeeded, else records the CUDA error and returns VSA2_ERR_CUDA.
vsa2_status check_launch(const char* what);

}  // namespace vsa2
