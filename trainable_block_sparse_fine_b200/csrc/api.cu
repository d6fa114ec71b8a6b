// C ABI of libvsa2: argument validation, workspace layout and dispatch to the kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
vsa2_status make_dims(const vsa2_problem* p, Dims* d) {
  if (!p || !d) return VSA2_ERR_INVALID_ARG;
  if (p->batch <= 0 || p->heads <= 0 || p->head_dim <= 0 || p->grid_t <= 0 || p->grid_h <= 0 || p->grid_w <= 0)
    return VSA2_ERR_INVALID_ARG;
  if (p->tile_t <= 0 || p->tile_h <= 0 || p->tile_w <= 0 || p->pool_t <= 0 || p->pool_h <= 0 || p->pool_w <= 0)
    return VSA2_ERR_INVALID_ARG;
  if (p->dtype != VSA2_BF16 && p->dtype != VSA2_FP32) return VSA2_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return VSA2_ERR_UNSUPPORTED;
  // 64-token tiles with 16-token sub-cubes (the pages' shapes), or 128-token tiles with 8-token
  // sub-cubes (the B = 128, R = 8 reading of the deep-read blog)
  const int Bt = p->tile_t * p->tile_h * p->tile_w, R = p->pool_t * p->pool_h * p->pool_w;
  if (!((Bt == 64 && R == 16) || (Bt == 128 && R == 8))) return VSA2_ERR_UNSUPPORTED;
  if (p->tile_t % p->pool_t || p->tile_h % p->pool_h || p->tile_w % p->pool_w) return VSA2_ERR_UNSUPPORTED;
  // a grid the tile does not divide is padded to whole tiles (§2.2 "Kernel Implementation")
  const bool padded = p->grid_t % p->tile_t || p->grid_h % p->tile_h || p->grid_w % p->tile_w;
  if (padded && Bt != 64) return VSA2_ERR_UNSUPPORTED;  // padding is built for 64-token tiles
  const int64_t pt = (p->grid_t + p->tile_t - 1) / p->tile_t * p->tile_t;
  const int64_t ph = (p->grid_h + p->tile_h - 1) / p->tile_h * p->tile_h;
  const int64_t pw = (p->grid_w + p->tile_w - 1) / p->tile_w * p->tile_w;
  if (pt > (1 << 20) || ph > (1 << 20) || pw > (1 << 20)) return VSA2_ERR_UNSUPPORTED;
  const int64_t L = pt * ph * pw;
  const int64_t N = L / Bt;
  const int64_t BH = p->batch * p->heads;
  // index arithmetic below uses 32-bit tile and row counts
  if (N > 32768 || BH > 65535 || BH * L > (int64_t(1) << 31)) return VSA2_ERR_UNSUPPORTED;
  d->B = (int)p->batch;
  d->H = (int)p->heads;
  d->D = (int)p->head_dim;
  d->BH = (int)BH;
  d->L = L;
  d->N = (int)N;
  d->Lr = (int)(L / R);
  d->dtype = p->dtype;
  d->esize = p->dtype == VSA2_BF16 ? 2 : 4;
  d->flags = p->flags;
  d->timeout_ns = (uint64_t)(p->wait_timeout_ms ? p->wait_timeout_ms : 2000u) * 1000000ull;
  d->gt = (int)p->grid_t, d->gh = (int)p->grid_h, d->gw = (int)p->grid_w;
  d->tt = p->tile_t, d->th = p->tile_h, d->tw = p->tile_w;
  d->rt = p->pool_t, d->rh = p->pool_h, d->rw = p->pool_w;
  d->padded = padded;
  d->Bt = Bt;
  d->R = R;
  d->G = Bt / R;
  return VSA2_OK;
}

WsLayout ws_layout(const Dims& d) {
  WsLayout w{};
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += align256(bytes);
    return at;
  };
  w.qr = take((size_t)d.BH * d.Lr * d.D * d.esize);
  w.kr = take((size_t)d.BH * d.Lr * d.D * d.esize);
  w.lse_r = take((size_t)d.BH * d.Lr * 4);
  w.hist = take((size_t)d.BH * 3 * 2048 * 4);
  w.state = take((size_t)d.BH * 8 * 4);
  w.row_gt = take((size_t)d.BH * d.N * 4);
  w.row_eq = take((size_t)d.BH * d.N * 4);
  w.row_take = take((size_t)d.BH * d.N * 4);
  w.col_cnt = take((size_t)d.BH * d.N * 4);
  w.words = (d.N + 31) / 32;
  w.col_bits = take((size_t)d.BH * d.N * w.words * 4);
  w.delta = take((size_t)d.BH * d.L * 4);
  w.nlse2 = take((size_t)d.BH * d.L * 4);
  w.Nc_tiles = (d.N + kTile - 1) / kTile;
  const size_t lc = (size_t)kTile * w.Nc_tiles;
  w.qc = take((size_t)d.BH * lc * d.D * d.esize);
  w.kc = take((size_t)d.BH * lc * d.D * d.esize);
  w.vc = take((size_t)d.BH * lc * d.D * d.esize);
  w.oc = take((size_t)d.BH * lc * d.D * d.esize);
  w.lse_c = take((size_t)d.BH * lc * 4);
  w.c_off = take((size_t)d.BH * (w.Nc_tiles + 1) * 4);
  w.c_idx = take((size_t)d.BH * w.Nc_tiles * w.Nc_tiles * 4);
  w.doc = take((size_t)d.BH * lc * d.D * d.esize);
  w.dqc = take((size_t)d.BH * lc * d.D * 4);
  w.dkc = take((size_t)d.BH * lc * d.D * 4);
  w.dvc = take((size_t)d.BH * lc * d.D * 4);
  w.tmask = take((size_t)d.N * 8);
  w.cand = take((size_t)d.BH * kCandCap * 4);
  w.cand_cnt = take((size_t)d.BH * 4);
  w.total = off;
  return w;
}

ExpLayout exp_layout(const Dims& d, int topk) {
  ExpLayout e{};
  size_t base = ws_layout(d).total;
  if (d.Bt != kTile) base = std::max(base, ws_layout(dims64(d)).total);
  e.total = base;
  if (d.Bt == kTile || topk <= 0) return e;
  auto take = [&](size_t bytes) {
    const size_t at = e.total;
    e.total += align256(bytes);
    return at;
  };
  const size_t n64 = (size_t)2 * d.N;
  e.off = take((size_t)d.BH * (n64 + 1) * 4);
  e.idx = take((size_t)d.BH * 4 * (size_t)d.N * topk * 4);
  e.qoff = take((size_t)d.BH * (n64 + 1) * 4);
  e.qidx = take((size_t)d.BH * 4 * (size_t)d.N * topk * 4);
  return e;
}

size_t ws_required(const Dims& d, int topk) { return exp_layout(d, topk).total; }

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Unique id of the CUDA context current on this thread (cuCtxGetId), so that state a library
// call keeps per device (a device address, streams, events) can tell a context that replaced
// an earlier one on the same device, for example after cudaDeviceReset.
bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess && cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) ==
                                                 cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrent>(a);
      get_id = reinterpret_cast<GetId>(b);
    }
  });
  CUcontext c = nullptr;
  if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

static thread_local int g_encode_result = 0;

// The encoder is a driver call: make the current device's primary context current on this
// thread first (a thread that has issued no runtime call yet, such as an autograd worker whose
// tensors all came from a caching allocator, may have none).
static bool bind_context() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess;
}

bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                       uint32_t box_cols, uint32_t box_rows) {
  auto enc = get_encode();
  g_encode_result = -1;
  if (!enc || !bind_context()) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  g_encode_result = (int)r;
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                       uint32_t box_rows) {
  auto enc = get_encode();
  g_encode_result = -1;
  if (!enc || !bind_context()) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  g_encode_result = (int)r;
  return r == CUDA_SUCCESS;
}

static std::atomic<const char*> g_last_cuda_error{"no CUDA error recorded"};
static thread_local char g_msg[256];

vsa2_status cuda_fail(const char* what) {
  g_last_cuda_error.store(what);
  return VSA2_ERR_CUDA;
}

vsa2_status tmap_fail(const char* what) {
  snprintf(g_msg, sizeof(g_msg), "%s (cuTensorMapEncodeTiled result %d, -1 = no encoder or no context)", what,
           g_encode_result);
  g_last_cuda_error.store(g_msg);
  return VSA2_ERR_CUDA;
}

vsa2_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return VSA2_OK;
  snprintf(g_msg, sizeof(g_msg), "%s: %s", what, cudaGetErrorString(e));
  g_last_cuda_error.store(g_msg);
  return VSA2_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static vsa2_status check_ws(const Dims& d, void* ws, size_t ws_bytes, int topk = 0) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return VSA2_ERR_INVALID_ARG;
  if (ws_bytes < ws_required(d, topk)) return VSA2_ERR_INVALID_ARG;
  return VSA2_OK;
}

}  // namespace vsa2

using namespace vsa2;

extern "C" {

size_t vsa2_workspace_size(const vsa2_problem* p, int32_t topk) {
  Dims d;
  if (make_dims(p, &d) != VSA2_OK) return 0;
  return ws_required(d, topk);
}

vsa2_status vsa2_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeader || (reinterpret_cast<uintptr_t>(ws) & 255u)) return VSA2_ERR_INVALID_ARG;
  if (cudaMemsetAsync(ws, 0, kWsHeader, (cudaStream_t)stream) != cudaSuccess) return VSA2_ERR_CUDA;
  return VSA2_OK;
}

vsa2_status vsa2_router_scores(const vsa2_problem* p, const void* q, const void* k, float* scores, void* ws,
                               size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!q || !k || !scores) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes)) != VSA2_OK) return st;
  return launch_router(d, q, k, scores, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_topk_select(const vsa2_problem* p, const float* scores, int32_t topk, int32_t* kv_off,
                             int32_t* kv_idx, int32_t* q_off, int32_t* q_idx, void* ws, size_t ws_bytes,
                             void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!scores || !kv_off || !kv_idx) return VSA2_ERR_INVALID_ARG;
  if ((q_off == nullptr) != (q_idx == nullptr)) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (!aligned16(scores)) return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes)) != VSA2_OK) return st;
  return launch_topk(d, scores, topk, kv_off, kv_idx, q_off, q_idx, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_topk_select_per_row(const vsa2_problem* p, const float* scores, int32_t topk, int32_t* kv_off,
                                     int32_t* kv_idx, int32_t* q_off, int32_t* q_idx, void* ws, size_t ws_bytes,
                                     void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!scores || !kv_off || !kv_idx) return VSA2_ERR_INVALID_ARG;
  if ((q_off == nullptr) != (q_idx == nullptr)) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if ((st = check_ws(d, ws, ws_bytes)) != VSA2_OK) return st;
  return launch_topk_per_row(d, scores, topk, kv_off, kv_idx, q_off, q_idx, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_sparse_attn_fwd(const vsa2_problem* p, const void* q, const void* k, const void* v, int32_t topk,
                                 const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, void* ws,
                                 size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!q || !k || !v || !kv_off || !kv_idx || !o || !lse) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes, topk)) != VSA2_OK) return st;
  if (d.Bt != kTile && d.dtype == VSA2_BF16 && d.D == 128 && !d.padded)  // M=128 query tiles
    return attn_fwd_b128_tc(d, q, k, v, topk, kv_off, kv_idx, o, lse, (char*)ws, (cudaStream_t)stream);
  if (d.Bt != kTile) {  // 128-token tiles otherwise: expand the selection, run on 64-token tiles
    const ExpLayout e = exp_layout(d, topk);
    char* w = (char*)ws;
    int32_t* off64 = reinterpret_cast<int32_t*>(w + e.off);
    int32_t* idx64 = reinterpret_cast<int32_t*>(w + e.idx);
    if ((st = launch_expand_lists(d, topk, kv_off, kv_idx, off64, idx64, (cudaStream_t)stream)) != VSA2_OK) return st;
    return launch_attn_fwd(dims64(d), q, k, v, 2 * topk, off64, idx64, o, lse, w, (cudaStream_t)stream);
  }
  return launch_attn_fwd(d, q, k, v, topk, kv_off, kv_idx, o, lse, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_sparse_attn_fwd_gated(const vsa2_problem* p, const void* q, const void* k, const void* v,
                                       int32_t topk, const int32_t* kv_off, const int32_t* kv_idx,
                                       const float* gate_logits, const void* oc, void* o, float* lse, void* o_f,
                                       void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!q || !k || !v || !kv_off || !kv_idx || !gate_logits || !oc || !o || !lse) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(oc) ||
      !aligned16(gate_logits) || (o_f && !aligned16(o_f)))
    return VSA2_ERR_INVALID_ARG;
  if (o == o_f || o == q || o == k || o == v) return VSA2_ERR_INVALID_ARG;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // the merge repeats 64-token tiles
  if ((st = check_ws(d, ws, ws_bytes, topk)) != VSA2_OK) return st;
  const cudaStream_t s = (cudaStream_t)stream;
  if (d.dtype == VSA2_BF16 && d.D == 128)
    return attn_fwd_tc_gated(d, q, k, v, topk, kv_off, kv_idx, gate_logits, oc, o, lse, o_f, (char*)ws, s);
  // CUDA-core shapes (fp32, head_dim 64): the same merge in the CUDA-core forward's epilogue
  uint64_t* tmask = nullptr;
  if (d.padded) {
    tmask = reinterpret_cast<uint64_t*>((char*)ws + ws_layout(d).tmask);
    if ((st = launch_tile_masks(d, tmask, s)) != VSA2_OK) return st;
  }
  return attn_fwd_simt(d, q, k, v, topk, kv_off, kv_idx, o, lse, (char*)ws, d.L, tmask, s, gate_logits, oc, o_f);
}

vsa2_status vsa2_sparse_attn_bwd(const vsa2_problem* p, const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dout, int32_t topk, const int32_t* kv_off,
                                 const int32_t* kv_idx,
                                 const int32_t* q_off, const int32_t* q_idx, float* dq, float* dk, float* dv,
                                 void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!q || !k || !v || !o || !lse || !dout || !kv_off || !kv_idx || !q_off || !q_idx || !dq || !dk || !dv)
    return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(lse))
    return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes, topk)) != VSA2_OK) return st;
  if (d.Bt != kTile) {  // 128-token tiles: expand the CSR and the CSC, run on 64-token tiles
    const ExpLayout e = exp_layout(d, topk);
    char* w = (char*)ws;
    const cudaStream_t s = (cudaStream_t)stream;
    int32_t* off64 = reinterpret_cast<int32_t*>(w + e.off);
    int32_t* idx64 = reinterpret_cast<int32_t*>(w + e.idx);
    int32_t* qoff64 = reinterpret_cast<int32_t*>(w + e.qoff);
    int32_t* qidx64 = reinterpret_cast<int32_t*>(w + e.qidx);
    if (d.dtype == VSA2_BF16 && d.D == 128 && !d.padded) {
      // dQ on the 128-token CSR (M=128 query tiles); dK, dV on the expanded CSC
      if ((st = launch_expand_lists(d, topk, q_off, q_idx, qoff64, qidx64, s)) != VSA2_OK) return st;
      const Dims d64 = dims64(d);
      float* ndelta = reinterpret_cast<float*>(w + ws_layout(d64).delta);
      float* nlse2 = reinterpret_cast<float*>(w + ws_layout(d64).nlse2);
      if ((st = attn_bwd_dq_b128_tc(d, q, k, v, o, lse, dout, kv_off, kv_idx, dq, ndelta, nlse2, topk, w, s)) !=
          VSA2_OK)
        return st;
      return attn_bwd_dkdv_only_tc(d64, q, k, v, dout, qoff64, qidx64, dk, dv, 2 * topk, w, s);
    }
    if ((st = launch_expand_lists(d, topk, kv_off, kv_idx, off64, idx64, s)) != VSA2_OK) return st;
    if ((st = launch_expand_lists(d, topk, q_off, q_idx, qoff64, qidx64, s)) != VSA2_OK) return st;
    return launch_attn_bwd(dims64(d), q, k, v, o, lse, dout, 2 * topk, off64, idx64, qoff64, qidx64, dq, dk, dv, w, s);
  }
  return launch_attn_bwd(d, q, k, v, o, lse, dout, topk, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, (char*)ws,
                         (cudaStream_t)stream);
}

vsa2_status vsa2_coarse_attn(const vsa2_problem* p, const void* q, const void* k, const void* v, void* oc,
                             float* lse_c, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // the coarse branch and the merge take 64-token tiles
  if (!q || !k || !v || !oc) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(oc) || (lse_c && !aligned16(lse_c)))
    return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes)) != VSA2_OK) return st;
  return launch_coarse_attn(d, q, k, v, oc, lse_c, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_gated_merge(const vsa2_problem* p, const void* o_f, const float* gate_logits, const void* oc,
                             void* o, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // the coarse branch and the merge take 64-token tiles
  if (!o_f || !gate_logits || !oc || !o) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(o_f) || !aligned16(gate_logits) || !aligned16(oc) || !aligned16(o)) return VSA2_ERR_INVALID_ARG;
  return launch_gated_merge(d, o_f, gate_logits, oc, o, (cudaStream_t)stream);
}

vsa2_status vsa2_gated_merge_bwd(const vsa2_problem* p, const void* dout, const float* gate_logits, const void* oc,
                                 float* d_logits, float* d_oc, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // the coarse branch and the merge take 64-token tiles
  if (!dout || !gate_logits || !oc || !d_logits || !d_oc) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(gate_logits) || !aligned16(oc) || !aligned16(d_logits) || !aligned16(d_oc))
    return VSA2_ERR_INVALID_ARG;
  return launch_gated_merge_bwd(d, dout, gate_logits, oc, d_logits, d_oc, (cudaStream_t)stream);
}

vsa2_status vsa2_coarse_attn_bwd(const vsa2_problem* p, const void* q, const void* k, const void* v, const void* oc,
                                 const float* lse_c, const float* d_oc, float* dq, float* dk, float* dv, void* ws,
                                 size_t ws_bytes, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // the coarse branch and the merge take 64-token tiles
  if (!q || !k || !v || !oc || !lse_c || !d_oc || !dq || !dk || !dv) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(oc) || !aligned16(lse_c) || !aligned16(d_oc) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return VSA2_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws, ws_bytes)) != VSA2_OK) return st;
  return launch_coarse_attn_bwd(d, q, k, v, oc, lse_c, d_oc, dq, dk, dv, (char*)ws, (cudaStream_t)stream);
}

vsa2_status vsa2_permute_tokens(const vsa2_problem* p, const void* src, void* dst, int32_t to_cube_major,
                                void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!src || !dst || src == dst) return VSA2_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return VSA2_ERR_INVALID_ARG;
  return launch_permute(d, p, src, dst, to_cube_major != 0, (cudaStream_t)stream);
}

vsa2_status vsa2_topk_select_noalloc(const vsa2_problem* p, const float* scores, int32_t topk, int32_t* kv_off,
                                     int32_t* kv_idx, void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!scores || !kv_off || !kv_idx) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (!aligned16(scores)) return VSA2_ERR_INVALID_ARG;
  if (topk_noalloc_bytes(d) > topk_noalloc_capacity()) return VSA2_ERR_UNSUPPORTED;
  return launch_topk_noalloc(d, scores, topk, kv_off, kv_idx, (cudaStream_t)stream);
}

vsa2_status vsa2_get_device_error(void* ws, void* stream) {
  if (!ws) return VSA2_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return VSA2_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return VSA2_ERR_CUDA;
  if (code != 0) {
    int zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return VSA2_ERR_CUDA;
  }
  return (vsa2_status)code;
}

vsa2_status vsa2_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t timeout_ms, void* stream) {
  if (!ws || ws_bytes < kWsHeader || (reinterpret_cast<uintptr_t>(ws) & 255u)) return VSA2_ERR_INVALID_ARG;
  if (timeout_ms == 0 || timeout_ms > 10000) return VSA2_ERR_INVALID_ARG;
  return launch_wait_timeout_probe((int*)ws, (uint64_t)timeout_ms * 1000000ull, (cudaStream_t)stream);
}

const char* vsa2_status_string(vsa2_status s) {
  switch (s) {
    case VSA2_OK: return "VSA2_OK";
    case VSA2_ERR_INVALID_ARG: return "VSA2_ERR_INVALID_ARG";
    case VSA2_ERR_UNSUPPORTED: return "VSA2_ERR_UNSUPPORTED";
    case VSA2_ERR_CUDA: return "VSA2_ERR_CUDA";
    case VSA2_ERR_TIMEOUT: return "VSA2_ERR_TIMEOUT";
    case VSA2_ERR_BAD_INDEX: return "VSA2_ERR_BAD_INDEX";
  }
  return "VSA2_UNKNOWN_STATUS";
}

int32_t vsa2_version(void) { return 200; }  // 0.2.0: coarse branch, gated merge, permutation, host-buffer forward

const char* vsa2_last_cuda_error(void) { return g_last_cuda_error.load(); }

}  // extern "C"
