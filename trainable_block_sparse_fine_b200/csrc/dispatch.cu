// Kernel selection for the attention entry points, and the bounded-wait self-test kernel.
#include "common.cuh"
#include "internal.h"

namespace vsa2 {

namespace {
// One thread waits on an mbarrier that nothing completes; the bounded wait records
// VSA2_ERR_TIMEOUT in the error word and the kernel returns.
__global__ void wait_timeout_probe_kernel(int* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x != 0) return;
  abort_sh = 0;
  mbar_init(&bar, 1);
  fence_mbar_init();
  DevCtx ctx{err, timeout_ns, 0};
  mbar_wait(&bar, 0, &abort_sh, ctx);
}
}  // namespace

vsa2_status launch_wait_timeout_probe(int* err, uint64_t timeout_ns, cudaStream_t s) {
  wait_timeout_probe_kernel<<<1, 32, 0, s>>>(err, timeout_ns);
  return check_launch(__func__);
}

vsa2_status launch_attn_fwd(const Dims& d, const void* q, const void* k, const void* v, int topk,
                            const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                            cudaStream_t s) {
  if (d.dtype == VSA2_BF16 && d.D == 128) return attn_fwd_tc(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, s);
  uint64_t* tmask = nullptr;
  if (d.padded) {
    tmask = reinterpret_cast<uint64_t*>(ws + ws_layout(d).tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
  }
  return attn_fwd_simt(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, d.L, tmask, s);
}

vsa2_status launch_attn_bwd(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dout, int topk, const int32_t* kv_off,
                            const int32_t* kv_idx, const int32_t* q_off, const int32_t* q_idx, float* dq, float* dk,
                            float* dv, char* ws, cudaStream_t s) {
  uint64_t* tmask = nullptr;
  if (d.padded) {  // padding keys are masked and padding query rows (lse = -inf) add nothing
    tmask = reinterpret_cast<uint64_t*>(ws + ws_layout(d).tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
  }
  if (d.dtype == VSA2_BF16 && d.D == 128)
    return attn_bwd_tc(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, topk, ws, tmask, s);
  return attn_bwd_simt(d, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, topk, ws, tmask, s);
}

}  // namespace vsa2
