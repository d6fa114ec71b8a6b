// Tensor-core forward entry; until the tcgen05 kernel lands the CUDA-core kernel serves it.
#include "common.cuh"
#include "internal.h"
namespace vsa2 {
vsa2_status attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v, int topk, const int32_t* kv_off,
                        const int32_t* kv_idx, void* o, float* lse, char* ws, cudaStream_t s) {
  return attn_fwd_simt(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, s);
}
}  // namespace vsa2
