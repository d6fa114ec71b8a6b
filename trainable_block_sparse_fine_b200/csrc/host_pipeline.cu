// End-to-end forward from host buffers: router -> TopK -> block-sparse attention per group of
// heads, with the PCIe copies of neighbouring groups overlapped with the kernels.
//
// Every (b, h) is an independent problem: the router's softmax runs over the keys of its own
// (b, h) (Eq. 6), the TopK budget is per sequence (Eq. 8-9) and the attention of Eq. 12 reads
// only its own head. So a contiguous range of flat (b, h) indices is itself a valid problem
// (batch 1, heads = range length), and its inputs and outputs are contiguous in the
// [batch, heads, L, D] layout. The call runs the groups as three concurrent chains:
//   copy-in stream : H2D of group g's Q, K, V into staging slot g % kSlots
//   caller stream  : router, TopK and forward of group g on that slot
//   copy-out stream: D2H of group g's O (and LSE) from that slot
// Slots are reused only after their previous group's kernels (inputs) and D2H (outputs) ended.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int kSlots = 3;
constexpr int kMaxDevices = 64;
constexpr int64_t kAutoChunkTokens = 65536;  // automatic group size: at least this many tokens

struct Pipe {
  bool ready = false;
  unsigned long long ctx_id = 0;  // context the streams and events were created in
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t fork = nullptr, join_in = nullptr, join_out = nullptr;
  cudaEvent_t in_ready[kSlots] = {}, comp_done[kSlots] = {}, out_done[kSlots] = {};
};

std::mutex g_pipe_mu;
Pipe g_pipes[kMaxDevices];

// Streams and events of the current device, created on first use and kept for the process;
// created again if the device's context has been replaced since (the old handles died with it).
vsa2_status get_pipe(Pipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail("cudaGetDevice");
  if (cudaSetDevice(dev) != cudaSuccess) return cuda_fail("cudaSetDevice");
  Pipe& p = g_pipes[dev];  // the caller holds g_pipe_mu
  unsigned long long id = 0;
  if (current_context_id(&id) && p.ready && p.ctx_id != id) p = Pipe{};
  if (!p.ready) {
    const unsigned ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.fork, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.join_in, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.join_out, ef) == cudaSuccess;
    for (int s = 0; ok && s < kSlots; ++s)
      ok = cudaEventCreateWithFlags(&p.in_ready[s], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.comp_done[s], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.out_done[s], ef) == cudaSuccess;
    if (!ok) return cuda_fail("creating the copy streams and events of vsa2_forward_host");
    p.ready = true;
    p.ctx_id = id;
  }
  *out = &p;
  return VSA2_OK;
}

struct HostLayout {
  int per;                 // heads (flat b*H + h indices) per group
  int groups;
  size_t kernel_ws;        // workspace of one group's kernels, at offset 0
  size_t scores, kv_off, kv_idx;
  size_t slot0, slot_bytes;  // slot s at slot0 + s*slot_bytes: Q, K, V, O, LSE of one group
  size_t q, k, v, o, lse;    // offsets inside a slot
  size_t total;
};

bool host_layout(const Dims& d, const vsa2_problem* p, int topk, int heads_per_group, HostLayout* h) {
  int per = heads_per_group;
  if (per <= 0) per = (int)std::min<int64_t>(d.BH, std::max<int64_t>(1, (kAutoChunkTokens + d.L - 1) / d.L));
  per = std::min(per, d.BH);
  vsa2_problem sub = *p;
  sub.batch = 1;
  sub.heads = per;
  Dims ds;
  if (make_dims(&sub, &ds) != VSA2_OK) return false;
  h->per = per;
  h->groups = (d.BH + per - 1) / per;
  size_t off = ws_layout(ds).total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  h->kernel_ws = 0;
  h->scores = take((size_t)per * d.N * d.N * 4);
  h->kv_off = take((size_t)per * (d.N + 1) * 4);
  h->kv_idx = take((size_t)per * d.N * topk * 4);
  const size_t x = align256((size_t)per * d.L * d.D * d.esize);
  h->q = 0;
  h->k = x;
  h->v = 2 * x;
  h->o = 3 * x;
  h->lse = 4 * x;
  h->slot_bytes = 4 * x + align256((size_t)per * d.L * 4);
  h->slot0 = off;
  h->total = off + kSlots * h->slot_bytes;
  return true;
}

}  // namespace
}  // namespace vsa2

using namespace vsa2;

extern "C" {

size_t vsa2_forward_host_workspace_size(const vsa2_problem* p, int32_t topk, int32_t heads_per_group) {
  Dims d;
  HostLayout h;
  if (make_dims(p, &d) != VSA2_OK || topk < 1 || topk > d.N || heads_per_group < 0 || d.Bt != kTile) return 0;
  if (!host_layout(d, p, topk, heads_per_group, &h)) return 0;
  return h.total;
}

vsa2_status vsa2_forward_host(const vsa2_problem* p, const void* q, const void* k, const void* v, int32_t topk,
                              int32_t heads_per_group, void* o, float* lse, void* ws, size_t ws_bytes,
                              void* stream) {
  Dims d;
  vsa2_status st = make_dims(p, &d);
  if (st != VSA2_OK) return st;
  if (!q || !k || !v || !o) return VSA2_ERR_INVALID_ARG;
  if (topk < 1 || topk > d.N) return VSA2_ERR_UNSUPPORTED;
  if (heads_per_group < 0) return VSA2_ERR_INVALID_ARG;
  if (d.Bt != kTile) return VSA2_ERR_UNSUPPORTED;  // 64-token tiles
  HostLayout h;
  if (!host_layout(d, p, topk, heads_per_group, &h)) return VSA2_ERR_UNSUPPORTED;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < h.total) return VSA2_ERR_INVALID_ARG;

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  Pipe* pp = nullptr;
  if ((st = get_pipe(&pp)) != VSA2_OK) return st;
  Pipe& P = *pp;
  const cudaStream_t cs = (cudaStream_t)stream;
  char* base = (char*)ws;
  const size_t head_x = (size_t)d.L * d.D * d.esize;  // bytes of one head of Q/K/V/O
  const size_t head_l = (size_t)d.L * 4;              // bytes of one head of LSE

  // the copy streams start after everything already queued on the caller's stream
  if (cudaEventRecord(P.fork, cs) != cudaSuccess || cudaStreamWaitEvent(P.in, P.fork, 0) != cudaSuccess ||
      cudaStreamWaitEvent(P.out, P.fork, 0) != cudaSuccess)
    return cuda_fail("vsa2_forward_host: fork of the copy streams");

  for (int g = 0; g < h.groups && st == VSA2_OK; ++g) {
    const int s = g % kSlots;
    const int bh0 = g * h.per;
    const int n = std::min(h.per, d.BH - bh0);
    vsa2_problem sub = *p;
    sub.batch = 1;
    sub.heads = n;
    Dims ds;
    if ((st = make_dims(&sub, &ds)) != VSA2_OK) break;
    char* slot = base + h.slot0 + (size_t)s * h.slot_bytes;
    const size_t off_x = (size_t)bh0 * head_x, bytes_x = (size_t)n * head_x;

    // inputs: the slot's previous group must have finished reading it
    bool ok = g < kSlots || cudaStreamWaitEvent(P.in, P.comp_done[s], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(slot + h.q, (const char*)q + off_x, bytes_x, cudaMemcpyHostToDevice, P.in) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(slot + h.k, (const char*)k + off_x, bytes_x, cudaMemcpyHostToDevice, P.in) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(slot + h.v, (const char*)v + off_x, bytes_x, cudaMemcpyHostToDevice, P.in) == cudaSuccess;
    ok = ok && cudaEventRecord(P.in_ready[s], P.in) == cudaSuccess;
    // kernels: inputs in place, and the slot's previous outputs copied out
    ok = ok && cudaStreamWaitEvent(cs, P.in_ready[s], 0) == cudaSuccess;
    ok = ok && (g < kSlots || cudaStreamWaitEvent(cs, P.out_done[s], 0) == cudaSuccess);
    if (!ok) {
      st = cuda_fail("vsa2_forward_host: input copies");
      break;
    }
    float* scores = (float*)(base + h.scores);
    int32_t* kv_off = (int32_t*)(base + h.kv_off);
    int32_t* kv_idx = (int32_t*)(base + h.kv_idx);
    if ((st = launch_router(ds, slot + h.q, slot + h.k, scores, base, cs)) != VSA2_OK) break;
    if ((st = launch_topk(ds, scores, topk, kv_off, kv_idx, nullptr, nullptr, base, cs)) != VSA2_OK) break;
    if ((st = launch_attn_fwd(ds, slot + h.q, slot + h.k, slot + h.v, topk, kv_off, kv_idx, slot + h.o,
                              (float*)(slot + h.lse), base, cs)) != VSA2_OK)
      break;
    // outputs
    ok = cudaEventRecord(P.comp_done[s], cs) == cudaSuccess && cudaStreamWaitEvent(P.out, P.comp_done[s], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync((char*)o + off_x, slot + h.o, bytes_x, cudaMemcpyDeviceToHost, P.out) == cudaSuccess;
    if (lse)
      ok = ok && cudaMemcpyAsync((char*)lse + (size_t)bh0 * head_l, slot + h.lse, (size_t)n * head_l,
                                 cudaMemcpyDeviceToHost, P.out) == cudaSuccess;
    ok = ok && cudaEventRecord(P.out_done[s], P.out) == cudaSuccess;
    if (!ok) st = cuda_fail("vsa2_forward_host: output copies");
  }

  // join, also after an error: the caller's stream then covers every copy this call queued
  const bool joined = cudaEventRecord(P.join_in, P.in) == cudaSuccess &&
                      cudaEventRecord(P.join_out, P.out) == cudaSuccess &&
                      cudaStreamWaitEvent(cs, P.join_in, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(cs, P.join_out, 0) == cudaSuccess;
  if (st == VSA2_OK && !joined) st = cuda_fail("vsa2_forward_host: join of the copy streams");
  return st;
}

}  // extern "C"
