/*
 * vsa2.h - C ABI of the VSA2 hot path on NVIDIA B200 (sm_100a): fine-grained router,
 * per-sequence TopK, block-sparse attention forward / backward, and the coarse branch with
 * its gated merge.
 *
 * Method: "Improving Video Sparse Attention with Fine-grained Router and Sparse Rebasing"
 * (arXiv 2609.32882), §2.2 VSA2: Eq. 5-7 (router), Eq. 8-9 (per-sequence TopK), Eq. 12
 * (block-sparse fine branch), Eq. 1-4 (coarse branch), Eq. 13-14 (gated merge). §2.1
 * Background gives the attention definition with the -inf block mask; Fig. 5 gives the
 * two-pass (LSE, then softmax + on-chip pooling) router.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller, except the host buffers of
 *    vsa2_forward_host. The library never allocates or frees device memory and never
 *    synchronises, except vsa2_get_device_error.
 *    Every compute call only enqueues kernels on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and returns.
 *  - Token layout: Q, K, V, O, dO, dQ, dK, dV are [batch, heads, L, head_dim] row-major
 *    (head_dim innermost), L = grid_t*grid_h*grid_w in CUBE-MAJOR order (§2.2 "Permutation"):
 *    tiles of tile_t x tile_h x tile_w tokens in raster order over the tile grid; inside a
 *    tile, the router sub-cubes of pool_t x pool_h x pool_w tokens in raster order; inside a
 *    sub-cube, tokens in raster order. So tile i is rows [i*Bt, (i+1)*Bt) and its G = Bt/R
 *    sub-cubes are consecutive groups of R rows.
 *  - Sizes: Bt = tile_t*tile_h*tile_w is 64 with R = pool_t*pool_h*pool_w = 16 (G = 4), or
 *    128 with R = 8 (G = 16); the tile must be divisible by the pool; head_dim is 64 or 128;
 *    N = L/Bt tiles; 1 <= topk <= N. A grid the 64-token tile does not divide is padded to
 *    whole tiles (§2.2 "Kernel Implementation"): L then counts the padded grid, and padding
 *    tokens are masked everywhere (see vsa2_permute_tokens, which fills them). The coarse
 *    branch and the merge take 64-token tiles only. Other shapes return VSA2_ERR_UNSUPPORTED.
 *  - dtype covers Q, K, V, O and dO. Router scores, LSE and gradients are fp32; index lists
 *    are int32. Pointers must be 16-byte aligned.
 *  - Softmax scale is 1/sqrt(head_dim) everywhere (§2.1).
 *  - Errors: argument errors are reported synchronously by the return value and nothing is
 *    enqueued. A failed launch returns VSA2_ERR_CUDA. Faults found on the device (a bounded
 *    wait that expired, an index out of range when VSA2_FLAG_VALIDATE is set) are written to
 *    an error word at the start of the workspace and read back by vsa2_get_device_error.
 *  - Workspace: `ws` is caller-owned device memory of at least vsa2_workspace_size() bytes,
 *    256-byte aligned, zeroed once by vsa2_workspace_init before first use. One workspace
 *    must not be used by two calls that may run concurrently.
 */
#ifndef VSA2_H_
#define VSA2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VSA2_OK = 0,
  VSA2_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, small workspace */
  VSA2_ERR_UNSUPPORTED = 2, /* shape or dtype outside the supported set */
  VSA2_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  VSA2_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired (kernel returned early) */
  VSA2_ERR_BAD_INDEX = 5    /* validate mode: an offset or index was out of range */
} vsa2_status;

typedef enum { VSA2_BF16 = 0, VSA2_FP32 = 1 } vsa2_dtype;

enum {
  VSA2_FLAG_VALIDATE = 1u << 0, /* kernels bounds-check every offset and index they read */
  /* Eq. 1's pooled Q and K (the coarse branch's 64-token means) from the router's read of Q and
   * K: with this flag, vsa2_router_scores also writes them into the workspace, and
   * vsa2_coarse_attn reads them from there and pools only V. The caller must call
   * vsa2_router_scores with the flag on the same q, k and workspace before vsa2_coarse_attn
   * with the flag. Takes effect for bf16, D = 128, 64-token tiles with 16-token sub-cubes; the
   * two calls ignore it otherwise (vsa2_coarse_attn then pools Q and K itself). */
  VSA2_FLAG_COARSE_POOL_IN_ROUTER = 1u << 1
};

typedef struct vsa2_problem {
  int64_t batch, heads, head_dim;   /* Bsz, H, D */
  int64_t grid_t, grid_h, grid_w;   /* latent token grid T x H x W */
  int32_t tile_t, tile_h, tile_w;   /* block (tile) cube, 4 x 4 x 4 -> Bt = 64 */
  int32_t pool_t, pool_h, pool_w;   /* router pooling sub-cube, 2 x 2 x 4 -> R = 16 */
  int32_t dtype;                    /* vsa2_dtype */
  uint32_t flags;                   /* VSA2_FLAG_* */
  uint32_t wait_timeout_ms;         /* bound on any single device-side wait; 0 = 2000 ms */
  uint32_t reserved;
} vsa2_problem;

/* Bytes of workspace that every call below needs for this problem and budget. */
size_t vsa2_workspace_size(const vsa2_problem* p, int32_t topk);

/* Zero the workspace header (the device error word); enqueued on `stream`. Call once after
 * allocating a workspace. Returns VSA2_ERR_INVALID_ARG for a null or too-small workspace. */
vsa2_status vsa2_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Router scores, Eq. 5-7 with the two-pass fused kernel of Fig. 5.
 *   q, k    : [batch, heads, L, D] of dtype, cube-major (read only)
 *   scores  : [batch, heads, N, N] fp32 (written). scores[b,h,i,j] =
 *             (1/G) * sum_{a in tile i} sum_{c in tile j} softmax_c(qr_a . kr_c / sqrt(D)),
 *             qr, kr the means of Q, K over each R-token sub-cube (Eq. 5), the softmax over all
 *             L/R pooled keys of (b, h) (Eq. 6), pooled G x G (Eq. 7) and scaled by G so each
 *             row sums to 1 (the pages' MeanPool_{GxG} divided by G; TopK is unaffected).
 * The pooled Qr, Kr and per-row LSE live in the workspace; the L/R x L/R matrix is never
 * written to memory. With VSA2_FLAG_COARSE_POOL_IN_ROUTER the pooling pass also writes the
 * coarse branch's Qc, Kc (Eq. 1) into the workspace for a following vsa2_coarse_attn.
 */
vsa2_status vsa2_router_scores(const vsa2_problem* p, const void* q, const void* k, float* scores,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * Per-sequence TopK, Eq. 8-9: for each (b, h) keep the N*topk largest of the N*N scores;
 * equal scores are ranked by flat index i*N + j, lower first (the pages fix no tie order).
 *   scores  : [batch, heads, N, N] fp32, every entry >= 0 and finite (read only)
 *   kv_off  : [batch, heads, N+1] int32 (written) CSR row offsets, kv_off[.,.,0] = 0,
 *             kv_off[.,.,N] = N*topk
 *   kv_idx  : [batch, heads, N*topk] int32 (written) selected KV tiles of query tile i in
 *             kv_idx[kv_off[i] .. kv_off[i+1]), ascending
 *   q_off, q_idx : optional (both NULL or both non-NULL) CSC of the same selection: query
 *             tiles that selected KV tile j, ascending; needed by the backward pass
 * A query tile may receive zero KV tiles; the total per (b, h) is always N*topk.
 */
vsa2_status vsa2_topk_select(const vsa2_problem* p, const float* scores, int32_t topk,
                             int32_t* kv_off, int32_t* kv_idx, int32_t* q_off, int32_t* q_idx,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Per-query-tile TopK: the selection of VSA that §2.2 contrasts with Eq. 8-9 (§2.1
 * Background, TopK(Q_c K_c^T) row by row). Every query tile keeps its own topk largest scores,
 * so each row holds exactly topk KV tiles; equal scores within a row go to the lower KV tile.
 * Arguments, output format and errors as for vsa2_topk_select (kv_off[.,.,i] = i*topk). The
 * CSR feeds vsa2_sparse_attn_fwd / _bwd unchanged.
 */
vsa2_status vsa2_topk_select_per_row(const vsa2_problem* p, const float* scores, int32_t topk,
                                     int32_t* kv_off, int32_t* kv_idx, int32_t* q_off, int32_t* q_idx,
                                     void* ws, size_t ws_bytes, void* stream);

/*
 * Block-sparse attention forward, Eq. 12 with the §2.1 definition. For every query token t
 * of tile i: o_t = sum_u softmax_u(q_t . k_u / sqrt(D)) v_u over the tokens u of the KV tiles
 * listed for tile i; lse_t = ln sum_u exp(q_t . k_u / sqrt(D)). A tile with an empty list
 * gets o = 0 and lse = -inf.
 *   q, k, v        : [batch, heads, L, D] of dtype (read only)
 *   topk           : the budget the CSR was built with; kv_idx holds N*topk entries per (b, h)
 *   kv_off, kv_idx : CSR from vsa2_topk_select, or any CSR of distinct tiles per row with
 *                    offsets local to each (b, h) and kv_off[., ., N] <= N*topk (read only)
 *   o              : [batch, heads, L, D] of dtype (written)
 *   lse            : [batch, heads, L] fp32, natural log (written)
 */
vsa2_status vsa2_sparse_attn_fwd(const vsa2_problem* p, const void* q, const void* k, const void* v,
                                 int32_t topk, const int32_t* kv_off, const int32_t* kv_idx,
                                 void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * The fine branch of Eq. 12 with the gated merge of Eq. 13-14 in the same pass (§2.2 "Gated
 * Merge"): o = tanh(gate_logits) * Repeat_B(oc) + O_f, where O_f is what vsa2_sparse_attn_fwd
 * computes, without writing O_f and reading it back.
 *   q, k, v, topk, kv_off, kv_idx, lse : as for vsa2_sparse_attn_fwd (lse is the fine branch's)
 *   gate_logits : [batch, heads, L] fp32, the per-token logits X W_g of Eq. 13 (read only)
 *   oc          : [batch, heads, N, D] of dtype, the coarse output from vsa2_coarse_attn (read only)
 *   o           : [batch, heads, L, D] of dtype (written); must not alias q, k, v or o_f
 *   o_f         : NULL, or [batch, heads, L, D] of dtype receiving O_f (the backward forms
 *                 rowsum(dO * O_f) from it)
 * The merge is applied to O_f before its rounding to dtype. A tile with an empty list gets
 * o = tanh(g) * oc[tile], O_f = 0 and lse = -inf.
 */
vsa2_status vsa2_sparse_attn_fwd_gated(const vsa2_problem* p, const void* q, const void* k, const void* v,
                                       int32_t topk, const int32_t* kv_off, const int32_t* kv_idx,
                                       const float* gate_logits, const void* oc, void* o, float* lse, void* o_f,
                                       void* ws, size_t ws_bytes, void* stream);

/*
 * Block-sparse attention backward (gradients of Eq. 12; the router receives none, §2.1).
 *   q, k, v, o, dout : [batch, heads, L, D] of dtype (read only); o and lse from the forward
 *   lse              : [batch, heads, L] fp32 (read only)
 *   topk             : budget of the selection (index lists hold N*topk entries per (b, h))
 *   kv_off, kv_idx   : CSR of the selection; q_off, q_idx : its CSC (read only)
 *   dq, dk, dv       : [batch, heads, L, D] fp32 (written; fully overwritten)
 * With P = exp(S - lse), dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)),
 * dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D), each restricted to the selected tile pairs.
 * On a padded grid the padding keys take no part and the outputs of padding query rows are
 * dropped, so dout there reaches nothing: dQ, dK, dV of padding tokens are 0.
 */
vsa2_status vsa2_sparse_attn_bwd(const vsa2_problem* p, const void* q, const void* k, const void* v,
                                 const void* o, const float* lse, const void* dout, int32_t topk,
                                 const int32_t* kv_off, const int32_t* kv_idx,
                                 const int32_t* q_off, const int32_t* q_idx,
                                 float* dq, float* dk, float* dv,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * Coarse branch, Eq. 1-3 (§2.2 "Coarse Branch"): cube-level dense attention.
 *   Qc, Kc, Vc = the mean of Q, K, V over each tile of 64 tokens (Eq. 1), one row per tile;
 *   oc[b,h,i] = sum_j softmax_j(Qc_i . Kc_j / sqrt(D)) Vc_j over all N tiles (Eq. 2-3);
 *   lse_c[b,h,i] = ln sum_j exp(Qc_i . Kc_j / sqrt(D)).
 *   q, k, v : [batch, heads, L, D] of dtype (read only)
 *   oc      : [batch, heads, N, D] of dtype (written): O_c_hat, before Repeat_B (Eq. 4)
 *   lse_c   : [batch, heads, N] fp32 (written), or NULL
 * The pooled rows are rounded to dtype before the attention (as the inputs of the fine branch
 * are); the softmax and accumulation are fp32. Uses the workspace of vsa2_workspace_size().
 * With VSA2_FLAG_COARSE_POOL_IN_ROUTER (see the flag) Qc and Kc are the ones the preceding
 * vsa2_router_scores call left in the workspace, and only V is read here.
 */
vsa2_status vsa2_coarse_attn(const vsa2_problem* p, const void* q, const void* k, const void* v, void* oc,
                             float* lse_c, void* ws, size_t ws_bytes, void* stream);

/*
 * Gated merge, Eq. 4 and Eq. 13-14 (§2.2 "Gated Merge"):
 *   o[b,h,t,:] = tanh(gate_logits[b,h,t]) * oc[b,h,t/64,:] + o_f[b,h,t,:]
 *   o_f         : [batch, heads, L, D] of dtype (read only): the fine branch output (Eq. 12)
 *   gate_logits : [batch, heads, L] fp32 (read only): X W_g of Eq. 13, one value per token and
 *                 head (the projection of the hidden states is the caller's, like Q, K, V)
 *   oc          : [batch, heads, N, D] of dtype (read only): O_c_hat from vsa2_coarse_attn
 *   o           : [batch, heads, L, D] of dtype (written); may be the same buffer as o_f
 * The result is formed in fp32 (one fused multiply-add) and rounded once to dtype. Takes no
 * workspace.
 */
vsa2_status vsa2_gated_merge(const vsa2_problem* p, const void* o_f, const float* gate_logits, const void* oc,
                             void* o, void* stream);

/*
 * Gradients of the gated merge, Eq. 4 and Eq. 13-14. With G = tanh(gate_logits):
 *   d_logits[b,h,t] = (1 - G[t]^2) * sum_d dout[b,h,t,d] * oc[b,h,t/64,d]
 *   d_oc[b,h,i,:]   = sum over the 64 tokens t of tile i of G[t] * dout[b,h,t,:]
 * The fine branch's output gradient is dout itself (pass dout to vsa2_sparse_attn_bwd).
 *   dout        : [batch, heads, L, D] of dtype (read only), the gradient of o
 *   gate_logits : [batch, heads, L] fp32 (read only); oc : [batch, heads, N, D] of dtype
 *   d_logits    : [batch, heads, L] fp32 (written); d_oc : [batch, heads, N, D] fp32 (written)
 * On a padded grid the outputs of padding rows are dropped: d_logits is 0 there and d_oc sums
 * the real tokens of each tile. Takes no workspace.
 */
vsa2_status vsa2_gated_merge_bwd(const vsa2_problem* p, const void* dout, const float* gate_logits, const void* oc,
                                 float* d_logits, float* d_oc, void* stream);

/*
 * Gradients of the coarse branch, Eq. 1-3, ADDED to dq, dk, dv. With P_c and O_c_hat = oc:
 *   dS = P_c * (d_oc Vc^T - rowsum(d_oc * oc)),  dQc = dS Kc / sqrt(D),  dKc = dS^T Qc / sqrt(D),
 *   dVc = P_c^T d_oc, and MeanPool_B's adjoint spreads them: dq[t] += dQc[t/64] / 64 (same for
 *   dk, dv); on a padded grid the n real tokens of a tile get dQc / n and padding tokens
 *   nothing. Call it after vsa2_sparse_attn_bwd (which overwrites dq, dk, dv) to obtain the
 *   gradients of the whole Eq. 14 output.
 *   q, k, v : [batch, heads, L, D] of dtype (read only)
 *   oc      : [batch, heads, N, D] of dtype and lse_c : [batch, heads, N] fp32, from
 *             vsa2_coarse_attn (read only)
 *   d_oc    : [batch, heads, N, D] fp32 (read only), e.g. from vsa2_gated_merge_bwd; rounded to
 *             dtype for the tensor cores
 *   dq, dk, dv : [batch, heads, L, D] fp32 (read and written: +=)
 * Uses the workspace of vsa2_workspace_size().
 */
vsa2_status vsa2_coarse_attn_bwd(const vsa2_problem* p, const void* q, const void* k, const void* v, const void* oc,
                                 const float* lse_c, const float* d_oc, float* dq, float* dk, float* dv, void* ws,
                                 size_t ws_bytes, void* stream);

/*
 * Token permutation, §2.2 "Permutation": between raster order (t, h, w), t slowest, and the
 * cube-major order every other call takes (tiles of tile_t x tile_h x tile_w tokens in raster
 * order; inside a tile its pool_t x pool_h x pool_w sub-cubes in raster order; inside a
 * sub-cube its tokens in raster order). The paper applies it once at the start of the
 * transformer; it costs one read and one write of the tensor.
 *   src, dst      : [batch, heads, L, D] of dtype, non-overlapping buffers (dst written);
 *                   src == dst returns VSA2_ERR_INVALID_ARG
 *   to_cube_major : nonzero: src is in raster order, dst in cube-major order; zero: the inverse
 * Takes no workspace.
 */
vsa2_status vsa2_permute_tokens(const vsa2_problem* p, const void* src, void* dst, int32_t to_cube_major,
                                void* stream);

/*
 * End-to-end forward from HOST memory: router (Eq. 5-7), per-sequence TopK (Eq. 8-9) and
 * block-sparse attention (Eq. 12) for inputs and outputs that live in host memory. It computes
 * exactly what vsa2_router_scores + vsa2_topk_select + vsa2_sparse_attn_fwd compute on device
 * copies of the same inputs (bit-identical O and LSE).
 *   q, k, v  : HOST pointers, [batch, heads, L, D] of dtype (read only). Page-locked memory
 *              (cudaHostAlloc / cudaHostRegister) lets the copies overlap the kernels; pageable
 *              memory works but the host-to-device copies then block the calling thread.
 *   topk     : per-tile budget as for vsa2_topk_select
 *   heads_per_group : flat (b, h) indices processed per group, >= 0; 0 picks a group of at
 *              least 65536 tokens (one head at 720p)
 *   o        : HOST pointer, [batch, heads, L, D] of dtype (written)
 *   lse      : HOST pointer, [batch, heads, L] fp32 (written), or NULL
 *   ws       : DEVICE workspace of vsa2_forward_host_workspace_size() bytes, 256-byte aligned,
 *              initialised by vsa2_workspace_init. It holds the kernels' workspace (its error
 *              word is read by vsa2_get_device_error), one group's scores and CSR, and three
 *              staging slots of one group's Q, K, V, O and LSE.
 * The flat (b, h) range is cut into groups; group g's host-to-device copies, its kernels on
 * `stream`, and its device-to-host copies run as three chains, so that the copies of
 * neighbouring groups overlap group g's kernels. The copies run on two library-owned streams
 * that wait for the work already queued on `stream` and that `stream` waits for before any
 * later work: the outputs are in host memory once `stream` has been synchronised. The library
 * creates those two streams and a few events on the first call on each device and keeps them
 * for the process; concurrent calls from several host threads are serialised while they
 * enqueue. Argument errors return before anything is enqueued; a failed copy or launch
 * returns VSA2_ERR_CUDA after the streams have been joined.
 */
size_t vsa2_forward_host_workspace_size(const vsa2_problem* p, int32_t topk, int32_t heads_per_group);

vsa2_status vsa2_forward_host(const vsa2_problem* p, const void* q, const void* k, const void* v, int32_t topk,
                              int32_t heads_per_group, void* o, float* lse, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Per-sequence TopK like vsa2_topk_select (same ranking, same CSR output, no CSC), for callers
 * that cannot allocate device memory when they call in: for example a host program whose device
 * memory is entirely owned by another allocator or pool, or a call site where the implicit
 * synchronisation of cudaMalloc is not acceptable. It takes no workspace and allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine). This entry point has no counterpart
 * in the paper.
 *   scores, topk, kv_off, kv_idx : as for vsa2_topk_select
 * Scratch: a fixed 8 MiB array in the library's device image, held by every GPU that loads
 * the library until the process exits. One call needs
 *   256 + 256*ceil(batch*heads*24576/256) + 256*ceil(batch*heads*32/256) + 3*256*ceil(batch*heads*N*4/256)
 * bytes of it (about batch*heads*(24.6 KiB + 12*N)); larger problems return VSA2_ERR_UNSUPPORTED
 * before anything is enqueued. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and should come before any stream capture. Every call shares the one
 * array, which keeps the previous call's contents (the call clears what must start at zero):
 * calls that may overlap on the GPU, on any streams, race. VSA2_FLAG_VALIDATE is ignored.
 */
vsa2_status vsa2_topk_select_noalloc(const vsa2_problem* p, const float* scores, int32_t topk,
                                     int32_t* kv_off, int32_t* kv_idx, void* stream);

/* Synchronise `stream`, read and clear the device error word of `ws`. Returns VSA2_OK,
 * VSA2_ERR_TIMEOUT, VSA2_ERR_BAD_INDEX, or VSA2_ERR_CUDA if the synchronisation failed. */
vsa2_status vsa2_get_device_error(void* ws, void* stream);

/* Diagnostic: enqueue one kernel that waits, with the problem's bounded wait, on a barrier
 * that nothing completes. It returns after `timeout_ms` and records VSA2_ERR_TIMEOUT in the
 * workspace error word; no GPU state other than that word is touched. */
vsa2_status vsa2_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t timeout_ms, void* stream);

/* Human-readable name of a status code (static storage). */
const char* vsa2_status_string(vsa2_status s);

/* Message of the last failed CUDA call or launch inside the library (static or per-thread
 * storage; valid until the next failure on the same thread). */
const char* vsa2_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t vsa2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA2_H_ */
