"""VSA2 hot path on B200: fine-grained router -> per-sequence TopK -> block-sparse attention.

Every step runs in the CUDA kernels of libvsa2.so (see include/vsa2.h); this module only
allocates device memory with PyTorch and marshals arguments. Method: "Improving Video Sparse
Attention with Fine-grained Router and Sparse Rebasing" (arXiv 2609.32882), §2.2.

Inputs are [batch, heads, L, D] tensors in cube-major token order (tiles of 4x4x4 tokens,
router sub-cubes of 2x2x4 tokens inside each tile).
"""
from __future__ import annotations

import torch

from ._capi import (VSA2_FLAG_COARSE_POOL_IN_ROUTER, VSA2_FLAG_VALIDATE, Problem, Vsa2Error, lib, make_problem, vsa2_coarse_attn,
                    vsa2_coarse_attn_bwd, vsa2_forward_host, vsa2_forward_host_workspace_size, vsa2_gated_merge,
                    vsa2_gated_merge_bwd, vsa2_get_device_error, vsa2_permute_tokens, vsa2_router_scores,
                    vsa2_selftest_wait_timeout, vsa2_sparse_attn_bwd, vsa2_sparse_attn_fwd,
                    vsa2_sparse_attn_fwd_gated, vsa2_status_string,
                    vsa2_topk_select, vsa2_topk_select_per_row, vsa2_version, vsa2_workspace_init, vsa2_workspace_size)

from .ulysses import heads_to_seq, seq_to_heads, ulysses_attention

__all__ = ["VSA2", "ulysses_attention", "seq_to_heads", "heads_to_seq", "Vsa2Error", "Problem", "make_problem", "block_sparse_attention", "lib", "VSA2_FLAG_VALIDATE", "VSA2_FLAG_COARSE_POOL_IN_ROUTER",
           "vsa2_router_scores", "vsa2_topk_select", "vsa2_sparse_attn_fwd", "vsa2_sparse_attn_bwd",
           "vsa2_workspace_size", "vsa2_workspace_init", "vsa2_get_device_error", "vsa2_selftest_wait_timeout",
           "vsa2_status_string", "vsa2_version", "vsa2_forward_host", "vsa2_forward_host_workspace_size",
           "vsa2_coarse_attn", "vsa2_gated_merge", "vsa2_gated_merge_bwd", "vsa2_coarse_attn_bwd", "vsa2_attention",
           "vsa2_permute_tokens"]


class VSA2:
    """One problem shape with its workspace; methods enqueue on the current CUDA stream."""

    def __init__(self, batch, heads, head_dim, grid, dtype="bf16", topk=64, device="cuda", flags=0,
                 wait_timeout_ms=0, tile=(4, 4, 4), pool=(2, 2, 4)):
        """tile / pool: the token cube of a tile and of a router sub-cube, 64 / 16 tokens (the
        pages' shapes, default) or 128 / 8 tokens (e.g. (4, 4, 8) / (2, 2, 2))."""
        if not torch.cuda.is_available():
            raise RuntimeError("VSA2 needs a CUDA device")
        lib()  # fail loudly if the native library is missing
        self.p = make_problem(batch, heads, head_dim, grid, dtype, tile=tuple(tile), pool=tuple(pool), flags=flags,
                              wait_timeout_ms=wait_timeout_ms)
        # the same problem for the whole-attention calls: the router's pass over Q and K also
        # writes the coarse branch's pooled Qc, Kc (Eq. 1), and the coarse call then reads only V
        self.p_fold = make_problem(batch, heads, head_dim, grid, dtype, tile=tuple(tile), pool=tuple(pool),
                                   flags=flags | VSA2_FLAG_COARSE_POOL_IN_ROUTER, wait_timeout_ms=wait_timeout_ms)
        self.tile, self.pool = tuple(tile), tuple(pool)
        self.batch, self.heads, self.head_dim, self.grid, self.topk = batch, heads, head_dim, tuple(grid), topk
        # a grid the 4x4x4 tile does not divide is padded to whole tiles (§2.2 "Kernel
        # Implementation"): every [B, H, L, D] tensor of the path holds the padded grid in
        # cube-major order; to_cube_major / to_raster pad and crop
        self.L_real = grid[0] * grid[1] * grid[2]
        self.grid_padded = tuple(-(-g // b) * b for g, b in zip(grid, self.tile))
        self.L = self.grid_padded[0] * self.grid_padded[1] * self.grid_padded[2]
        self.N = self.L // (self.tile[0] * self.tile[1] * self.tile[2])
        self.dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.device = torch.device(device)
        n = vsa2_workspace_size(self.p, topk)
        if n == 0:
            raise Vsa2Error(2, "vsa2_workspace_size")
        self.ws = torch.empty((n + 255) // 256 * 256, dtype=torch.uint8, device=self.device)
        vsa2_workspace_init(self.ws)

    # -- the calls of the hot path -----------------------------------------------------------
    def router_scores(self, q, k, out=None, coarse_pool=False):
        """Eq. 5-7 scores [B, H, N, N]. coarse_pool: also leave the coarse branch's pooled Q and K
        in the workspace for a following coarse_attn(..., pooled_qk=True)."""
        out = out if out is not None else torch.empty(self.batch, self.heads, self.N, self.N, dtype=torch.float32,
                                                      device=self.device)
        vsa2_router_scores(self.p_fold if coarse_pool else self.p, q, k, out, self.ws)
        return out

    def topk_select(self, scores, topk=None, csc=True):
        topk = self.topk if topk is None else topk
        bh = (self.batch, self.heads)
        i32 = dict(dtype=torch.int32, device=self.device)
        kv_off = torch.empty(*bh, self.N + 1, **i32)
        kv_idx = torch.empty(*bh, self.N * topk, **i32)
        q_off = torch.empty(*bh, self.N + 1, **i32) if csc else None
        q_idx = torch.empty(*bh, self.N * topk, **i32) if csc else None
        vsa2_topk_select(self.p, scores, topk, kv_off, kv_idx, q_off, q_idx, self.ws)
        return kv_off, kv_idx, q_off, q_idx

    def topk_select_per_row(self, scores, topk=None, csc=True):
        """VSA's per-query-tile TopK: every query tile keeps its own `topk` best KV tiles."""
        topk = self.topk if topk is None else topk
        bh = (self.batch, self.heads)
        i32 = dict(dtype=torch.int32, device=self.device)
        kv_off = torch.empty(*bh, self.N + 1, **i32)
        kv_idx = torch.empty(*bh, self.N * topk, **i32)
        q_off = torch.empty(*bh, self.N + 1, **i32) if csc else None
        q_idx = torch.empty(*bh, self.N * topk, **i32) if csc else None
        vsa2_topk_select_per_row(self.p, scores, topk, kv_off, kv_idx, q_off, q_idx, self.ws)
        return kv_off, kv_idx, q_off, q_idx

    def attn_fwd(self, q, k, v, kv_off, kv_idx, topk=None, o=None, lse=None):
        topk = self.topk if topk is None else topk
        o = o if o is not None else torch.empty_like(q)
        lse = lse if lse is not None else torch.empty(self.batch, self.heads, self.L, dtype=torch.float32,
                                                      device=self.device)
        vsa2_sparse_attn_fwd(self.p, q, k, v, topk, kv_off, kv_idx, o, lse, self.ws)
        return o, lse

    def attn_fwd_gated(self, q, k, v, kv_off, kv_idx, gate_logits, oc, topk=None, want_fine=False):
        """Eq. 12 with the gated merge of Eq. 13-14 in the same pass: returns (o, lse, o_f), o_f the
        fine output alone when want_fine (the backward needs it), else None."""
        topk = self.topk if topk is None else topk
        o = torch.empty_like(q)
        lse = torch.empty(self.batch, self.heads, self.L, dtype=torch.float32, device=self.device)
        o_f = torch.empty_like(q) if want_fine else None
        vsa2_sparse_attn_fwd_gated(self.p, q, k, v, topk, kv_off, kv_idx, gate_logits, oc, o, lse, o_f, self.ws)
        return o, lse, o_f

    def attn_bwd(self, q, k, v, o, lse, dout, kv_off, kv_idx, q_off, q_idx, topk=None):
        topk = self.topk if topk is None else topk
        f32 = dict(dtype=torch.float32, device=self.device)
        dq, dk, dv = (torch.empty(q.shape, **f32) for _ in range(3))
        vsa2_sparse_attn_bwd(self.p, q, k, v, o, lse, dout, topk, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, self.ws)
        return dq, dk, dv

    def forward(self, q, k, v, topk=None, csc=False):
        """Router -> TopK -> block-sparse attention forward. Returns (o, lse, selection)."""
        scores = self.router_scores(q, k)
        sel = self.topk_select(scores, topk, csc=csc)
        o, lse = self.attn_fwd(q, k, v, sel[0], sel[1], topk)
        return o, lse, sel

    def to_cube_major(self, x, out=None):
        """[B, H, T*H*W, D] (or [B, H, T, H, W, D]) in raster token order -> [B, H, L, D] cube-major
        (padding tokens of a grid the tile does not divide are written as zeros)."""
        out = out if out is not None else torch.empty(self.batch, self.heads, self.L, self.head_dim, dtype=x.dtype,
                                                      device=self.device)
        vsa2_permute_tokens(self.p, x, out, True)
        return out

    def to_raster(self, x, out=None):
        """[B, H, L, D] cube-major -> [B, H, T*H*W, D] in raster token order (t, h, w), padding
        tokens dropped."""
        out = out if out is not None else torch.empty(self.batch, self.heads, self.L_real, self.head_dim,
                                                      dtype=x.dtype, device=self.device)
        vsa2_permute_tokens(self.p, x, out, False)
        return out

    def coarse_attn(self, q, k, v, oc=None, lse_c=None, pooled_qk=False):
        """Coarse branch, Eq. 1-3: O_c_hat [B, H, N, D] (input dtype) and its LSE [B, H, N].
        pooled_qk: take Qc, Kc from the preceding router_scores(q, k, coarse_pool=True) call."""
        oc = oc if oc is not None else torch.empty(self.batch, self.heads, self.N, self.head_dim, dtype=q.dtype,
                                                   device=self.device)
        lse_c = lse_c if lse_c is not None else torch.empty(self.batch, self.heads, self.N, dtype=torch.float32,
                                                            device=self.device)
        vsa2_coarse_attn(self.p_fold if pooled_qk else self.p, q, k, v, oc, lse_c, self.ws)
        return oc, lse_c

    def gated_merge(self, o_f, gate_logits, oc, out=None):
        """Eq. 4, 13-14: tanh(gate_logits) * Repeat_B(oc) + o_f; out may be o_f (in place)."""
        out = out if out is not None else torch.empty_like(o_f)
        vsa2_gated_merge(self.p, o_f, gate_logits, oc, out)
        return out

    def gated_merge_bwd(self, dout, gate_logits, oc):
        """Gradients of Eq. 4, 13-14: (d_gate_logits [B, H, L], d_oc [B, H, N, D]), fp32."""
        d_logits = torch.empty(gate_logits.shape, dtype=torch.float32, device=self.device)
        d_oc = torch.empty(oc.shape, dtype=torch.float32, device=self.device)
        vsa2_gated_merge_bwd(self.p, dout, gate_logits, oc, d_logits, d_oc)
        return d_logits, d_oc

    def coarse_attn_bwd(self, q, k, v, oc, lse_c, d_oc, dq, dk, dv):
        """Adds the coarse branch's gradients (Eq. 1-3) to the fp32 tensors dq, dk, dv."""
        vsa2_coarse_attn_bwd(self.p, q, k, v, oc, lse_c, d_oc, dq, dk, dv, self.ws)
        return dq, dk, dv

    def attention(self, q, k, v, gate_logits, topk=None):
        """The whole VSA2 attention output, Eq. 14: fine branch (router, TopK, Eq. 12) plus the
        gated coarse branch. Returns o."""
        scores = self.router_scores(q, k, coarse_pool=True)
        kv_off, kv_idx, _, _ = self.topk_select(scores, topk, csc=False)
        oc, _ = self.coarse_attn(q, k, v, pooled_qk=True)
        return self.attn_fwd_gated(q, k, v, kv_off, kv_idx, gate_logits, oc, topk)[0]

    def forward_host(self, q, k, v, topk=None, o=None, lse=None, heads_per_group=0, want_lse=False):
        """Router -> TopK -> forward on HOST tensors, copies overlapped with the kernels per group of
        heads (vsa2_forward_host). Returns (o, lse) in host memory once the current stream has been
        synchronised; lse is None unless requested."""
        topk = self.topk if topk is None else topk
        n = vsa2_forward_host_workspace_size(self.p, topk, heads_per_group)
        if n == 0:
            raise Vsa2Error(2, "vsa2_forward_host_workspace_size")
        key = (topk, heads_per_group)
        if getattr(self, "_host_ws_key", None) != key:
            self.ws_host = torch.empty((n + 255) // 256 * 256, dtype=torch.uint8, device=self.device)
            vsa2_workspace_init(self.ws_host)
            self._host_ws_key = key
        o = o if o is not None else torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        if want_lse and lse is None:
            lse = torch.empty(self.batch, self.heads, self.L, dtype=torch.float32, pin_memory=True)
        vsa2_forward_host(self.p, q, k, v, topk, heads_per_group, o, lse, self.ws_host)
        return o, lse

    def device_error(self) -> int:
        err = vsa2_get_device_error(self.ws)
        if err == 0 and getattr(self, "ws_host", None) is not None:
            err = vsa2_get_device_error(self.ws_host)
        return err


class _BlockSparseAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, engine: VSA2, topk):
        with torch.no_grad():  # the router receives no gradient (§2.1)
            scores = engine.router_scores(q, k)
            kv_off, kv_idx, q_off, q_idx = engine.topk_select(scores, topk, csc=True)
        o, lse = engine.attn_fwd(q, k, v, kv_off, kv_idx, topk)
        ctx.save_for_backward(q, k, v, o, lse, kv_off, kv_idx, q_off, q_idx)
        ctx.engine, ctx.topk = engine, topk
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse, kv_off, kv_idx, q_off, q_idx = ctx.saved_tensors
        dq, dk, dv = ctx.engine.attn_bwd(q, k, v, o, lse, dout.contiguous(), kv_off, kv_idx, q_off, q_idx, ctx.topk)
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None


class _Vsa2Attention(torch.autograd.Function):
    """Eq. 14: o = tanh(gate_logits) * Repeat_B(coarse(q, k, v)) + fine(q, k, v; router TopK)."""

    @staticmethod
    def forward(ctx, q, k, v, gate_logits, engine: VSA2, topk):
        with torch.no_grad():  # the router receives no gradient (§2.1)
            scores = engine.router_scores(q, k, coarse_pool=True)
            kv_off, kv_idx, q_off, q_idx = engine.topk_select(scores, topk, csc=True)
        oc, lse_c = engine.coarse_attn(q, k, v, pooled_qk=True)
        o, lse, o_f = engine.attn_fwd_gated(q, k, v, kv_off, kv_idx, gate_logits.contiguous(), oc, topk,
                                            want_fine=True)
        ctx.save_for_backward(q, k, v, o_f, lse, kv_off, kv_idx, q_off, q_idx, oc, lse_c, gate_logits)
        ctx.engine, ctx.topk = engine, topk
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o_f, lse, kv_off, kv_idx, q_off, q_idx, oc, lse_c, gate_logits = ctx.saved_tensors
        e = ctx.engine
        dout = dout.contiguous()
        dq, dk, dv = e.attn_bwd(q, k, v, o_f, lse, dout, kv_off, kv_idx, q_off, q_idx, ctx.topk)
        d_logits, d_oc = e.gated_merge_bwd(dout, gate_logits, oc)
        e.coarse_attn_bwd(q, k, v, oc, lse_c, d_oc, dq, dk, dv)
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), d_logits.to(gate_logits.dtype), None, None


def vsa2_attention(q, k, v, gate_logits, engine: VSA2, topk=None):
    """The whole VSA2 attention (coarse branch, router, fine branch, gated merge; Eq. 1-14) as an
    autograd function. gate_logits = X W_g (Eq. 13), fp32 [B, H, L]."""
    return _Vsa2Attention.apply(q, k, v, gate_logits, engine, engine.topk if topk is None else topk)


def block_sparse_attention(q, k, v, engine: VSA2, topk=None):
    """VSA2 fine branch with its router: o = BlockSparseAttn(q, k, v; TopK_{NK}(router(q, k)))."""
    return _BlockSparseAttention.apply(q, k, v, engine, engine.topk if topk is None else topk)
