"""ctypes binding of libvsa2.so: the C entry points under the same names, with torch tensors
marshalled to device pointers. No arithmetic of the method happens here."""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvsa2.so")

VSA2_OK = 0
STATUS_NAMES = {0: "VSA2_OK", 1: "VSA2_ERR_INVALID_ARG", 2: "VSA2_ERR_UNSUPPORTED", 3: "VSA2_ERR_CUDA",
                4: "VSA2_ERR_TIMEOUT", 5: "VSA2_ERR_BAD_INDEX"}
VSA2_BF16, VSA2_FP32 = 0, 1
VSA2_FLAG_VALIDATE = 1
VSA2_FLAG_COARSE_POOL_IN_ROUTER = 2

# every symbol the header declares
EXPORTS = ("vsa2_workspace_size", "vsa2_workspace_init", "vsa2_router_scores", "vsa2_topk_select",
           "vsa2_sparse_attn_fwd", "vsa2_sparse_attn_bwd", "vsa2_get_device_error",
           "vsa2_selftest_wait_timeout", "vsa2_status_string", "vsa2_version", "vsa2_last_cuda_error",
           "vsa2_topk_select_noalloc", "vsa2_forward_host", "vsa2_forward_host_workspace_size",
           "vsa2_coarse_attn", "vsa2_gated_merge", "vsa2_gated_merge_bwd", "vsa2_coarse_attn_bwd",
           "vsa2_permute_tokens", "vsa2_topk_select_per_row", "vsa2_sparse_attn_fwd_gated")


class Vsa2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("heads", ctypes.c_int64), ("head_dim", ctypes.c_int64),
                ("grid_t", ctypes.c_int64), ("grid_h", ctypes.c_int64), ("grid_w", ctypes.c_int64),
                ("tile_t", ctypes.c_int32), ("tile_h", ctypes.c_int32), ("tile_w", ctypes.c_int32),
                ("pool_t", ctypes.c_int32), ("pool_h", ctypes.c_int32), ("pool_w", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32), ("wait_timeout_ms", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libvsa2.so (built in-tree). Fails loudly when it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with trainable_block_sparse_fine_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Problem)
        vp, sz, i32, u32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint32
        L.vsa2_workspace_size.argtypes = [P, i32]
        L.vsa2_workspace_size.restype = sz
        L.vsa2_workspace_init.argtypes = [vp, sz, vp]
        L.vsa2_router_scores.argtypes = [P, vp, vp, vp, vp, sz, vp]
        L.vsa2_topk_select.argtypes = [P, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_sparse_attn_fwd.argtypes = [P, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_sparse_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_topk_select_noalloc.argtypes = [P, vp, i32, vp, vp, vp]
        L.vsa2_topk_select_per_row.argtypes = [P, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_sparse_attn_fwd_gated.argtypes = [P, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_forward_host_workspace_size.argtypes = [P, i32, i32]
        L.vsa2_forward_host_workspace_size.restype = sz
        L.vsa2_forward_host.argtypes = [P, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.vsa2_coarse_attn.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_gated_merge.argtypes = [P, vp, vp, vp, vp, vp]
        L.vsa2_gated_merge_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.vsa2_permute_tokens.argtypes = [P, vp, vp, i32, vp]
        L.vsa2_coarse_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.vsa2_get_device_error.argtypes = [vp, vp]
        L.vsa2_selftest_wait_timeout.argtypes = [vp, sz, u32, vp]
        L.vsa2_status_string.argtypes = [ctypes.c_int]
        L.vsa2_status_string.restype = ctypes.c_char_p
        L.vsa2_version.restype = i32
        L.vsa2_last_cuda_error.restype = ctypes.c_char_p
        for name in ("vsa2_workspace_init", "vsa2_router_scores", "vsa2_topk_select", "vsa2_topk_select_noalloc",
                     "vsa2_topk_select_per_row", "vsa2_sparse_attn_fwd_gated",
                     "vsa2_sparse_attn_fwd", "vsa2_forward_host", "vsa2_coarse_attn", "vsa2_gated_merge",
                     "vsa2_gated_merge_bwd", "vsa2_coarse_attn_bwd", "vsa2_permute_tokens",
                     "vsa2_sparse_attn_bwd", "vsa2_get_device_error", "vsa2_selftest_wait_timeout"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != VSA2_OK:
        if status == 3:
            where = f"{where} ({lib().vsa2_last_cuda_error().decode()})"
        raise Vsa2Error(status, where)


def make_problem(batch, heads, head_dim, grid, dtype="bf16", tile=(4, 4, 4), pool=(2, 2, 4), flags=0,
                 wait_timeout_ms=0) -> Problem:
    return Problem(batch, heads, head_dim, *grid, *tile, *pool, VSA2_BF16 if dtype == "bf16" else VSA2_FP32,
                   flags, wait_timeout_ms, 0)


def vsa2_workspace_size(p: Problem, topk: int) -> int:
    return lib().vsa2_workspace_size(ctypes.byref(p), topk)


def vsa2_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().vsa2_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "vsa2_workspace_init")


def vsa2_router_scores(p: Problem, q, k, scores, ws, stream=None) -> None:
    _check(lib().vsa2_router_scores(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(scores), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "vsa2_router_scores")


def vsa2_topk_select(p: Problem, scores, topk, kv_off, kv_idx, q_off, q_idx, ws, stream=None) -> None:
    _check(lib().vsa2_topk_select(ctypes.byref(p), _ptr(scores), topk, _ptr(kv_off), _ptr(kv_idx), _ptr(q_off),
                                  _ptr(q_idx), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "vsa2_topk_select")


def vsa2_topk_select_per_row(p: Problem, scores, topk, kv_off, kv_idx, q_off, q_idx, ws, stream=None) -> None:
    _check(lib().vsa2_topk_select_per_row(ctypes.byref(p), _ptr(scores), topk, _ptr(kv_off), _ptr(kv_idx),
                                          _ptr(q_off), _ptr(q_idx), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream(stream)), "vsa2_topk_select_per_row")


def vsa2_topk_select_noalloc(p: Problem, scores, topk, kv_off, kv_idx, stream=None) -> None:
    """TopK (CSR only) that allocates nothing: its scratch is a fixed device array in the library."""
    _check(lib().vsa2_topk_select_noalloc(ctypes.byref(p), _ptr(scores), topk, _ptr(kv_off), _ptr(kv_idx),
                                          _stream(stream)), "vsa2_topk_select_noalloc")


def vsa2_sparse_attn_fwd(p: Problem, q, k, v, topk, kv_off, kv_idx, o, lse, ws, stream=None) -> None:
    _check(lib().vsa2_sparse_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), topk, _ptr(kv_off), _ptr(kv_idx),
                                      _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "vsa2_sparse_attn_fwd")


def vsa2_sparse_attn_fwd_gated(p: Problem, q, k, v, topk, kv_off, kv_idx, gate_logits, oc, o, lse, o_f, ws,
                               stream=None) -> None:
    _check(lib().vsa2_sparse_attn_fwd_gated(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), topk, _ptr(kv_off),
                                            _ptr(kv_idx), _ptr(gate_logits), _ptr(oc), _ptr(o), _ptr(lse), _ptr(o_f),
                                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "vsa2_sparse_attn_fwd_gated")


def vsa2_sparse_attn_bwd(p: Problem, q, k, v, o, lse, dout, topk, kv_off, kv_idx, q_off, q_idx, dq, dk, dv, ws,
                         stream=None) -> None:
    _check(lib().vsa2_sparse_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                      topk, _ptr(kv_off), _ptr(kv_idx), _ptr(q_off), _ptr(q_idx), _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "vsa2_sparse_attn_bwd")


def vsa2_coarse_attn(p: Problem, q, k, v, oc, lse_c, ws, stream=None) -> None:
    _check(lib().vsa2_coarse_attn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(oc), _ptr(lse_c), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "vsa2_coarse_attn")


def vsa2_gated_merge(p: Problem, o_f, gate_logits, oc, o, stream=None) -> None:
    _check(lib().vsa2_gated_merge(ctypes.byref(p), _ptr(o_f), _ptr(gate_logits), _ptr(oc), _ptr(o), _stream(stream)),
           "vsa2_gated_merge")


def vsa2_gated_merge_bwd(p: Problem, dout, gate_logits, oc, d_logits, d_oc, stream=None) -> None:
    _check(lib().vsa2_gated_merge_bwd(ctypes.byref(p), _ptr(dout), _ptr(gate_logits), _ptr(oc), _ptr(d_logits),
                                      _ptr(d_oc), _stream(stream)), "vsa2_gated_merge_bwd")


def vsa2_coarse_attn_bwd(p: Problem, q, k, v, oc, lse_c, d_oc, dq, dk, dv, ws, stream=None) -> None:
    _check(lib().vsa2_coarse_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(oc), _ptr(lse_c), _ptr(d_oc),
                                      _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "vsa2_coarse_attn_bwd")


def vsa2_permute_tokens(p: Problem, src, dst, to_cube_major: bool, stream=None) -> None:
    _check(lib().vsa2_permute_tokens(ctypes.byref(p), _ptr(src), _ptr(dst), 1 if to_cube_major else 0,
                                     _stream(stream)), "vsa2_permute_tokens")


def vsa2_forward_host_workspace_size(p: Problem, topk: int, heads_per_group: int = 0) -> int:
    return lib().vsa2_forward_host_workspace_size(ctypes.byref(p), topk, heads_per_group)


def vsa2_forward_host(p: Problem, q, k, v, topk, heads_per_group, o, lse, ws, stream=None) -> None:
    """q, k, v, o, lse are HOST tensors (page-locked for overlap); lse may be None."""
    for t in (q, k, v, o, lse):
        if isinstance(t, torch.Tensor) and t.is_cuda:
            raise ValueError("vsa2_forward_host takes host tensors")
    _check(lib().vsa2_forward_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), topk, heads_per_group, _ptr(o),
                                   _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "vsa2_forward_host")


def vsa2_get_device_error(ws, stream=None) -> int:
    return lib().vsa2_get_device_error(_ptr(ws), _stream(stream))


def vsa2_selftest_wait_timeout(ws, timeout_ms: int, stream=None) -> None:
    _check(lib().vsa2_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), timeout_ms, _stream(stream)),
           "vsa2_selftest_wait_timeout")


def vsa2_status_string(status: int) -> str:
    return lib().vsa2_status_string(status).decode()


def vsa2_version() -> int:
    return lib().vsa2_version()
