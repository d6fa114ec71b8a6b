"""Host-side checks of the C ABI that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments synchronously (nothing is enqueued)."""
import ctypes
import os
import re

import pytest

import synthetic as S
from trainable_block_sparse_fine_b200 import _capi as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "vsa2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa2_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = C.lib()
    declared = _declared_symbols()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(C.EXPORTS)


def test_problem_struct_layout():
    assert ctypes.sizeof(C.Problem) == 88
    assert C.Problem.dtype.offset == 72


def test_flag_values_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "vsa2.h")).read(), flags=re.S)
    flags = {name: 1 << int(bit) for name, bit in re.findall(r"\b(VSA2_FLAG_[A-Z_]+)\s*=\s*1u\s*<<\s*(\d+)", text)}
    assert flags == {"VSA2_FLAG_VALIDATE": C.VSA2_FLAG_VALIDATE,
                     "VSA2_FLAG_COARSE_POOL_IN_ROUTER": C.VSA2_FLAG_COARSE_POOL_IN_ROUTER}


def test_status_strings_and_version():
    for code, name in C.STATUS_NAMES.items():
        assert C.vsa2_status_string(code) == name
    assert C.vsa2_version() >= 100


@pytest.mark.parametrize("name", list(S.WORKLOADS))
def test_workspace_size_for_every_workload(name):
    wl = S.WORKLOADS[name]
    p = C.make_problem(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype)
    n = C.vsa2_workspace_size(p, wl.topk)
    assert n > 0 and n % 256 == 0
    # pooled Q and K dominate; the workspace stays far below device memory
    assert n < 1 << 30


def test_unsupported_shapes_give_zero_workspace():
    assert C.vsa2_workspace_size(C.make_problem(1, 2, 96, (8, 16, 16)), 8) == 0  # head_dim
    assert C.vsa2_workspace_size(C.make_problem(1, 2, 64, (8, 16, 16), pool=(2, 2, 2)), 8) == 0  # R != 16
    assert C.vsa2_workspace_size(C.make_problem(1, 2, 64, (8, 16, 16), tile=(4, 4, 4), pool=(3, 2, 4)), 8) == 0


def test_128_token_tiles_take_a_budget_dependent_workspace():
    """B = 128, R = 8: the workspace holds the selection expanded to 64-token tiles, so it grows
    with the budget; grids the 128-token tile does not divide are not taken."""
    p = C.make_problem(1, 2, 128, (8, 16, 32), tile=(4, 4, 8), pool=(2, 2, 2))
    a, b = C.vsa2_workspace_size(p, 2), C.vsa2_workspace_size(p, 8)
    assert 0 < a < b
    assert C.vsa2_workspace_size(p, 0) > 0  # the router and the TopK need no expansion
    assert C.vsa2_workspace_size(C.make_problem(1, 2, 128, (8, 16, 30), tile=(4, 4, 8), pool=(2, 2, 2)), 2) == 0
    assert C.vsa2_workspace_size(C.make_problem(1, 2, 128, (8, 16, 32), tile=(4, 4, 8), pool=(2, 2, 4)), 2) == 0


def test_grid_the_tile_does_not_divide_is_padded():
    """6x7x10 pads to 8x8x12 (24 tiles): the workspace is the padded problem's, as for 8x8x12."""
    padded = C.vsa2_workspace_size(C.make_problem(1, 2, 64, (6, 7, 10)), 3)
    whole = C.vsa2_workspace_size(C.make_problem(1, 2, 64, (8, 8, 12)), 3)
    assert padded > 0 and padded == whole


def test_argument_errors_are_synchronous():
    lib = C.lib()
    p = C.make_problem(1, 2, 64, (8, 16, 16), "fp32")
    bp = ctypes.byref(p)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails before any launch
    ws = ctypes.c_void_p(1 << 24)
    n = C.vsa2_workspace_size(p, 8)
    # null pointers
    assert lib.vsa2_router_scores(bp, None, fake, fake, ws, n, None) == 1
    # misaligned pointer
    assert lib.vsa2_router_scores(bp, ctypes.c_void_p((1 << 20) + 4), fake, fake, ws, n, None) == 1
    # workspace too small
    assert lib.vsa2_router_scores(bp, fake, fake, fake, ws, n - 256, None) == 1
    # topk out of range
    assert lib.vsa2_topk_select(bp, fake, 0, fake, fake, None, None, ws, n, None) == 2
    assert lib.vsa2_topk_select(bp, fake, 33, fake, fake, None, None, ws, n, None) == 2
    # CSC pointers must come as a pair
    assert lib.vsa2_topk_select(bp, fake, 8, fake, fake, fake, None, ws, n, None) == 1
    assert lib.vsa2_topk_select_per_row(bp, fake, 8, fake, fake, fake, None, ws, n, None) == 1
    assert lib.vsa2_topk_select_per_row(bp, fake, 0, fake, fake, None, None, ws, n, None) == 2
    assert lib.vsa2_topk_select_per_row(bp, fake, 8, fake, fake, None, None, ws, n - 256, None) == 1
    assert lib.vsa2_sparse_attn_fwd(bp, fake, fake, fake, 8, fake, None, fake, fake, ws, n, None) == 1
    assert lib.vsa2_sparse_attn_bwd(bp, fake, fake, fake, fake, fake, fake, 8, fake, fake, None, fake, fake, fake,
                                    fake, ws, n, None) == 1
    bad = C.make_problem(1, 2, 64, (8, 16, 16), "fp32")
    bad.dtype = 7
    assert lib.vsa2_router_scores(ctypes.byref(bad), fake, fake, fake, ws, n, None) == 2
    assert lib.vsa2_selftest_wait_timeout(ws, n, 0, None) == 1


def test_forward_host_workspace_and_argument_errors():
    lib = C.lib()
    p = C.make_problem(1, 5, 128, (8, 16, 20))  # N = 40, L = 2560
    bp = ctypes.byref(p)
    one = C.vsa2_forward_host_workspace_size(p, 6, 1)
    two = C.vsa2_forward_host_workspace_size(p, 6, 2)
    auto = C.vsa2_forward_host_workspace_size(p, 6, 0)
    everything = C.vsa2_forward_host_workspace_size(p, 6, 5)
    assert 0 < one < two < auto and one % 256 == 0
    assert auto == everything  # 65536 tokens round up to all five heads here
    assert C.vsa2_forward_host_workspace_size(p, 6, 9) == everything  # clamped to the head count
    # three staging slots of Q, K, V, O (bf16) and LSE (fp32) for one head at least
    assert one >= 3 * (4 * 2560 * 128 * 2 + 2560 * 4)
    assert C.vsa2_forward_host_workspace_size(p, 0, 1) == 0
    assert C.vsa2_forward_host_workspace_size(p, 41, 1) == 0
    assert C.vsa2_forward_host_workspace_size(p, 6, -1) == 0
    host = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails before any copy
    ws = ctypes.c_void_p(1 << 24)
    assert lib.vsa2_forward_host(bp, None, host, host, 6, 1, host, None, ws, one, None) == 1
    assert lib.vsa2_forward_host(bp, host, host, host, 6, 1, None, None, ws, one, None) == 1
    assert lib.vsa2_forward_host(bp, host, host, host, 6, 1, host, None, ws, one - 256, None) == 1
    assert lib.vsa2_forward_host(bp, host, host, host, 6, 1, host, None, ctypes.c_void_p((1 << 24) + 16), one,
                                 None) == 1
    assert lib.vsa2_forward_host(bp, host, host, host, 6, -1, host, None, ws, one, None) == 1
    assert lib.vsa2_forward_host(bp, host, host, host, 0, 1, host, None, ws, one, None) == 2


def test_coarse_and_merge_argument_errors():
    lib = C.lib()
    p = C.make_problem(1, 2, 128, (8, 16, 20))
    bp = ctypes.byref(p)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails before any launch
    ws = ctypes.c_void_p(1 << 24)
    n = C.vsa2_workspace_size(p, 6)
    assert lib.vsa2_coarse_attn(bp, fake, fake, None, fake, None, ws, n, None) == 1
    assert lib.vsa2_coarse_attn(bp, fake, fake, fake, ctypes.c_void_p((1 << 20) + 8), None, ws, n, None) == 1
    assert lib.vsa2_coarse_attn(bp, fake, fake, fake, fake, None, ws, n - 256, None) == 1
    assert lib.vsa2_gated_merge(bp, fake, None, fake, fake, None) == 1
    assert lib.vsa2_gated_merge(bp, fake, fake, fake, ctypes.c_void_p((1 << 20) + 2), None) == 1
    bad = C.make_problem(1, 2, 96, (8, 16, 20))
    assert lib.vsa2_gated_merge(ctypes.byref(bad), fake, fake, fake, fake, None) == 2


def test_permute_argument_errors():
    lib = C.lib()
    p = C.make_problem(1, 2, 128, (8, 16, 20))
    bp = ctypes.byref(p)
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)  # never dereferenced
    assert lib.vsa2_permute_tokens(bp, a, a, 1, None) == 1  # in place
    assert lib.vsa2_permute_tokens(bp, None, b, 1, None) == 1
    assert lib.vsa2_permute_tokens(bp, a, ctypes.c_void_p((1 << 24) + 4), 0, None) == 1
    bad = C.make_problem(1, 2, 128, (8, 16, 20), tile=(4, 4, 2))  # tile of 32 tokens
    assert lib.vsa2_permute_tokens(ctypes.byref(bad), a, b, 1, None) == 2
