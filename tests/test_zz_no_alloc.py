"""The allocation-free TopK entry point (vsa2_topk_select_noalloc).

Some callers cannot allocate device memory when they call in (their device memory is owned by
another allocator, or cudaMalloc's implicit synchronisation is not allowed where they call);
this entry point serves them from a fixed scratch array inside the library. These tests check
that it returns exactly what the workspace-based vsa2_topk_select returns, on two calls in a
row (the scratch keeps the previous call's contents), and that oversized problems are refused
before anything is enqueued. The file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S
from trainable_block_sparse_fine_b200 import _capi as C


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 1024 heads at 720p need far more than the 8 MiB scratch; refused on the host, no GPU needed
    p = C.make_problem(1, 1024, 128, (56, 48, 80))
    fake = ctypes.c_void_p(1 << 20)
    assert C.lib().vsa2_topk_select_noalloc(ctypes.byref(p), fake, 64, fake, fake, None) == 2


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [S.Workload("noalloc_small", 1, 2, 128, (8, 16, 20), 6, "bf16"),
                                S.WORKLOADS["480p_top64"]], ids=["small", "480p"])
def test_noalloc_matches_workspace_topk_twice(wl):
    import trainable_block_sparse_fine_b200 as V

    rng = np.random.default_rng(7)
    N = wl.num_tiles
    e = V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk)
    for call in range(2):
        s = rng.random((wl.batch, wl.heads, N, N)).astype(np.float32)
        s[..., : N // 3, :] = np.round(s[..., : N // 3, :] * 16) / 16  # exact ties in part of the rows
        scores = torch.from_numpy(s).cuda()
        want_off, want_idx, _, _ = e.topk_select(scores, wl.topk, csc=False)
        kv_off = torch.full((wl.batch, wl.heads, N + 1), -1, dtype=torch.int32, device="cuda")
        kv_idx = torch.full((wl.batch, wl.heads, N * wl.topk), -1, dtype=torch.int32, device="cuda")
        C.vsa2_topk_select_noalloc(e.p, scores, wl.topk, kv_off, kv_idx)
        torch.cuda.synchronize()
        assert torch.equal(kv_off, want_off), f"call {call}: offsets differ"
        assert torch.equal(kv_idx, want_idx), f"call {call}: indices differ"
    assert e.device_error() == 0
