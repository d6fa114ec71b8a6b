"""GPU parity for the 128-token tile with 8-token router sub-cubes (B = 128, R = 8, G = 16): the
tile and pooling sizes the deep-read blog infers for VSA2 (its section 07, "fine-grained router"),
a variant of the pages' 64 / 16 shapes. Tiles are 4x4x8 tokens, sub-cubes 2x2x2.

The router pools 8-token sub-cubes and sums 16 x 16 sub-cube pairs per tile pair (Eq. 5-7); the
per-sequence TopK ranks N x N tiles (Eq. 8-9); with bf16 and head_dim 128 the forward and the dQ
kernel run M=128 query tiles against whole 128-token KV tiles, while dK/dV and the other paths
(fp32, head_dim 64) run on the library's 64-token kernels after the selection of every
128-token tile is expanded to its two 64-token halves (the same softmax over the same keys). Everything is compared with the oracle at
tile_tokens = 128, pool_tokens = 8, with the tolerances of the 64-token tests.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import trainable_block_sparse_fine_b200 as V

TILE, POOL = (4, 4, 8), (2, 2, 2)
CASES = {
    "small_bf16": S.Workload("b128_small", 1, 2, 128, (8, 16, 32), 5, "bf16", tile=TILE, pool=POOL),      # N = 32
    "fp32_d64": S.Workload("b128_f32", 1, 2, 64, (8, 8, 32), 4, "fp32", tile=TILE, pool=POOL),            # N = 16
    "480p_like": S.Workload("b128_480", 1, 2, 128, (28, 32, 48), 32, "bf16", tile=TILE, pool=POOL),       # N = 336
}


def _dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _engine(wl):
    return V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk, tile=TILE, pool=POOL)


def _close(got, want, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= 2e-2 and rel <= 5e-3, f"{what}: max abs {err.max():.3e}, rel L2 {rel:.3e}"


@pytest.mark.parametrize("case", list(CASES))
def test_b128_router_topk_forward_backward(case):
    wl = CASES[case]
    x = {n: S.make_tensor(wl, n) for n in ("q", "k", "v", "do")}
    e = _engine(wl)
    assert e.N == wl.tokens // 128
    xd = {n: _dev(x[n], wl.dtype) for n in x}
    scores = e.router_scores(xd["q"], xd["k"]).cpu().numpy()
    heads = range(wl.heads)
    o_sc = np.zeros_like(scores)
    for h in heads:
        want = O.router_scores(x["q"][0, h], x["k"][0, h], tile_tokens=128, pool_tokens=8)
        g = scores[0, h].astype(np.float64)
        rel = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert rel <= 5e-3 and np.abs(g - want).max() <= 1e-2 * want.max(), (h, rel)
        np.testing.assert_allclose(g.sum(1), 1.0, atol=5e-3)
        o_sc[0, h] = want.astype(np.float32)
    kv_off, kv_idx, q_off, q_idx = e.topk_select(torch.from_numpy(o_sc).cuda(), wl.topk, csc=True)
    o, lse = e.attn_fwd(xd["q"], xd["k"], xd["v"], kv_off, kv_idx)
    dq, dk, dv = e.attn_bwd(xd["q"], xd["k"], xd["v"], o, lse, xd["do"], kv_off, kv_idx, q_off, q_idx)
    assert e.device_error() == 0
    o = o.float().cpu().numpy()
    for h in heads:
        sel = O.topk_select(o_sc[0, h], wl.topk)
        for name, got in zip(("kv_off", "kv_idx", "q_off", "q_idx"), (kv_off, kv_idx, q_off, q_idx)):
            assert np.array_equal(got[0, h].cpu().numpy(), sel[name]), name
        wo, wlse = O.sparse_attn_fwd(x["q"][0, h], x["k"][0, h], x["v"][0, h], sel["kv_off"], sel["kv_idx"],
                                     tile_tokens=128)
        _close(o[0, h], wo, f"o h{h}")
        grads = O.sparse_attn_bwd(x["q"][0, h], x["k"][0, h], x["v"][0, h], x["do"][0, h], sel["kv_off"],
                                  sel["kv_idx"], tile_tokens=128)
        for n, got, w in zip(("dq", "dk", "dv"), (dq, dk, dv), grads):
            _close(got[0, h].cpu().numpy(), w, f"{n} h{h}")


def _lists(masks):
    """Boolean tile masks [H, N, N] -> CSR (kv_off, kv_idx) with room for the largest row budget."""
    H, N, _ = masks.shape
    topk = max(1, max(int(np.ceil(m.sum() / N)) for m in masks))
    kv_off = np.zeros((1, H, N + 1), np.int32)
    kv_idx = np.zeros((1, H, N * topk), np.int32)
    for h in range(H):
        kv_off[0, h, 1:] = np.cumsum(masks[h].sum(1))
        r = np.nonzero(masks[h])[1]
        kv_idx[0, h, :r.size] = r
    return kv_off, kv_idx, topk


def _edge_masks(pattern, H, N, rng):
    masks = np.zeros((H, N, N), bool)
    for h in range(H):
        m = masks[h]
        if pattern == "empty_rows":
            m[:] = rng.random((N, N)) < 6 / N
            m[::3] = False
        elif pattern == "single":
            m[np.arange(N), rng.integers(0, N, N)] = True
        elif pattern == "odd":
            for i in range(N):
                m[i, rng.choice(N, size=min(N, 2 * (i % 5) + 1), replace=False)] = True
        elif pattern == "dense":
            m[:] = True
        else:  # "long": a few rows take every tile (more indices than the kernel keeps on chip)
            m[:] = rng.random((N, N)) < 4 / N
            m[rng.choice(N, size=6, replace=False)] = True
    return masks


@pytest.mark.parametrize("case,pattern", [("small_bf16", p) for p in ("empty_rows", "single", "odd", "dense")]
                         + [("480p_like", "long")])
def test_b128_fwd_edge_selections(case, pattern):
    """The forward on 128-token tiles (M=128 query tiles against whole 128-token KV tiles) on
    selections at its edges: rows with no tile (o = 0, lse = -inf), one tile (a single S and O
    op), odd lengths, every tile, and rows of all 336 tiles (past the indices kept in shared
    memory); O and LSE against the oracle."""
    wl = CASES[case]
    rng = np.random.default_rng(11)
    x = {n: S.make_tensor(wl, n) for n in ("q", "k", "v")}
    xd = {n: _dev(x[n], wl.dtype) for n in x}
    masks = _edge_masks(pattern, wl.heads, wl.tokens // 128, rng)
    kv_off, kv_idx, topk = _lists(masks)
    e = V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, topk, tile=TILE, pool=POOL)
    o, lse = e.attn_fwd(xd["q"], xd["k"], xd["v"], torch.from_numpy(kv_off).cuda(), torch.from_numpy(kv_idx).cuda(),
                        topk)
    assert e.device_error() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(wl.heads):
        wo, wlse = O.sparse_attn_fwd(x["q"][0, h], x["k"][0, h], x["v"][0, h], kv_off[0, h], kv_idx[0, h],
                                     tile_tokens=128)
        _close(o[0, h], wo, f"{pattern} o h{h}")
        fin = np.isfinite(wlse)
        assert np.array_equal(np.isfinite(lse[0, h]), fin), f"{pattern} lse -inf rows h{h}"
        assert np.abs(lse[0, h][fin] - wlse[fin]).max() <= 2e-3 * max(1.0, np.abs(wlse[fin]).max()), pattern


def test_b128_refuses_what_it_does_not_take():
    """Padded grids and the coarse branch are built for 64-token tiles only."""
    with pytest.raises(V.Vsa2Error):
        V.VSA2(1, 1, 128, (8, 16, 30), "bf16", 4, tile=TILE, pool=POOL)
    wl = CASES["small_bf16"]
    e = _engine(wl)
    z = torch.zeros(1, wl.heads, wl.tokens, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(V.Vsa2Error) as ex:
        e.coarse_attn(z, z, z)
    assert ex.value.status == 2
