"""GPU parity: every step of the hot path, called through the C ABI, against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation):
  * attention outputs and gradients: max |err| <= 2e-2 and relative L2 <= 5e-3;
  * router scores: relative L2 <= 5e-3 and max |err| <= 1e-2 * max(score);
  * TopK: bit-exact CSR and CSC when both sides rank the same fp32 scores (the oracle's);
    with the GPU's own scores, the selection must be valid within the measured score error.
Attention parity uses the same index lists on both sides, so selection near ties cannot
affect it.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import trainable_block_sparse_fine_b200 as V
    from trainable_block_sparse_fine_b200 import _capi as C

SMALL = S.Workload("small_bf16", 1, 2, 128, (8, 16, 20), 6, "bf16")  # N=40, Lr=160: ragged blocks
SMALL64 = S.Workload("small_bf16_d64", 2, 1, 64, (4, 16, 24), 5, "bf16")  # N=24, batch 2
TINY = S.WORKLOADS["tiny"]
C480 = S.WORKLOADS["480p_top64"]


def dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def engine(wl, topk=None, flags=0):
    return V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk if topk is None else topk, flags=flags)


_cache = {}


def inputs(wl, names=("q", "k", "v")):
    key = (wl.name, wl.grid, wl.head_dim, wl.batch, wl.heads, wl.dtype, names)
    if key not in _cache:
        _cache[key] = {n: S.make_tensor(wl, n) for n in names}
    return _cache[key]


def assert_attn_close(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= 2e-2 and rel <= 5e-3, f"{what}: max abs {err.max():.3e}, rel L2 {rel:.3e}"


def oracle_csr(wl, scores32):
    """Per-(b,h) oracle TopK on fp32 scores -> padded [B,H,...] CSR/CSC arrays."""
    B, H, N = wl.batch, wl.heads, wl.num_tiles
    kv_off = np.zeros((B, H, N + 1), np.int32)
    kv_idx = np.zeros((B, H, N * wl.topk), np.int32)
    q_off = np.zeros((B, H, N + 1), np.int32)
    q_idx = np.zeros((B, H, N * wl.topk), np.int32)
    for b in range(B):
        for h in range(H):
            sel = O.topk_select(scores32[b, h], wl.topk)
            kv_off[b, h], kv_idx[b, h] = sel["kv_off"], sel["kv_idx"]
            q_off[b, h], q_idx[b, h] = sel["q_off"], sel["q_idx"]
    return kv_off, kv_idx, q_off, q_idx


def oracle_scores(wl, x, heads=None):
    out = {}
    for b in range(wl.batch):
        for h in (range(wl.heads) if heads is None else heads):
            out[(b, h)] = O.router_scores(x["q"][b, h], x["k"][b, h])
    return out


# ------------------------------------------------------------------------------------------
# router
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("wl,heads", [(TINY, None), (SMALL, None), (SMALL64, None), (C480, [0, 7])],
                         ids=["tiny_fp32", "small_bf16", "small_bf16_d64", "480p"])
def test_router_scores(wl, heads):
    x = inputs(wl, ("q", "k"))
    e = engine(wl)
    got = e.router_scores(dev(x["q"], wl.dtype), dev(x["k"], wl.dtype)).cpu().numpy()
    assert e.device_error() == 0
    for (b, h), want in oracle_scores(wl, x, heads).items():
        g = got[b, h].astype(np.float64)
        rel = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert rel <= 5e-3, (b, h, rel)
        assert np.abs(g - want).max() <= 1e-2 * want.max(), (b, h)
        np.testing.assert_allclose(g.sum(1), 1.0, atol=5e-3)


# ------------------------------------------------------------------------------------------
# TopK
# ------------------------------------------------------------------------------------------
def _topk_case(wl, scores32):
    e = engine(wl)
    kv_off, kv_idx, q_off, q_idx = e.topk_select(torch.from_numpy(scores32).cuda(), wl.topk, csc=True)
    assert e.device_error() == 0
    want = oracle_csr(wl, scores32)
    for name, g, w in zip(("kv_off", "kv_idx", "q_off", "q_idx"), (kv_off, kv_idx, q_off, q_idx), want):
        assert np.array_equal(g.cpu().numpy(), w), name


@pytest.mark.parametrize("wl", [TINY, SMALL, SMALL64, C480], ids=["tiny", "small", "small64", "480p"])
def test_topk_bit_exact_on_oracle_scores(wl):
    x = inputs(wl, ("q", "k"))
    sc = oracle_scores(wl, x)
    s32 = np.stack([np.stack([sc[(b, h)] for h in range(wl.heads)]) for b in range(wl.batch)]).astype(np.float32)
    _topk_case(wl, s32)


@pytest.mark.parametrize("topk", [1, 7, 40])
def test_topk_ties_and_extremes(topk):
    wl = SMALL.with_(topk=topk)
    rng = np.random.default_rng(topk)
    s = (rng.integers(0, 9, (1, 2, 40, 40)) / 16.0).astype(np.float32)  # heavy ties
    s[0, 1, 3] = 0.0  # a row that can only be reached by ties
    _topk_case(wl, s)
    _topk_case(wl, np.full((1, 2, 40, 40), 0.025, np.float32))  # all equal: first N*K flat


def test_topk_odd_tile_count():
    wl = S.Workload("odd", 1, 3, 64, (12, 12, 20), 4, "bf16")  # N = 45
    rng = np.random.default_rng(5)
    _topk_case(wl, rng.random((1, 3, 45, 45)).astype(np.float32))


def test_topk_on_gpu_scores_is_valid_within_score_error():
    wl = C480
    x = inputs(wl, ("q", "k"))
    e = engine(wl)
    g = e.router_scores(dev(x["q"], "bf16"), dev(x["k"], "bf16"))
    kv_off, kv_idx, _, _ = e.topk_select(g, wl.topk, csc=False)
    g = g.cpu().numpy()
    kv_off, kv_idx = kv_off.cpu().numpy(), kv_idx.cpu().numpy()
    for h in (0, 13):
        want = O.router_scores(x["q"][0, h], x["k"][0, h])
        tau = np.abs(g[0, h] - want).max()
        N = wl.num_tiles
        mask = np.zeros((N, N), bool)
        for i in range(N):
            mask[i, kv_idx[0, h, kv_off[0, h, i]:kv_off[0, h, i + 1]]] = True
        assert mask.sum() == N * wl.topk
        vstar = np.sort(want.ravel())[::-1][N * wl.topk - 1]
        assert want[mask].min() >= vstar - 2 * tau
        assert want[~mask].max() <= vstar + 2 * tau


# ------------------------------------------------------------------------------------------
# forward
# ------------------------------------------------------------------------------------------
def _fwd_case(wl, x, kv_off, kv_idx, heads=None, tiles=None):
    e = engine(wl)
    o, lse = e.attn_fwd(*(dev(x[n], wl.dtype) for n in "qkv"), torch.from_numpy(kv_off).cuda(),
                        torch.from_numpy(kv_idx).cuda(), wl.topk)
    assert e.device_error() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for b in range(wl.batch):
        for h in (range(wl.heads) if heads is None else heads):
            wo, wl_ = O.sparse_attn_fwd(x["q"][b, h], x["k"][b, h], x["v"][b, h], kv_off[b, h], kv_idx[b, h],
                                        query_tiles=tiles)
            rows = slice(None) if tiles is None else np.concatenate([np.arange(64 * i, 64 * i + 64) for i in tiles])
            assert_attn_close(o[b, h][rows], wo[rows], f"o[{b},{h}]")
            fin = np.isfinite(wl_[rows])
            assert np.array_equal(fin, np.isfinite(lse[b, h][rows]))
            assert np.abs(lse[b, h][rows][fin] - wl_[rows][fin]).max() <= 2e-3 * max(1.0, np.abs(wl_[rows][fin]).max())
            assert np.all(o[b, h][rows][~fin] == 0)


@pytest.mark.parametrize("wl", [TINY, SMALL, SMALL64], ids=["tiny_fp32", "small_bf16", "small_bf16_d64"])
def test_fwd_on_oracle_selection(wl):
    x = inputs(wl)
    sc = oracle_scores(wl, x)
    s32 = np.stack([np.stack([sc[(b, h)] for h in range(wl.heads)]) for b in range(wl.batch)]).astype(np.float32)
    kv_off, kv_idx, _, _ = oracle_csr(wl, s32)
    _fwd_case(wl, x, kv_off, kv_idx)


@pytest.mark.parametrize("pattern", ["empty_rows", "dense", "single", "odd_lengths"])
def test_fwd_edge_selections(pattern):
    wl = SMALL
    x = inputs(wl)
    N = wl.num_tiles
    rng = np.random.default_rng(3)
    masks = []
    for h in range(wl.heads):
        if pattern == "empty_rows":
            m = rng.random((N, N)) < wl.topk / N
            m[::3] = False
        elif pattern == "dense":
            m = np.ones((N, N), bool)
        elif pattern == "single":
            m = np.zeros((N, N), bool)
            m[np.arange(N), rng.integers(0, N, N)] = True
        else:
            m = np.zeros((N, N), bool)
            for i in range(N):
                m[i, rng.choice(N, size=2 * (i % 5) + 1, replace=False)] = True
        masks.append(m)
    topk = max(int(np.ceil(m.sum() / N)) for m in masks)
    wl = wl.with_(topk=topk)
    kv_off = np.zeros((1, wl.heads, N + 1), np.int32)
    kv_idx = np.zeros((1, wl.heads, N * topk), np.int32)
    for h, m in enumerate(masks):
        kv_off[0, h, 1:] = np.cumsum(m.sum(1))
        idx = np.nonzero(m)[1]
        kv_idx[0, h, :idx.size] = idx
    _fwd_case(wl, x, kv_off, kv_idx)


def test_fwd_480p_sampled_heads():
    wl = C480
    x = inputs(wl)
    e = engine(wl)
    q, k = dev(x["q"], "bf16"), dev(x["k"], "bf16")
    kv_off, kv_idx, _, _ = e.topk_select(e.router_scores(q, k), wl.topk, csc=False)
    _fwd_case(wl, x, kv_off.cpu().numpy(), kv_idx.cpu().numpy(), heads=[0, 19], tiles=[0, 1, 100, 363, 364, 727])


# ------------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("wl", [TINY, SMALL, SMALL64], ids=["tiny_fp32", "small_bf16", "small_bf16_d64"])
def test_bwd_on_oracle_selection(wl):
    x = inputs(wl, ("q", "k", "v", "do"))
    sc = oracle_scores(wl, x)
    s32 = np.stack([np.stack([sc[(b, h)] for h in range(wl.heads)]) for b in range(wl.batch)]).astype(np.float32)
    kv_off, kv_idx, q_off, q_idx = oracle_csr(wl, s32)
    e = engine(wl)
    q, k, v, do = (dev(x[n], wl.dtype) for n in ("q", "k", "v", "do"))
    t = lambda a: torch.from_numpy(a).cuda()
    o, lse = e.attn_fwd(q, k, v, t(kv_off), t(kv_idx))
    dq, dk, dv = e.attn_bwd(q, k, v, o, lse, do, t(kv_off), t(kv_idx), t(q_off), t(q_idx))
    assert e.device_error() == 0
    for b in range(wl.batch):
        for h in range(wl.heads):
            want = O.sparse_attn_bwd(x["q"][b, h], x["k"][b, h], x["v"][b, h], x["do"][b, h], kv_off[b, h],
                                     kv_idx[b, h])
            for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
                assert_attn_close(g[b, h].cpu().numpy(), w, f"{name}[{b},{h}]")


def test_autograd_function_matches_explicit_calls():
    wl = SMALL
    x = inputs(wl, ("q", "k", "v", "do"))
    e = engine(wl)
    q, k, v, do = (dev(x[n], "bf16") for n in ("q", "k", "v", "do"))
    qg, kg, vg = (t.clone().requires_grad_() for t in (q, k, v))
    o = V.block_sparse_attention(qg, kg, vg, e)
    o.backward(do)
    o2, lse, sel = e.forward(q, k, v, csc=True)
    dq, dk, dv = e.attn_bwd(q, k, v, o2, lse, do, *sel)
    assert torch.equal(o, o2)
    assert torch.equal(qg.grad, dq.to(torch.bfloat16))
    assert torch.equal(vg.grad, dv.to(torch.bfloat16))


# ------------------------------------------------------------------------------------------
# error paths (no fault, no hang: bounded waits and index checks)
# ------------------------------------------------------------------------------------------
def test_bounded_wait_timeout_status():
    e = engine(SMALL)
    V.vsa2_selftest_wait_timeout(e.ws, 50)
    assert e.device_error() == 4
    assert e.device_error() == 0  # reading clears the word
    x = inputs(SMALL, ("q", "k"))
    e.router_scores(dev(x["q"], "bf16"), dev(x["k"], "bf16"))
    assert e.device_error() == 0


def test_validate_mode_flags_bad_indices():
    wl = SMALL
    x = inputs(wl)
    e = engine(wl, flags=V.VSA2_FLAG_VALIDATE)
    N = wl.num_tiles
    kv_off = np.tile((np.arange(N + 1) * wl.topk).astype(np.int32), (1, wl.heads, 1))
    kv_idx = np.tile((np.arange(N * wl.topk) % N).astype(np.int32), (1, wl.heads, 1))
    kv_idx[0, 1, 17] = N + 5  # out of range
    e.attn_fwd(*(dev(x[n], "bf16") for n in "qkv"), torch.from_numpy(kv_off).cuda(), torch.from_numpy(kv_idx).cuda())
    assert e.device_error() == 5
    kv_idx[0, 1, 17] = 3
    kv_off[0, 0, 5] = -7  # broken offsets
    e.attn_fwd(*(dev(x[n], "bf16") for n in "qkv"), torch.from_numpy(kv_off).cuda(), torch.from_numpy(kv_idx).cuda())
    assert e.device_error() == 5
