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
C720 = S.WORKLOADS["720p_top64"]
C480_128 = S.WORKLOADS["480p_top128"]  # same tensors as 480p_top64 (same grid and seeds), twice the budget


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


def lists_from_masks(masks, topk):
    """Boolean tile masks [B, H, N, N] -> padded CSR (kv_off, kv_idx) and CSC (q_off, q_idx)."""
    B, H, N, _ = masks.shape
    kv_off = np.zeros((B, H, N + 1), np.int32)
    kv_idx = np.zeros((B, H, N * topk), np.int32)
    q_off = np.zeros((B, H, N + 1), np.int32)
    q_idx = np.zeros((B, H, N * topk), np.int32)
    for b in range(B):
        for h in range(H):
            m = masks[b, h]
            assert m.sum() <= N * topk
            kv_off[b, h, 1:] = np.cumsum(m.sum(1))
            r = np.nonzero(m)[1]
            kv_idx[b, h, :r.size] = r
            q_off[b, h, 1:] = np.cumsum(m.sum(0))
            c = np.nonzero(m.T)[1]
            q_idx[b, h, :c.size] = c
    return kv_off, kv_idx, q_off, q_idx


def edge_masks(pattern, wl, seed=3):
    """Selections the method can produce or that stress the kernels' edges: rows with no tile,
    every tile, one tile per row, and odd list lengths (a half block at the end of a row)."""
    N = wl.num_tiles
    rng = np.random.default_rng(seed)
    masks = np.zeros((wl.batch, wl.heads, N, N), bool)
    for b in range(wl.batch):
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
            masks[b, h] = m
    topk = max(int(np.ceil(masks[b, h].sum() / N)) for b in range(wl.batch) for h in range(wl.heads))
    return masks, topk


_sel480 = {}


def c480_lists(heads):
    """480p selection: the oracle's router + TopK on the heads in `heads`, and on every other
    head a fixed band pattern (row i takes tiles i + 7t mod N, t < topk), so that the kernels
    run at full size while the oracle only needs the sampled heads."""
    wl = C480
    key = tuple(heads)
    if key not in _sel480:
        x = inputs(wl)
        N = wl.num_tiles
        masks = np.zeros((1, wl.heads, N, N), bool)
        for h in range(wl.heads):
            if h in heads:
                sc = O.router_scores(x["q"][0, h], x["k"][0, h]).astype(np.float32)
                masks[0, h] = O.topk_select(sc, wl.topk)["mask"]
            else:
                rows = np.repeat(np.arange(N), wl.topk)
                masks[0, h, rows, (rows + 7 * np.tile(np.arange(wl.topk), N)) % N] = True
        _sel480[key] = masks
    return _sel480[key]


def c720_head0():
    """720p (the headline size): head 0 of Q, K, V from the seeded generator, its oracle router
    scores (fp64) and the oracle's TopK on them. Only head 0 is compared; the kernels still run
    all 20 heads, as the benchmark does."""
    if "720p_h0" not in _cache:
        x0 = {n: S.make_slice(C720, n, 0, 0) for n in ("q", "k", "v")}
        sc = O.router_scores(x0["q"], x0["k"])
        sel = O.topk_select(sc.astype(np.float32), C720.topk)
        _cache["720p_h0"] = (x0, sc, sel)
    return _cache["720p_h0"]


def c720_device(x0, names=("q", "k", "v")):
    """[1, 20, L, D] bf16 device tensors: head 0 = the generator's slice, heads 1-19 seeded
    normals (their outputs are not compared)."""
    g = torch.Generator(device="cuda").manual_seed(720)
    out = {}
    for n in names:
        t = torch.randn((1, C720.heads, C720.tokens, C720.head_dim), generator=g, device="cuda") * 1.1
        t[0, 0] = torch.from_numpy(x0[n]).cuda()
        out[n] = t.to(torch.bfloat16)
        del t
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


def _topk_per_row_case(wl, scores32, topk):
    e = engine(wl)
    got = e.topk_select_per_row(torch.from_numpy(scores32).cuda(), topk, csc=True)
    assert e.device_error() == 0
    for b in range(wl.batch):
        for h in range(wl.heads):
            want = O.topk_select_per_row(scores32[b, h], topk)
            for name, g in zip(("kv_off", "kv_idx", "q_off", "q_idx"), got):
                assert np.array_equal(g[b, h].cpu().numpy(), want[name]), (name, b, h)


@pytest.mark.parametrize("wl", [TINY, SMALL, C480], ids=["tiny", "small", "480p"])
def test_topk_per_row_bit_exact_on_oracle_scores(wl):
    """VSA's per-query-tile TopK on the oracle's fp32 router scores: CSR and CSC bit-exact."""
    x = inputs(wl, ("q", "k"))
    heads = None if wl is not C480 else [0, 5, 19]
    sc = oracle_scores(wl, x, heads)
    s32 = np.random.default_rng(9).random((wl.batch, wl.heads, wl.num_tiles, wl.num_tiles), dtype=np.float32)
    for (b, h), v in sc.items():
        s32[b, h] = v.astype(np.float32)
    _topk_per_row_case(wl, s32, wl.topk)


@pytest.mark.parametrize("topk", [1, 7, 45])
def test_topk_per_row_ties_and_extremes(topk):
    """Heavy ties (equal scores go to the lower KV tile), topk 1 and topk = N, N = 45 (not a
    multiple of the 256-column chunk or of 4)."""
    wl = S.Workload("odd", 1, 3, 64, (12, 12, 20), topk, "bf16")  # N = 45
    rng = np.random.default_rng(topk)
    s = (rng.integers(0, 5, (1, 3, 45, 45)) / 8.0).astype(np.float32)
    s[0, 2] = 0.5  # a head of equal scores: every row keeps its first topk columns
    _topk_per_row_case(wl, s, topk)


def test_fwd_on_per_row_selection():
    """The forward takes VSA's per-query-tile CSR unchanged."""
    wl = SMALL
    x = inputs(wl)
    e = engine(wl)
    sc = e.router_scores(dev(x["q"], "bf16"), dev(x["k"], "bf16"))
    kv_off, kv_idx, _, _ = e.topk_select_per_row(sc, wl.topk, csc=False)
    _fwd_case(wl, x, kv_off.cpu().numpy(), kv_idx.cpu().numpy())


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
    masks, topk = edge_masks(pattern, SMALL)
    wl = SMALL.with_(topk=topk)
    kv_off, kv_idx, _, _ = lists_from_masks(masks, topk)
    _fwd_case(wl, inputs(wl), kv_off, kv_idx)


def test_router_720p_head0():
    x0, want, _ = c720_head0()
    x = c720_device(x0, ("q", "k"))
    e = engine(C720)
    got = e.router_scores(x["q"], x["k"])
    assert e.device_error() == 0
    g = got[0, 0].cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(g - want) / np.linalg.norm(want)
    assert rel <= 5e-3, rel
    assert np.abs(g - want).max() <= 1e-2 * want.max()
    np.testing.assert_allclose(g.sum(1), 1.0, atol=5e-3)


def test_topk_720p_head0_bit_exact_on_oracle_scores():
    _, sc, sel = c720_head0()
    N = C720.num_tiles
    rng = np.random.default_rng(7)
    s32 = rng.random((1, C720.heads, N, N), dtype=np.float32)
    s32[0, 0] = sc.astype(np.float32)
    e = engine(C720)
    kv_off, kv_idx, q_off, q_idx = e.topk_select(torch.from_numpy(s32).cuda(), C720.topk, csc=True)
    assert e.device_error() == 0
    for name, got in zip(("kv_off", "kv_idx", "q_off", "q_idx"), (kv_off, kv_idx, q_off, q_idx)):
        assert np.array_equal(got[0, 0].cpu().numpy(), sel[name]), name


def test_fwd_720p_sampled_head0():
    """The 720p top64 forward in the benchmark's launch configuration (20 heads); head 0 runs on
    the oracle's selection and is compared on sampled query tiles (first, last, middle, ragged
    rows of the selection)."""
    x0, _, sel = c720_head0()
    x = c720_device(x0)
    N = C720.num_tiles
    masks = np.zeros((1, C720.heads, N, N), bool)
    masks[0, 0] = sel["mask"]
    rows = np.repeat(np.arange(N), C720.topk)
    for h in range(1, C720.heads):
        masks[0, h, rows, (rows + 11 * h + 7 * np.tile(np.arange(C720.topk), N)) % N] = True
    kv_off, kv_idx, _, _ = lists_from_masks(masks, C720.topk)
    e = engine(C720)
    o, lse = e.attn_fwd(x["q"], x["k"], x["v"], torch.from_numpy(kv_off).cuda(), torch.from_numpy(kv_idx).cuda())
    assert e.device_error() == 0
    lens = sel["kv_off"][1:] - sel["kv_off"][:-1]
    tiles = sorted({0, 1, N // 2, N - 1, int(np.argmin(lens)), int(np.argmax(lens))})
    wo, wlse = O.sparse_attn_fwd(x0["q"], x0["k"], x0["v"], sel["kv_off"], sel["kv_idx"], query_tiles=tiles)
    r = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in tiles])
    assert_attn_close(o[0, 0].float().cpu().numpy()[r], wo[r], "o[0,0]")
    lg = lse[0, 0].cpu().numpy()[r]
    assert np.abs(lg - wlse[r]).max() <= 2e-3 * max(1.0, np.abs(wlse[r]).max())


def test_fwd_720p_edge_rows():
    """720p-length sequences (3360 tiles) on a 2-head problem with hand-made rows: an empty
    row, rows wholly in the lower or the upper half of the tile range, a single tile, odd
    lengths, a descending (unsorted) row, two adjacent tiles, and random rows elsewhere."""
    wl = C720.with_(heads=2)
    N, L, D = wl.num_tiles, wl.tokens, wl.head_dim
    rng = np.random.default_rng(72)
    g = torch.Generator(device="cuda").manual_seed(721)
    x = {n: (torch.randn((1, 2, L, D), generator=g, device="cuda") * 1.1).to(torch.bfloat16) for n in "qkv"}
    rows = [np.sort(rng.choice(N, 64, replace=False)) for _ in range(N)]
    half = N // 2
    special = {0: np.array([], np.int64),
               1: np.sort(rng.choice(half, 40, replace=False)),
               2: np.sort(half + rng.choice(N - half, 33, replace=False)),
               3: np.array([half]),
               4: np.sort(np.concatenate([rng.choice(half, 7, replace=False), half + rng.choice(half, 8, replace=False)])),
               5: np.sort(rng.choice(N, 50, replace=False))[::-1].copy(),
               6: np.array([half - 1, half])}
    for i, r in special.items():
        rows[i] = r
    kv_off = np.zeros((1, 2, N + 1), np.int32)
    kv_idx = np.zeros((1, 2, N * wl.topk), np.int32)
    for h in range(2):
        lens = np.array([len(r) for r in rows])
        kv_off[0, h, 1:] = np.cumsum(lens)
        flat = np.concatenate(rows)
        kv_idx[0, h, :flat.size] = flat
    e = engine(wl)
    o, lse = e.attn_fwd(x["q"], x["k"], x["v"], torch.from_numpy(kv_off).cuda(), torch.from_numpy(kv_idx).cuda())
    assert e.device_error() == 0
    tiles = sorted(set(special) | {100, N // 2, N - 1})
    r = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in tiles])
    for h in range(2):
        xh = {n: x[n][0, h].float().cpu().numpy() for n in "qkv"}
        wo, wlse = O.sparse_attn_fwd(xh["q"], xh["k"], xh["v"], kv_off[0, h], kv_idx[0, h], query_tiles=tiles)
        got = o[0, h].float().cpu().numpy()[r]
        assert_attn_close(got, wo[r], f"o[0,{h}]")
        lg, lw = lse[0, h].cpu().numpy()[r], wlse[r]
        fin = np.isfinite(lw)
        assert np.array_equal(fin, np.isfinite(lg))
        assert np.abs(lg[fin] - lw[fin]).max() <= 2e-3 * max(1.0, np.abs(lw[fin]).max())
        assert np.all(got[~fin] == 0)


def test_fwd_480p_sampled_heads():
    wl = C480
    heads = [0, 19]
    kv_off, kv_idx, _, _ = lists_from_masks(c480_lists(heads), wl.topk)
    _fwd_case(wl, inputs(wl), kv_off, kv_idx, heads=heads, tiles=[0, 1, 100, 363, 364, 727])


def test_fwd_480p_full_head():
    """480p top64 in the benchmark's launch configuration (20 heads): head 0 runs on the oracle's
    selection and every one of its 728 query tiles is compared."""
    wl = C480
    kv_off, kv_idx, _, _ = lists_from_masks(c480_lists([0]), wl.topk)
    _fwd_case(wl, inputs(wl), kv_off, kv_idx, heads=[0])


def test_480p_top128_topk_bit_exact_and_forward_sampled():
    """480p with top128 (93,184 selected pairs per head): TopK on the oracle's fp32 scores of all
    20 heads is bit-exact, CSR and CSC, and the forward on that selection matches the oracle on
    sampled query tiles (first, last, middle) of two heads."""
    wl = C480_128
    x = inputs(C480)
    sc = oracle_scores(C480, x)
    s32 = np.stack([np.stack([sc[(0, h)] for h in range(wl.heads)])]).astype(np.float32)
    _topk_case(wl, s32)
    kv_off, kv_idx, _, _ = oracle_csr(wl, s32)
    _fwd_case(wl, x, kv_off, kv_idx, heads=[0, 19], tiles=[0, 1, 100, 363, 364, 727])


# ------------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------------
def _bwd_case(wl, x, lists, heads=None, q_tiles=None, kv_tiles=None):
    """Backward through the C ABI against the oracle. Both sides get the oracle's forward
    output (rounded to the storage dtype) and LSE, so the rowsum(dO * O) term is formed from
    the same O. With q_tiles / kv_tiles only the query tiles those gradients depend on are
    computed by the oracle (dQ of q_tiles, dK / dV of kv_tiles); the forward rows the compared
    gradients do not depend on are filled from the GPU forward."""
    kv_off, kv_idx, q_off, q_idx = lists
    e = engine(wl)
    q, k, v, do = (dev(x[n], wl.dtype) for n in ("q", "k", "v", "do"))
    t = lambda a: torch.from_numpy(a).cuda()
    o_gpu, lse_gpu = e.attn_fwd(q, k, v, t(kv_off), t(kv_idx))
    o_in = o_gpu.float().cpu().numpy()
    lse_in = lse_gpu.cpu().numpy()
    todo = {}
    for b in range(wl.batch):
        for h in (range(wl.heads) if heads is None else heads):
            if q_tiles is None:
                need = list(range(wl.num_tiles))
            else:
                need = set(q_tiles)
                for j in kv_tiles:
                    need.update(q_idx[b, h, q_off[b, h, j]:q_off[b, h, j + 1]].tolist())
                need = sorted(need)
            wo, wlse = O.sparse_attn_fwd(x["q"][b, h], x["k"][b, h], x["v"][b, h], kv_off[b, h], kv_idx[b, h],
                                         query_tiles=need)
            rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in need])
            o_in[b, h][rows] = S.round_to_dtype(wo[rows], wl.dtype)
            lse_in[b, h][rows] = wlse[rows]
            todo[(b, h)] = need
    dq, dk, dv = e.attn_bwd(q, k, v, dev(o_in, wl.dtype), torch.from_numpy(lse_in).cuda(), do, t(kv_off), t(kv_idx),
                            t(q_off), t(q_idx))
    assert e.device_error() == 0
    dq, dk, dv = (g.cpu().numpy() for g in (dq, dk, dv))
    for (b, h), need in todo.items():
        want = O.sparse_attn_bwd(x["q"][b, h], x["k"][b, h], x["v"][b, h], x["do"][b, h], kv_off[b, h],
                                 kv_idx[b, h], query_tiles=None if q_tiles is None else need, o=o_in[b, h])
        if q_tiles is None:
            for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
                assert_attn_close(g[b, h], w, f"{name}[{b},{h}]")
            continue
        qr = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in q_tiles])
        kr = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in kv_tiles])
        assert_attn_close(dq[b, h][qr], want[0][qr], f"dq[{b},{h}]")
        assert_attn_close(dk[b, h][kr], want[1][kr], f"dk[{b},{h}]")
        assert_attn_close(dv[b, h][kr], want[2][kr], f"dv[{b},{h}]")


@pytest.mark.parametrize("wl", [TINY, SMALL, SMALL64], ids=["tiny_fp32", "small_bf16", "small_bf16_d64"])
def test_bwd_on_oracle_selection(wl):
    x = inputs(wl, ("q", "k", "v", "do"))
    sc = oracle_scores(wl, x)
    s32 = np.stack([np.stack([sc[(b, h)] for h in range(wl.heads)]) for b in range(wl.batch)]).astype(np.float32)
    _bwd_case(wl, x, oracle_csr(wl, s32))


@pytest.mark.parametrize("pattern", ["empty_rows", "dense", "single", "odd_lengths"])
def test_bwd_edge_selections(pattern):
    masks, topk = edge_masks(pattern, SMALL)
    wl = SMALL.with_(topk=topk)
    lists = lists_from_masks(masks, topk)
    _bwd_case(wl, inputs(wl, ("q", "k", "v", "do")), lists)


def test_bwd_480p_sampled():
    wl = C480
    heads = [0, 19]
    lists = lists_from_masks(c480_lists(heads), wl.topk)
    _bwd_case(wl, inputs(wl, ("q", "k", "v", "do")), lists, heads=heads, q_tiles=[0, 363, 727],
              kv_tiles=[0, 364, 727])


def test_bwd_480p_full_head_from_own_forward():
    """The 480p top64 training step as it runs: the backward takes the forward output (bf16) and
    LSE that the GPU forward stored, and every row of dQ, dK and dV of head 0 (oracle selection)
    is compared with the oracle's exact gradient, which recomputes O in fp64 (no stored O)."""
    wl = C480
    x = inputs(wl, ("q", "k", "v", "do"))
    kv_off, kv_idx, q_off, q_idx = lists_from_masks(c480_lists([0]), wl.topk)
    e = engine(wl)
    q, k, v, do = (dev(x[n], wl.dtype) for n in ("q", "k", "v", "do"))
    t = lambda a: torch.from_numpy(a).cuda()
    o, lse = e.attn_fwd(q, k, v, t(kv_off), t(kv_idx))
    dq, dk, dv = e.attn_bwd(q, k, v, o, lse, do, t(kv_off), t(kv_idx), t(q_off), t(q_idx))
    assert e.device_error() == 0
    want = O.sparse_attn_bwd(x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["do"][0, 0], kv_off[0, 0], kv_idx[0, 0])
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        g = g[0, 0].cpu().numpy().astype(np.float64)
        rel = np.linalg.norm(g - w) / np.linalg.norm(w)
        print(f"480p head 0 {name}: max abs {np.abs(g - w).max():.3e}, rel L2 {rel:.3e}")
        assert_attn_close(g, w, f"{name}[0,0]")


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
