"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a brute-force restatement of
the definition on the raster token grid, a closed form, a special case that reduces to a library
routine, an invariant, or a value printed on the pages (tests/golden/).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TILE, POOL = (4, 4, 4), (2, 2, 4)


def _raster_inputs(grid, d, seed, smooth=True):
    rng = np.random.default_rng(seed)
    if smooth:
        return S.smoothed_field(rng, grid, d).astype(np.float64)
    return rng.standard_normal((*grid, d))


# --------------------------------------------------------------------------------------------
# synthetic inputs (layout contract shared by both sides)
# --------------------------------------------------------------------------------------------

def test_cube_major_roundtrip_and_tile_membership():
    grid = (8, 8, 12)
    x = np.arange(np.prod(grid) * 2, dtype=np.float64).reshape(*grid, 2)
    y = S.raster_to_cube_major(x, TILE, POOL)
    assert np.array_equal(S.cube_major_to_raster(y, grid, TILE, POOL), x)
    # every cube-major tile i holds exactly the tokens of one 4x4x4 cube, tiles in raster order
    nt, nh, nw = grid[0] // 4, grid[1] // 4, grid[2] // 4
    for i in range(nt * nh * nw):
        a, b, c = i // (nh * nw), (i // nw) % nh, i % nw
        cube = x[4 * a:4 * a + 4, 4 * b:4 * b + 4, 4 * c:4 * c + 4, 0].ravel()
        assert set(y[64 * i:64 * i + 64, 0]) == set(cube)
        # ... and each 16-row group is one 2x2x4 sub-cube
        for g in range(4):
            st, sh = g // 2, g % 2
            sub = x[4 * a + 2 * st:4 * a + 2 * st + 2, 4 * b + 2 * sh:4 * b + 2 * sh + 2, 4 * c:4 * c + 4, 0]
            assert set(y[64 * i + 16 * g:64 * i + 16 * g + 16, 0]) == set(sub.ravel())


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000)).astype(np.float32)
    ours = S.round_to_dtype(x, "bf16")
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, ref)


def test_field_statistics():
    wl = S.WORKLOADS["tiny"]
    x = S.make_slice(wl, "q", 0, 0)
    assert x.shape == (wl.tokens, wl.head_dim)
    assert abs(x.var() - 1.25) < 0.1
    # smooth: neighbouring tokens along w (adjacent rows inside a sub-cube) correlate strongly
    xr = S.cube_major_to_raster(x, wl.grid, wl.tile, wl.pool)
    c = np.corrcoef(xr[:, :, :-1].ravel(), xr[:, :, 1:].ravel())[0, 1]
    assert c > 0.5


# --------------------------------------------------------------------------------------------
# router, Eq. 5-7
# --------------------------------------------------------------------------------------------

def _router_bruteforce(xq, xk, grid):
    """Eq. 5-7 restated on the raster grid with explicit loops: pooled means over each
    2x2x4 sub-cube, softmax over all pooled keys, then sum over key sub-cubes and mean over
    query sub-cubes of each 4x4x4 tile."""
    T, H, W, D = xq.shape
    subs = []  # (tile index, pooled q, pooled k)
    nt, nh, nw = T // 4, H // 4, W // 4
    for a, b, c in itertools.product(range(nt), range(nh), range(nw)):
        tile = (a * nh + b) * nw + c
        for st, sh in itertools.product(range(2), range(2)):
            t0, h0, w0 = 4 * a + 2 * st, 4 * b + 2 * sh, 4 * c
            qs = np.zeros(D)
            ks = np.zeros(D)
            for dt, dh, dw in itertools.product(range(2), range(2), range(4)):
                qs += xq[t0 + dt, h0 + dh, w0 + dw]
                ks += xk[t0 + dt, h0 + dh, w0 + dw]
            subs.append((tile, qs / 16.0, ks / 16.0))
    N = nt * nh * nw
    out = np.zeros((N, N))
    for ti, qa, _ in subs:
        logits = [float(qa @ kb) / math.sqrt(D) for _, _, kb in subs]
        m = max(logits)
        ex = [math.exp(z - m) for z in logits]
        z = sum(ex)
        for (tj, _, _), e in zip(subs, ex):
            out[ti, tj] += e / z / 4.0
    return out


@pytest.mark.parametrize("grid,d", [((4, 8, 8), 8), ((8, 8, 8), 16)])
def test_router_matches_bruteforce_on_raster_grid(grid, d):
    xq = _raster_inputs(grid, d, 1)
    xk = _raster_inputs(grid, d, 2)
    want = _router_bruteforce(xq, xk, grid)
    got = O.router_scores(S.raster_to_cube_major(xq, TILE, POOL), S.raster_to_cube_major(xk, TILE, POOL))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)


def test_router_tile_constant_case_equals_coarse_attention():
    """If Q and K are constant inside every 4x4x4 tile, the router scores equal the coarse
    branch's block attention P_c = softmax(Qc Kc^T / sqrt(D)) of Eq. 1-2."""
    N, D = 12, 32
    rng = np.random.default_rng(5)
    qc = rng.standard_normal((N, D)) * 2
    kc = rng.standard_normal((N, D)) * 2
    q = np.repeat(qc, 64, axis=0)
    k = np.repeat(kc, 64, axis=0)
    pc = torch.softmax(torch.from_numpy(qc) @ torch.from_numpy(kc).T / math.sqrt(D), dim=-1).numpy()
    np.testing.assert_allclose(O.router_scores(q, k), pc, rtol=1e-12, atol=1e-15)


def test_router_rows_sum_to_one_and_are_probabilities():
    wl = S.WORKLOADS["tiny"]
    q = S.make_slice(wl, "q", 0, 1)
    k = S.make_slice(wl, "k", 0, 1)
    p = O.router_scores(q, k, row_chunk=64)  # several row blocks
    assert p.shape == (wl.num_tiles, wl.num_tiles)
    assert np.all(p >= 0) and np.all(p <= 1)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(p, O.router_scores(q, k, row_chunk=1 << 20), rtol=1e-13, atol=0)


def test_router_with_unit_pool_is_the_dense_oracle_router():
    """With R = 1 the pool-softmax-pool router is the token-level router of Eq. 10-11."""
    rng = np.random.default_rng(9)
    q = rng.standard_normal((256, 16))
    k = rng.standard_normal((256, 16))
    np.testing.assert_allclose(O.router_scores(q, k, 64, 1), O.router_scores_dense_attention(q, k, 64),
                               rtol=1e-12, atol=1e-16)


def test_router_uniform_keys_give_uniform_scores():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((512, 16))
    k = np.ones((512, 16))
    np.testing.assert_allclose(O.router_scores(q, k), 1.0 / 8, rtol=1e-13)


# --------------------------------------------------------------------------------------------
# per-sequence TopK, Eq. 8-9
# --------------------------------------------------------------------------------------------

def _check_topk_structure(sel, scores, topk):
    N = scores.shape[0]
    kv_off, kv_idx, q_off, q_idx, mask = sel["kv_off"], sel["kv_idx"], sel["q_off"], sel["q_idx"], sel["mask"]
    assert kv_off[0] == 0 and kv_off[-1] == N * topk == mask.sum()
    assert np.all(np.diff(kv_off) >= 0)
    assert kv_idx.min() >= 0 and kv_idx.max() < N
    for i in range(N):
        row = kv_idx[kv_off[i]:kv_off[i + 1]]
        assert np.all(np.diff(row) > 0)
        assert set(row) == set(np.nonzero(mask[i])[0])
    for j in range(N):
        col = q_idx[q_off[j]:q_off[j + 1]]
        assert np.all(np.diff(col) > 0)
        assert set(col) == set(np.nonzero(mask[:, j])[0])


def test_topk_bruteforce_sort_with_ties():
    rng = np.random.default_rng(11)
    N, K = 9, 3
    s = rng.integers(0, 6, (N, N)).astype(np.float32) / 8  # many exact ties
    sel = O.topk_select(s, K)
    ranked = sorted(((-float(s[i, j]), i * N + j) for i in range(N) for j in range(N)))
    want = np.zeros(N * N, bool)
    for _, f in ranked[:N * K]:
        want[f] = True
    assert np.array_equal(sel["mask"].ravel(), want)
    _check_topk_structure(sel, s, K)


def test_topk_invariants_on_router_scores():
    wl = S.WORKLOADS["tiny"]
    q, k = S.make_slice(wl, "q", 0, 0), S.make_slice(wl, "k", 0, 0)
    s = O.router_scores(q, k).astype(np.float32)
    sel = O.topk_select(s, wl.topk)
    _check_topk_structure(sel, s, wl.topk)
    m = sel["mask"]
    assert s[m].min() >= s[~m].max()
    thr = s[m].min()
    tied_in = np.flatnonzero(m.ravel() & (s.ravel() == thr))
    tied_out = np.flatnonzero(~m.ravel() & (s.ravel() == thr))
    if tied_out.size:
        assert tied_in.max() < tied_out.min()


def test_topk_full_budget_selects_everything():
    rng = np.random.default_rng(1)
    s = rng.random((7, 7)).astype(np.float32)
    sel = O.topk_select(s, 7)
    assert sel["mask"].all()


def test_topk_golden_uniform_scores():
    """All scores equal: the tie rule keeps the N*K lowest flat indices, i.e. rows 0..K-1."""
    path = os.path.join(GOLDEN, "topk_uniform_n8_k3.txt")
    lines = [l for l in open(path) if not l.startswith("#") and l.strip()]
    spec = dict(l.split("=", 1) for l in lines)
    N, K = int(spec["N"]), int(spec["K"])
    sel = O.topk_select(np.full((N, N), 1.0 / N, np.float32), K)
    assert list(sel["kv_off"]) == [int(v) for v in spec["kv_off"].split()]
    assert list(sel["kv_idx"]) == [int(v) for v in spec["kv_idx"].split()]
    assert list(sel["q_off"]) == [int(v) for v in spec["q_off"].split()]
    assert list(sel["q_idx"]) == [int(v) for v in spec["q_idx"].split()]


def test_sparsity_estimate_matches_printed_values():
    """App. B Eq. 15-16 with the budget the TopK actually spends, against the sparsities the
    deep-read blog derives for Table 2 (B=128, R=8)."""
    path = os.path.join(GOLDEN, "table2_sparsity.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    rng = np.random.default_rng(0)
    for L, B, R, K, printed in rows:
        L, B, R, K, printed = int(L), int(B), int(R), int(K), float(printed)
        N = L // B
        sel = O.topk_select(rng.random((N, N)).astype(np.float32), K)
        pairs = int(sel["kv_off"][-1])
        sparsity = 1.0 - (1.0 / R ** 2 + pairs * B * B / float(N * B) ** 2)
        assert abs(sparsity - printed) <= 0.0006, (L, K, sparsity, printed)


# --------------------------------------------------------------------------------------------
# block-sparse attention forward, Eq. 12
# --------------------------------------------------------------------------------------------

def _masked_attention_bruteforce(q, k, v, mask, bt=64):
    """softmax(Q K^T / sqrt(D) + M) V with M = -inf outside the selected tile pairs (§2.1),
    expanded to tokens; a row with no selected tile gives 0 and lse = -inf."""
    L, D = q.shape
    tok = np.repeat(np.repeat(mask, bt, axis=0), bt, axis=1)
    s = q @ k.T / math.sqrt(D)
    s = np.where(tok, s, -np.inf)
    o = np.zeros_like(q)
    lse = np.full(L, -np.inf)
    for t in range(L):
        if not tok[t].any():
            continue
        m = s[t][tok[t]].max()
        e = np.where(tok[t], np.exp(s[t] - m), 0.0)
        o[t] = e @ v / e.sum()
        lse[t] = m + math.log(e.sum())
    return o, lse


def _csr(mask):
    N = mask.shape[0]
    off = np.zeros(N + 1, np.int32)
    off[1:] = np.cumsum(mask.sum(1))
    return off, np.nonzero(mask)[1].astype(np.int32)


def test_fwd_matches_bruteforce_masked_attention():
    rng = np.random.default_rng(4)
    L, D = 6 * 64, 16
    q, k, v = (rng.standard_normal((L, D)) * 1.5 for _ in range(3))
    mask = rng.random((6, 6)) < 0.4
    mask[2] = False  # a query tile with no KV tile
    off, idx = _csr(mask)
    o, lse = O.sparse_attn_fwd(q, k, v, off, idx)
    o2, lse2 = _masked_attention_bruteforce(q, k, v, mask)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, rtol=1e-12, atol=1e-13)
    assert np.all(o[128:192] == 0) and np.all(np.isneginf(lse[128:192]))


def test_fwd_full_budget_equals_dense_attention():
    rng = np.random.default_rng(6)
    L, D = 4 * 64, 32
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    sel = O.topk_select(rng.random((4, 4)).astype(np.float32), 4)
    o, lse = O.sparse_attn_fwd(q, k, v, sel["kv_off"], sel["kv_idx"])
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()
    ref_lse = torch.logsumexp(torch.from_numpy(q @ k.T) / math.sqrt(D), dim=-1).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_fwd_constant_keys_closed_form():
    """Equal keys give equal weights: o_t is the mean of the selected value rows and
    lse_t = q_t.k/sqrt(D) + log(#selected tokens)."""
    rng = np.random.default_rng(8)
    L, D = 5 * 64, 8
    q, v = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    kvec = rng.standard_normal(D)
    k = np.tile(kvec, (L, 1))
    mask = rng.random((5, 5)) < 0.5
    mask[:, 0] = True
    off, idx = _csr(mask)
    o, lse = O.sparse_attn_fwd(q, k, v, off, idx)
    vt = v.reshape(5, 64, D)
    for i in range(5):
        sel = np.nonzero(mask[i])[0]
        np.testing.assert_allclose(o[64 * i:64 * i + 64], np.broadcast_to(vt[sel].reshape(-1, D).mean(0), (64, D)),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[64 * i:64 * i + 64], q[64 * i:64 * i + 64] @ kvec / math.sqrt(D) + math.log(64 * sel.size),
                                   rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------------------------

def _loss(q, k, v, do, off, idx):
    o, _ = O.sparse_attn_fwd(q, k, v, off, idx)
    return float(np.sum(o * do))


def test_bwd_central_finite_differences():
    rng = np.random.default_rng(12)
    L, D = 3 * 64, 8
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    mask = np.array([[1, 0, 1], [0, 0, 0], [1, 1, 0]], bool)
    off, idx = _csr(mask)
    dq, dk, dv = O.sparse_attn_bwd(q, k, v, do, off, idx)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        dirn = rng.standard_normal(x.shape)
        args = {"q": q, "k": k, "v": v}
        plus = dict(args, **{name: x + eps * dirn})
        minus = dict(args, **{name: x - eps * dirn})
        fd = (_loss(plus["q"], plus["k"], plus["v"], do, off, idx) - _loss(minus["q"], minus["k"], minus["v"], do, off, idx)) / (2 * eps)
        an = float(np.sum(g * dirn))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
    assert np.all(dq[64:128] == 0)


def test_bwd_full_budget_equals_dense_autograd():
    rng = np.random.default_rng(13)
    L, D = 3 * 64, 16
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    off, idx = _csr(np.ones((3, 3), bool))
    dq, dk, dv = O.sparse_attn_bwd(q, k, v, do, off, idx)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None])[0, 0]
    o.backward(torch.from_numpy(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_bwd_invariants():
    """Each softmax row's dS sums to zero, so the key gradients sum to zero; the probabilities
    of a non-empty row sum to one, so the value gradients sum to the sum of dO over
    non-empty query rows."""
    rng = np.random.default_rng(14)
    L, D = 5 * 64, 16
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    mask = rng.random((5, 5)) < 0.5
    mask[3] = False
    off, idx = _csr(mask)
    dq, dk, dv = O.sparse_attn_bwd(q, k, v, do, off, idx)
    np.testing.assert_allclose(dk.sum(0), 0, atol=1e-11)
    live = np.repeat(mask.any(1), 64)
    np.testing.assert_allclose(dv.sum(0), do[live].sum(0), rtol=1e-12, atol=1e-11)


def test_bwd_query_tile_subset_is_exact_where_complete():
    """Restricting the backward to a subset of query tiles leaves dQ on those tiles, and dK, dV
    on every KV tile selected only by tiles of the subset, equal to the full computation."""
    rng = np.random.default_rng(15)
    L, D = 6 * 64, 16
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    mask = rng.random((6, 6)) < 0.45
    mask[:, 4] = False
    mask[[0, 5], 4] = True  # KV tile 4 is selected by query tiles 0 and 5 only
    off, idx = _csr(mask)
    full = O.sparse_attn_bwd(q, k, v, do, off, idx)
    sub = O.sparse_attn_bwd(q, k, v, do, off, idx, query_tiles=[0, 5])
    for i in (0, 5):
        np.testing.assert_array_equal(sub[0][64 * i:64 * i + 64], full[0][64 * i:64 * i + 64])
    for g_sub, g_full in zip(sub[1:], full[1:]):
        np.testing.assert_allclose(g_sub[256:320], g_full[256:320], rtol=1e-12, atol=1e-13)
    assert np.all(sub[0][64:256] == 0)


def test_bwd_given_output_enters_only_through_rowsum():
    """Passing the exact forward output reproduces the default; the output only enters through
    rowsum(dO * O): a change orthogonal to each dO row changes nothing, and dV never depends
    on it. A change along dO shifts dQ by the closed form -P (dO . u) K / sqrt(D) per row."""
    rng = np.random.default_rng(16)
    L, D = 4 * 64, 16
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    mask = rng.random((4, 4)) < 0.6
    mask[:, 1] = True
    off, idx = _csr(mask)
    o, _ = O.sparse_attn_fwd(q, k, v, off, idx)
    base = O.sparse_attn_bwd(q, k, v, do, off, idx)
    same = O.sparse_attn_bwd(q, k, v, do, off, idx, o=o)
    for a, b in zip(base, same):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    u = rng.standard_normal((L, D))
    u -= (np.sum(u * do, 1) / np.sum(do * do, 1))[:, None] * do  # orthogonal to dO, row by row
    orth = O.sparse_attn_bwd(q, k, v, do, off, idx, o=o + 3.0 * u)
    for a, b in zip(base, orth):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)
    shift = O.sparse_attn_bwd(q, k, v, do, off, idx, o=o + 0.5 * do)
    np.testing.assert_array_equal(shift[2], base[2])
    # row t of tile i: Delta grows by 0.5 |dO_t|^2, so dS_t drops by 0.5 |dO_t|^2 P_t
    i = 0
    sel = idx[off[i]:off[i + 1]]
    ks = k.reshape(4, 64, D)[sel].reshape(-1, D)
    s = q[:64] @ ks.T / math.sqrt(D)
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    want = base[0][:64] - (0.5 * np.sum(do[:64] ** 2, 1))[:, None] * (p @ ks) / math.sqrt(D)
    np.testing.assert_allclose(shift[0][:64], want, rtol=1e-10, atol=1e-11)


# --------------------------------------------------------------------------------------------
# coarse branch, Eq. 1-4, and gated merge, Eq. 13-14
# --------------------------------------------------------------------------------------------

def _coarse_bruteforce(xq, xk, xv):
    """Eq. 1-3 restated on the raster grid with explicit loops: the mean of every 4x4x4 cube of
    Q, K and V (cubes in raster order), then softmax attention from each cube to all cubes."""
    T, H, W, D = xq.shape
    nt, nh, nw = T // 4, H // 4, W // 4
    means = {n: [] for n in "qkv"}
    for a, b, c in itertools.product(range(nt), range(nh), range(nw)):
        for n, x in zip("qkv", (xq, xk, xv)):
            acc = np.zeros(D)
            for dt, dh, dw in itertools.product(range(4), repeat=3):
                acc += x[4 * a + dt, 4 * b + dh, 4 * c + dw]
            means[n].append(acc / 64.0)
    N = len(means["q"])
    out, lse = np.zeros((N, D)), np.zeros(N)
    for i in range(N):
        logits = [float(means["q"][i] @ kj) / math.sqrt(D) for kj in means["k"]]
        m = max(logits)
        ex = [math.exp(z - m) for z in logits]
        z = sum(ex)
        out[i] = sum(e * vj for e, vj in zip(ex, means["v"])) / z
        lse[i] = m + math.log(z)
    return out, lse


@pytest.mark.parametrize("grid,d", [((4, 8, 8), 8), ((8, 8, 12), 16)])
def test_coarse_matches_bruteforce_on_raster_grid(grid, d):
    xq, xk, xv = (_raster_inputs(grid, d, s) for s in (11, 12, 13))
    want_o, want_lse = _coarse_bruteforce(xq, xk, xv)
    o, lse = O.coarse_attn(*(S.raster_to_cube_major(x, TILE, POOL) for x in (xq, xk, xv)))
    np.testing.assert_allclose(o, want_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, want_lse, rtol=1e-12, atol=1e-14)


def test_coarse_tile_constant_inputs_equal_dense_attention():
    """With Q, K, V constant inside every tile, each token of tile i sees 64 copies of the key
    and value of every tile j, so dense token-level attention (a library routine) equals
    Repeat_B of the coarse output, and its log-sum-exp is the coarse one plus log 64."""
    N, D = 7, 16
    rng = np.random.default_rng(21)
    qc, kc, vc = (rng.standard_normal((N, D)) * 1.5 for _ in range(3))
    q, k, v = (np.repeat(x, 64, axis=0) for x in (qc, kc, vc))
    o_c, lse_c = O.coarse_attn(q, k, v)
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()
    ref_lse = torch.logsumexp(torch.from_numpy(q @ k.T) / math.sqrt(D), dim=-1).numpy()
    np.testing.assert_allclose(np.repeat(o_c, 64, axis=0), ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(np.repeat(lse_c, 64) + math.log(64), ref_lse, rtol=1e-12, atol=1e-12)


def test_coarse_single_tile_and_equal_keys_closed_forms():
    rng = np.random.default_rng(22)
    D = 8
    # one tile: a softmax over one key is 1, so the output is the tile's mean value row
    q, k, v = (rng.standard_normal((64, D)) for _ in range(3))
    o, lse = O.coarse_attn(q, k, v)
    np.testing.assert_allclose(o[0], v.mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse[0], q.mean(axis=0) @ k.mean(axis=0) / math.sqrt(D), rtol=1e-13)
    # equal keys everywhere: uniform weights over the 5 tiles, so every row is the mean of V
    # and lse = qc . k / sqrt(D) + log 5
    q5, v5 = rng.standard_normal((5 * 64, D)), rng.standard_normal((5 * 64, D))
    kvec = rng.standard_normal(D)
    o, lse = O.coarse_attn(q5, np.tile(kvec, (5 * 64, 1)), v5)
    np.testing.assert_allclose(o, np.tile(v5.mean(axis=0), (5, 1)), rtol=1e-12, atol=1e-14)
    qc = q5.reshape(5, 64, D).mean(axis=1)
    np.testing.assert_allclose(lse, qc @ kvec / math.sqrt(D) + math.log(5), rtol=1e-12, atol=1e-14)


def test_gated_merge_closed_forms():
    rng = np.random.default_rng(23)
    L, D = 3 * 64, 4
    o_f = rng.standard_normal((L, D))
    o_c_hat = rng.standard_normal((3, D))
    # G = tanh(0) = 0: the fine branch alone. §2.3 (Sparse Rebasing) relies on this: W_g starts
    # at zero, so a model switched to VSA2 outputs only O_f at first.
    np.testing.assert_array_equal(O.gated_merge(o_f, o_c_hat, np.zeros(L)), o_f)
    # saturated gates: tanh(+-40) rounds to +-1 in fp64
    sign = np.where(np.arange(L) % 2 == 0, 1.0, -1.0)
    want = o_f + sign[:, None] * np.repeat(o_c_hat, 64, axis=0)
    np.testing.assert_allclose(O.gated_merge(o_f, o_c_hat, 40.0 * sign), want, rtol=0, atol=1e-15)
    # G = 1/2 at the logit atanh(1/2) = ln(3)/2; token 130 lies in tile 2
    out = O.gated_merge(o_f, o_c_hat, np.full(L, math.log(3) / 2))
    np.testing.assert_allclose(out[130], o_f[130] + 0.5 * o_c_hat[2], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(out[63], o_f[63] + 0.5 * o_c_hat[0], rtol=1e-14, atol=1e-15)


def _central_diff(f, x, h=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + h
        up = f()
        x[idx] = old - h
        dn = f()
        x[idx] = old
        g[idx] = (up - dn) / (2 * h)
    return g


def test_coarse_bwd_central_finite_differences():
    rng = np.random.default_rng(24)
    L, D = 3 * 64, 4
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    w = rng.standard_normal((3, D))  # loss = sum(w * O_c_hat), so dLoss/dO_c_hat = w
    dq, dk, dv = O.coarse_attn_bwd(q, k, v, w)
    for x, got in ((q, dq), (k, dk), (v, dv)):
        num = _central_diff(lambda: float((w * O.coarse_attn(q, k, v)[0]).sum()), x)
        np.testing.assert_allclose(got, num, rtol=1e-6, atol=1e-9)


def test_coarse_bwd_tile_constant_case_equals_dense_autograd():
    """With Q, K, V and dO constant inside every tile, dense token attention and the coarse
    branch give the same output, and by symmetry the same gradient at every token: each token's
    dense-attention gradient is the pooled gradient divided by 64 (torch autograd, fp64)."""
    N, D = 5, 8
    rng = np.random.default_rng(25)
    qc, kc, vc, gc = (rng.standard_normal((N, D)) for _ in range(4))
    q, k, v, g = (np.repeat(x, 64, axis=0) for x in (qc, kc, vc, gc))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None])[0, 0]
    (out * torch.from_numpy(g)).sum().backward()
    # dLoss/dO_c_hat for the coarse branch: the 64 tokens of a tile share one output row
    dq, dk, dv = O.coarse_attn_bwd(q, k, v, 64.0 * gc)
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_gated_merge_bwd_finite_differences_and_zero_gate():
    rng = np.random.default_rng(26)
    L, D = 2 * 64, 3
    o_f = rng.standard_normal((L, D))
    oc = rng.standard_normal((2, D))
    logits = rng.standard_normal(L)
    dout = rng.standard_normal((L, D))
    d_of, d_oc, d_logits = O.gated_merge_bwd(dout, oc, logits)
    loss = lambda: float((dout * O.gated_merge(o_f, oc, logits)).sum())
    np.testing.assert_array_equal(d_of, dout)
    np.testing.assert_allclose(d_oc, _central_diff(loss, oc), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(d_logits, _central_diff(loss, logits), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(_central_diff(loss, o_f), dout, rtol=1e-7, atol=1e-9)
    # closed forms at G = 0: no gradient reaches O_c_hat, and the logit gradient is dout . O_c
    _, d_oc0, d_l0 = O.gated_merge_bwd(dout, oc, np.zeros(L))
    assert np.all(d_oc0 == 0)
    np.testing.assert_allclose(d_l0, (dout * np.repeat(oc, 64, axis=0)).sum(axis=1), rtol=1e-15)


def test_coarse_bwd_given_output_enters_only_through_rowsum():
    """Passing the exact forward output reproduces the default; a perturbed output changes
    the gradients only through Delta = rowsum(d_oc * O): dV does not move."""
    rng = np.random.default_rng(27)
    L, D = 3 * 64, 4
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    w = rng.standard_normal((3, D))
    o, _ = O.coarse_attn(q, k, v)
    base = O.coarse_attn_bwd(q, k, v, w)
    same = O.coarse_attn_bwd(q, k, v, w, o_c_hat=o)
    for a, b in zip(base, same):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)
    moved = O.coarse_attn_bwd(q, k, v, w, o_c_hat=o + 0.01)
    np.testing.assert_array_equal(moved[2], base[2])
    assert np.abs(moved[0] - base[0]).max() > 1e-6


# --------------------------------------------------------------------------------------------
# token permutation, §2.2 "Permutation"
# --------------------------------------------------------------------------------------------

@pytest.mark.parametrize("grid,tile,pool", [((8, 16, 20), (4, 4, 4), (2, 2, 4)), ((4, 8, 16), (2, 4, 8), (1, 2, 8)),
                                            ((12, 12, 8), (4, 4, 4), (2, 2, 4))])
def test_permutation_matches_reshape_transpose_and_round_trips(grid, tile, pool):
    """Against the input generator's reshape/transpose formulation (a different construction of
    the same order), and the inverse restores the raster tensor exactly."""
    x = np.random.default_rng(28).standard_normal((*grid, 3))
    y = O.permute_to_cube_major(x, tile, pool)
    np.testing.assert_array_equal(y, S.raster_to_cube_major(x, tile, pool))
    np.testing.assert_array_equal(O.permute_to_raster(y, grid, tile, pool), x)


def test_permutation_tile_and_subcube_membership():
    """Row block i of 64 holds exactly the tokens of the i-th 4x4x4 cube in raster order of the
    cube grid, and each block of 16 inside it one 2x2x4 sub-cube."""
    grid = (8, 8, 8)
    T, H, W = grid
    idx = np.arange(T * H * W, dtype=np.float64).reshape(T, H, W, 1)  # value = raster index
    y = O.permute_to_cube_major(idx)[:, 0].astype(int)
    t, h, w = np.unravel_index(y, grid)
    tiles = (t // 4) * (H // 4) * (W // 4) + (h // 4) * (W // 4) + (w // 4)
    np.testing.assert_array_equal(tiles, np.repeat(np.arange(T * H * W // 64), 64))
    sub = ((t % 4) // 2) * 2 + (h % 4) // 2
    np.testing.assert_array_equal(sub, np.tile(np.repeat(np.arange(4), 16), T * H * W // 64))


# --------------------------------------------------------------------------------------------
# grids the tile does not divide: padding and masks (§2.2 "Kernel Implementation")
# --------------------------------------------------------------------------------------------

def _padded_cube_major(x, tile=TILE, pool=POOL):
    xp, valid = O.pad_to_tiles(x, tile)
    vm = O.permute_to_cube_major(valid[..., None].astype(np.float64), tile, pool)[:, 0] > 0
    return O.permute_to_cube_major(xp, tile, pool), vm, xp.shape[:3]


def test_padded_functions_equal_the_unpadded_ones_on_divisible_grids():
    grid, d, topk = (8, 8, 12), 8, 3
    xq, xk, xv = (_raster_inputs(grid, d, s) for s in (61, 62, 63))
    g = np.random.default_rng(64).standard_normal(grid)
    q, k, v = (S.raster_to_cube_major(x, TILE, POOL) for x in (xq, xk, xv))
    valid = np.ones(q.shape[0], bool)
    sc = O.router_scores(q, k)
    np.testing.assert_allclose(O.router_scores_padded(q, k, valid), sc, rtol=1e-12, atol=1e-15)
    sel = O.topk_select(sc.astype(np.float32), topk)
    o_f, _ = O.sparse_attn_fwd(q, k, v, sel["kv_off"], sel["kv_idx"])
    np.testing.assert_allclose(O.sparse_attn_fwd_padded(q, k, v, sel["kv_off"], sel["kv_idx"], valid), o_f,
                               rtol=1e-12, atol=1e-14)
    o_c, _ = O.coarse_attn(q, k, v)
    np.testing.assert_allclose(O.coarse_attn_padded(q, k, v, valid), o_c, rtol=1e-12, atol=1e-14)
    o_all, _ = O.vsa2_forward_padded(xq, xk, xv, g, topk)
    want = O.gated_merge(o_f, o_c, S.raster_to_cube_major(g[..., None], TILE, POOL)[:, 0])
    np.testing.assert_allclose(o_all, S.cube_major_to_raster(want, grid, TILE, POOL), rtol=1e-12, atol=1e-14)


def test_padding_values_change_no_real_output():
    """Fill the padding with large values instead of zeros: every output on real tokens is
    bit-identical, so the padding is masked everywhere (pooling, router softmax, both branches)."""
    grid, d = (6, 7, 10), 8
    rng = np.random.default_rng(65)
    x = {n: _raster_inputs(grid, d, s) for n, s in zip("qkv", (66, 67, 68))}
    cm = {n: _padded_cube_major(x[n]) for n in "qkv"}
    q, vm, grid_p = cm["q"]
    k, v = cm["k"][0], cm["v"][0]
    noisy = {n: np.where(vm[:, None], a, 50.0 * rng.standard_normal(a.shape)) for n, a in (("q", q), ("k", k), ("v", v))}
    sc = O.router_scores_padded(q, k, vm)
    np.testing.assert_array_equal(O.router_scores_padded(noisy["q"], noisy["k"], vm), sc)
    np.testing.assert_allclose(sc.sum(axis=1), 1.0, rtol=1e-12)
    sel = O.topk_select(sc.astype(np.float32), 4)
    o = O.sparse_attn_fwd_padded(q, k, v, sel["kv_off"], sel["kv_idx"], vm)
    o2 = O.sparse_attn_fwd_padded(noisy["q"], noisy["k"], noisy["v"], sel["kv_off"], sel["kv_idx"], vm)
    np.testing.assert_array_equal(o2[vm], o[vm])
    np.testing.assert_array_equal(O.coarse_attn_padded(noisy["q"], noisy["k"], noisy["v"], vm),
                                  O.coarse_attn_padded(q, k, v, vm))


def test_padded_full_budget_fine_branch_is_dense_attention_over_real_tokens():
    grid, d = (5, 6, 9), 8
    x = {n: _raster_inputs(grid, d, s) for n, s in zip("qkv", (69, 70, 71))}
    (q, vm, grid_p), (k, _, _), (v, _, _) = (_padded_cube_major(x[n]) for n in "qkv")
    N = q.shape[0] // 64
    sel = O.topk_select(np.ones((N, N), np.float32), N)  # every tile pair
    o = O.sparse_attn_fwd_padded(q, k, v, sel["kv_off"], sel["kv_idx"], vm)
    got = O.permute_to_raster(o, grid_p)[:grid[0], :grid[1], :grid[2]].reshape(-1, d)
    tq, tk, tv = (torch.from_numpy(x[n].reshape(-1, d))[None, None] for n in "qkv")
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def _padded_case(grid=(5, 6, 7), d=8, seed=90):
    """Padded cube-major q, k, v, dO (real rows smooth fields, padding rows large noise, which
    must not matter) and the real-token mask."""
    rng = np.random.default_rng(seed)
    cm = [_padded_cube_major(_raster_inputs(grid, d, seed + i, smooth=False)) for i in range(4)]
    vm = cm[0][1]
    q, k, v, do = (np.where(vm[:, None], c[0], 30.0 * rng.standard_normal(c[0].shape)) for c in cm)
    return q, k, v, do, vm


def test_padded_backward_equals_the_unpadded_one_on_divisible_grids():
    rng = np.random.default_rng(91)
    L, D = 3 * 64, 8
    q, k, v, do = (rng.standard_normal((L, D)) for _ in range(4))
    valid = np.ones(L, bool)
    off, idx = _csr(np.array([[1, 0, 1], [0, 0, 0], [1, 1, 0]], bool))
    for got, want in zip(O.sparse_attn_bwd_padded(q, k, v, do, off, idx, valid), O.sparse_attn_bwd(q, k, v, do, off, idx)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)
    d_oc = rng.standard_normal((3, D))
    for got, want in zip(O.coarse_attn_bwd_padded(q, k, v, d_oc, valid), O.coarse_attn_bwd(q, k, v, d_oc)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)
    oc, g = rng.standard_normal((3, D)), rng.standard_normal(L)
    for got, want in zip(O.gated_merge_bwd_padded(do, oc, g, valid), O.gated_merge_bwd(do, oc, g)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def _fd_check(loss, args, grads, rng, eps=1e-6):
    """Central differences of `loss` along a random direction of every argument (padding rows
    included) against the analytic directional derivative."""
    for name in grads:
        dirn = rng.standard_normal(args[name].shape)
        plus = dict(args, **{name: args[name] + eps * dirn})
        minus = dict(args, **{name: args[name] - eps * dirn})
        fd = (loss(**plus) - loss(**minus)) / (2 * eps)
        an = float(np.sum(grads[name] * dirn))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_padded_fine_backward_central_finite_differences():
    """The loss sums dO * O over real rows only (padding rows are dropped); padding tokens of
    q, k, v are perturbed too and must have zero gradient."""
    q, k, v, do, vm = _padded_case()
    N = q.shape[0] // 64
    rng = np.random.default_rng(92)
    mask = rng.random((N, N)) < 0.4
    mask[1] = False  # an empty row
    mask[2, 3] = True
    off, idx = _csr(mask)

    def loss(q, k, v):
        o = O.sparse_attn_fwd_padded(q, k, v, off, idx, vm)
        return float(np.sum((o * do)[vm]))

    dq, dk, dv = O.sparse_attn_bwd_padded(q, k, v, do, off, idx, vm)
    for g in (dq, dk, dv):
        assert np.all(g[~vm] == 0)
    assert np.all(dq[64:128] == 0)
    _fd_check(loss, {"q": q, "k": k, "v": v}, {"q": dq, "k": dk, "v": dv}, rng)


def test_padded_coarse_and_merge_backward_central_finite_differences():
    q, k, v, do, vm = _padded_case(seed=93)
    N, D = q.shape[0] // 64, q.shape[1]
    rng = np.random.default_rng(94)
    d_oc = rng.standard_normal((N, D))

    def loss_c(q, k, v):
        return float(np.sum(O.coarse_attn_padded(q, k, v, vm) * d_oc))

    dq, dk, dv = O.coarse_attn_bwd_padded(q, k, v, d_oc, vm)
    for g in (dq, dk, dv):
        assert np.all(g[~vm] == 0)
    _fd_check(loss_c, {"q": q, "k": k, "v": v}, {"q": dq, "k": dk, "v": dv}, rng)
    o_f, oc, g = rng.standard_normal((q.shape[0], D)), rng.standard_normal((N, D)), rng.standard_normal(q.shape[0])

    def loss_m(o_f, oc, g):
        return float(np.sum((O.gated_merge(o_f, oc, g) * do)[vm]))

    d_of, d_oc2, d_g = O.gated_merge_bwd_padded(do, oc, g, vm)
    assert np.all(d_of[~vm] == 0) and np.all(d_g[~vm] == 0)
    _fd_check(loss_m, {"o_f": o_f, "oc": oc, "g": g}, {"o_f": d_of, "oc": d_oc2, "g": d_g}, rng)


def _router_padded_bruteforce(xq, xk, grid):
    """Eq. 5-7 with padding on the raster grid, explicit loops: pad to whole 4x4x4 tiles; each
    2x2x4 sub-cube's pooled vectors average its real tokens; sub-cubes without one are skipped
    as queries and keys; the score of tile pair (i, j) is the mean over i's real query
    sub-cubes of the softmax mass on j's sub-cubes."""
    T, H, W = grid
    D = xq.shape[-1]
    nt, nh, nw = -(-T // 4), -(-H // 4), -(-W // 4)
    subs = []
    for a, b, c in itertools.product(range(nt), range(nh), range(nw)):
        tile = (a * nh + b) * nw + c
        for st, sh in itertools.product(range(2), range(2)):
            qs, ks, n = np.zeros(D), np.zeros(D), 0
            for dt, dh, dw in itertools.product(range(2), range(2), range(4)):
                t, h, w = 4 * a + 2 * st + dt, 4 * b + 2 * sh + dh, 4 * c + dw
                if t < T and h < H and w < W:
                    qs += xq[t, h, w]
                    ks += xk[t, h, w]
                    n += 1
            if n:
                subs.append((tile, qs / n, ks / n))
    N = nt * nh * nw
    out = np.zeros((N, N))
    g = np.zeros(N)
    for ti, qa, _ in subs:
        g[ti] += 1
        logits = [float(qa @ kb) / math.sqrt(D) for _, _, kb in subs]
        m = max(logits)
        ex = [math.exp(z - m) for z in logits]
        z = sum(ex)
        for (tj, _, _), e in zip(subs, ex):
            out[ti, tj] += e / z
    return out / g[:, None]


def _coarse_padded_bruteforce(xq, xk, xv, grid):
    T, H, W = grid
    D = xq.shape[-1]
    nt, nh, nw = -(-T // 4), -(-H // 4), -(-W // 4)
    means = {n: [] for n in "qkv"}
    for a, b, c in itertools.product(range(nt), range(nh), range(nw)):
        for n, x in zip("qkv", (xq, xk, xv)):
            acc, cnt = np.zeros(D), 0
            for dt, dh, dw in itertools.product(range(4), repeat=3):
                t, h, w = 4 * a + dt, 4 * b + dh, 4 * c + dw
                if t < T and h < H and w < W:
                    acc += x[t, h, w]
                    cnt += 1
            means[n].append(acc / cnt)
    out = []
    for qi in means["q"]:
        logits = [float(qi @ kj) / math.sqrt(D) for kj in means["k"]]
        m = max(logits)
        ex = [math.exp(z - m) for z in logits]
        out.append(sum(e * vj for e, vj in zip(ex, means["v"])) / sum(ex))
    return np.array(out)


@pytest.mark.parametrize("grid", [(6, 7, 10), (5, 8, 5)])
def test_router_and_coarse_padded_match_bruteforce_on_raster_grid(grid):
    d = 8
    xq, xk, xv = (_raster_inputs(grid, d, s) for s in (72, 73, 74))
    (q, vm, _), (k, _, _), (v, _, _) = (_padded_cube_major(x) for x in (xq, xk, xv))
    np.testing.assert_allclose(O.router_scores_padded(q, k, vm), _router_padded_bruteforce(xq, xk, grid),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(O.coarse_attn_padded(q, k, v, vm), _coarse_padded_bruteforce(xq, xk, xv, grid),
                               rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------------------------
# per-query-tile TopK (VSA's selection, the variant of §2.2)
# --------------------------------------------------------------------------------------------

def test_topk_per_row_bruteforce_with_ties():
    rng = np.random.default_rng(81)
    N, K = 9, 4
    s = (rng.integers(0, 4, (N, N)) / 4).astype(np.float32)  # heavy ties
    sel = O.topk_select_per_row(s, K)
    for i in range(N):
        want = sorted(sorted(range(N), key=lambda j: (-float(s[i, j]), j))[:K])
        assert list(sel["kv_idx"][sel["kv_off"][i]:sel["kv_off"][i + 1]]) == want
    assert np.all(sel["mask"].sum(axis=1) == K)
    # the CSC lists the same pairs, column by column
    for j in range(N):
        assert list(sel["q_idx"][sel["q_off"][j]:sel["q_off"][j + 1]]) == list(np.nonzero(sel["mask"][:, j])[0])


def test_topk_per_row_separable_scores_closed_form():
    """Scores f(i) + g(j): every row ranks the KV tiles by g alone, so all rows keep the K tiles
    of largest g."""
    rng = np.random.default_rng(82)
    N, K = 12, 5
    f, g = rng.standard_normal(N), rng.permutation(N).astype(np.float64)
    s = (f[:, None] + g[None, :]).astype(np.float32)  # g's gaps of 1 survive fp32 rounding
    sel = O.topk_select_per_row(s, K)
    best = np.sort(np.argsort(-g)[:K])
    for i in range(N):
        np.testing.assert_array_equal(sel["kv_idx"][i * K:(i + 1) * K], best)


def test_topk_per_row_full_budget_equals_per_sequence():
    s = np.random.default_rng(83).random((7, 7)).astype(np.float32)
    a, b = O.topk_select_per_row(s, 7), O.topk_select(s, 7)
    for key in ("kv_off", "kv_idx", "q_off", "q_idx"):
        np.testing.assert_array_equal(a[key], b[key])
