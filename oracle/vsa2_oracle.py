"""Plain fp64 CPU oracle for the VSA2 hot path. TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check of the package entry module and the benchmark's CPU
baseline leg may import this module. The product path (the CUDA library and its Python
binding) never calls it and shares no code with it.

Source: "Improving Video Sparse Attention with Fine-grained Router and Sparse Rebasing"
(arXiv 2609.32882), §2.1 Background and §2.2 VSA2: Eq. 5-9 (router, TopK), Eq. 12 (fine
branch), Eq. 1-4 (coarse branch) and Eq. 13-14 (gated merge).

Layout: every per-(b, h) tensor is (L, D) in cube-major token order (§2.2 "Permutation"):
tile i is rows [i*Bt, (i+1)*Bt); inside it, router sub-cube a is rows [a*R, (a+1)*R), so tile i
owns sub-cubes G*i .. G*i+G-1 with G = Bt / R.

Readings of the pages that this oracle commits to (each is listed in the design notes):
  * Eq. 7 "MeanPool_{GxG}" is emitted scaled by G (mean over the G query sub-cubes, sum over the
    G key sub-cubes), so each score row sums to 1. G is a power of two, so the scaling is exact
    and leaves the TopK result unchanged.
  * Eq. 8-9 TopK: scores are ranked in fp32 (the kernel's precision), descending; equal scores
    go to the lower flat index i*N + j. The budget N*K is per (batch, head).
  * Eq. 12 for a query tile with no selected KV tile: output 0, LSE = -inf, zero gradients.
  * Softmax scale 1/sqrt(D) (§2.1).
  * Eq. 13's gate G = tanh(X W_g) takes the projection X W_g (one value per token and head) as
    its input: the projection of the hidden states belongs with the layer's input projections.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "mean_pool",
    "router_scores",
    "router_scores_dense_attention",
    "topk_select",
    "topk_select_per_row",
    "sparse_attn_fwd",
    "sparse_attn_bwd",
    "coarse_attn",
    "gated_merge",
    "coarse_attn_bwd",
    "gated_merge_bwd",
    "permute_to_cube_major",
    "permute_to_raster",
    "pad_to_tiles",
    "router_scores_padded",
    "sparse_attn_fwd_padded",
    "coarse_attn_padded",
    "vsa2_forward_padded",
    "sparse_attn_bwd_padded",
    "coarse_attn_bwd_padded",
    "gated_merge_bwd_padded",
]


def mean_pool(x: np.ndarray, group: int) -> np.ndarray:
    """MeanPool over consecutive groups of `group` tokens of a cube-major (L, D) tensor (Eq. 5)."""
    x = np.asarray(x, dtype=np.float64)
    L, D = x.shape
    return x.reshape(L // group, group, D).mean(axis=1)


def router_scores(q: np.ndarray, k: np.ndarray, tile_tokens: int = 64, pool_tokens: int = 16,
                  row_chunk: int = 2048) -> np.ndarray:
    """Tile-level router scores Pr (N, N) for one (b, h), Eq. 5-7.

    Qr, Kr = MeanPool_R(Q, K)                        (Eq. 5)
    P_hat  = row-softmax(Qr Kr^T / sqrt(D))          (Eq. 6), over all L/R pooled keys
    Pr[i,j] = (1/G) sum_{a in i} sum_{b in j} P_hat[a,b]   (Eq. 7, scaled by G; rows sum to 1)

    P_hat is formed exactly (max-subtracted fp64), a block of pooled query rows at a time; each
    block holds complete rows, so the softmax is the textbook one.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    L, D = q.shape
    G = tile_tokens // pool_tokens
    N = L // tile_tokens
    qr = mean_pool(q, pool_tokens)
    kr = mean_pool(k, pool_tokens)
    Lr = qr.shape[0]
    scale = 1.0 / np.sqrt(D)
    out = np.empty((N, N), dtype=np.float64)
    rows_per = max(G, (row_chunk // G) * G)
    for a0 in range(0, Lr, rows_per):
        a1 = min(Lr, a0 + rows_per)
        s = (qr[a0:a1] @ kr.T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        # pool: G query sub-rows of each tile (mean) x G key sub-cubes of each tile (sum)
        blk = p.reshape((a1 - a0) // G, G, N, G).sum(axis=(1, 3)) / G
        out[a0 // G:a1 // G] = blk
    return out


def router_scores_dense_attention(q: np.ndarray, k: np.ndarray, tile_tokens: int = 64) -> np.ndarray:
    """The compute-unbounded router of Eq. 10-11: token-level softmax, then tile pooling
    (scaled like `router_scores` so rows sum to 1). Diagnostic only (router recall)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    L, D = q.shape
    N = L // tile_tokens
    s = (q @ k.T) / np.sqrt(D)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p.reshape(N, tile_tokens, N, tile_tokens).sum(axis=(1, 3)) / tile_tokens


def topk_select(scores: np.ndarray, topk: int) -> dict:
    """Per-sequence TopK over the flattened N x N tile scores (Eq. 8-9).

    `scores` must be float32 (the precision in which both sides rank). Entries are ordered by
    (score descending, flat index ascending) and the first N*topk are kept. Returns the boolean
    mask and its CSR (per query tile, ascending KV tile) and CSC (per KV tile, ascending query
    tile) index lists as int32 arrays.
    """
    s = np.asarray(scores)
    if s.dtype != np.float32:
        raise TypeError("rank in fp32: pass float32 scores")
    N = s.shape[0]
    if s.shape != (N, N):
        raise ValueError("scores must be square")
    if not (1 <= topk <= N):
        raise ValueError("need 1 <= topk <= N")
    flat = s.reshape(-1)
    budget = N * topk
    order = np.lexsort((np.arange(N * N), -flat.astype(np.float64)))
    mask = np.zeros(N * N, dtype=bool)
    mask[order[:budget]] = True
    mask = mask.reshape(N, N)
    counts = mask.sum(axis=1)
    kv_off = np.zeros(N + 1, dtype=np.int32)
    kv_off[1:] = np.cumsum(counts)
    kv_idx = np.nonzero(mask)[1].astype(np.int32)  # row-major scan: ascending j within row i
    ccounts = mask.sum(axis=0)
    q_off = np.zeros(N + 1, dtype=np.int32)
    q_off[1:] = np.cumsum(ccounts)
    q_idx = np.nonzero(mask.T)[1].astype(np.int32)
    return {"mask": mask, "kv_off": kv_off, "kv_idx": kv_idx, "q_off": q_off, "q_idx": q_idx}


def topk_select_per_row(scores: np.ndarray, topk: int) -> dict:
    """The per-query-tile TopK of VSA, the variant §2.2 contrasts with Eq. 8-9: every query tile
    keeps its own `topk` best KV tiles, so each row has exactly `topk` entries. Ranked in fp32,
    descending; equal scores go to the lower KV tile. Same output format as `topk_select`."""
    s = np.asarray(scores)
    if s.dtype != np.float32:
        raise TypeError("rank in fp32: pass float32 scores")
    N = s.shape[0]
    if s.shape != (N, N) or not (1 <= topk <= N):
        raise ValueError("need square scores and 1 <= topk <= N")
    mask = np.zeros((N, N), dtype=bool)
    for i in range(N):
        order = np.lexsort((np.arange(N), -s[i].astype(np.float64)))
        mask[i, order[:topk]] = True
    kv_off = np.arange(N + 1, dtype=np.int32) * topk
    kv_idx = np.nonzero(mask)[1].astype(np.int32)
    q_off = np.zeros(N + 1, dtype=np.int32)
    q_off[1:] = np.cumsum(mask.sum(axis=0))
    q_idx = np.nonzero(mask.T)[1].astype(np.int32)
    return {"mask": mask, "kv_off": kv_off, "kv_idx": kv_idx, "q_off": q_off, "q_idx": q_idx}


def _tiles(x: np.ndarray, tile_tokens: int) -> np.ndarray:
    L, D = x.shape
    return x.reshape(L // tile_tokens, tile_tokens, D)


def sparse_attn_fwd(q, k, v, kv_off, kv_idx, tile_tokens: int = 64, query_tiles=None):
    """Block-sparse attention forward for one (b, h), Eq. 12 with the §2.1 definition:
    for each query token t of tile i, o_t = sum_u softmax_u(q_t . k_u / sqrt(D)) v_u over the
    tokens u of the KV tiles selected for tile i; lse_t = log sum_u exp(q_t . k_u / sqrt(D)).

    Returns (o (L, D) fp64, lse (L,) fp64). With `query_tiles` given, only those tiles are
    computed (rows of other tiles are left as NaN) - used to time a bounded sample.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, D = q.shape
    N = L // tile_tokens
    scale = 1.0 / np.sqrt(D)
    qt, kt, vt = _tiles(q, tile_tokens), _tiles(k, tile_tokens), _tiles(v, tile_tokens)
    o = np.full((N, tile_tokens, D), np.nan)
    lse = np.full((N, tile_tokens), np.nan)
    for i in (range(N) if query_tiles is None else query_tiles):
        sel = np.asarray(kv_idx[kv_off[i]:kv_off[i + 1]])
        if sel.size == 0:
            o[i] = 0.0
            lse[i] = -np.inf
            continue
        ks = kt[sel].reshape(-1, D)
        vs = vt[sel].reshape(-1, D)
        s = (qt[i] @ ks.T) * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[i] = (p @ vs) / l
        lse[i] = (m + np.log(l))[:, 0]
    return o.reshape(L, D), lse.reshape(L)


def sparse_attn_bwd(q, k, v, do, kv_off, kv_idx, tile_tokens: int = 64, query_tiles=None, o=None):
    """Gradients (dQ, dK, dV) of the Eq. 12 output for one (b, h) given upstream dO.

    Textbook softmax-attention backward restricted to the selected tile pairs (the router
    receives no gradient, §2.1): with P the softmax of S = Q K_S^T / sqrt(D) per query row,
    dV_S = P^T dO, dP = dO V_S^T, dS = P * (dP - rowsum(dO * O)), dQ = dS K_S / sqrt(D),
    dK_S = dS^T Q / sqrt(D). The softmax is recomputed here in fp64 from Q, K, V.

    With `query_tiles` given, only those query tiles contribute: dQ is then exact on them, and
    dK, dV are exact on every KV tile all of whose selecting query tiles are in the subset.

    `o` is the forward output the rowsum(dO * O) term is formed from, as in a backward pass
    that receives the stored output of the forward (for instance rounded to the storage
    dtype); by default the exact O recomputed here.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    L, D = q.shape
    N = L // tile_tokens
    scale = 1.0 / np.sqrt(D)
    qt, kt, vt, dot = (_tiles(x, tile_tokens) for x in (q, k, v, do))
    ot = None if o is None else _tiles(np.asarray(o, dtype=np.float64), tile_tokens)
    dq = np.zeros_like(qt)
    dk = np.zeros_like(kt)
    dv = np.zeros_like(vt)
    for i in (range(N) if query_tiles is None else query_tiles):
        sel = np.asarray(kv_idx[kv_off[i]:kv_off[i + 1]])
        if sel.size == 0:
            continue
        ks = kt[sel].reshape(-1, D)
        vs = vt[sel].reshape(-1, D)
        s = (qt[i] @ ks.T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        oi = p @ vs if ot is None else ot[i]
        delta = np.sum(dot[i] * oi, axis=1, keepdims=True)
        dvs = p.T @ dot[i]
        dp = dot[i] @ vs.T
        ds = p * (dp - delta)
        dq[i] = (ds @ ks) * scale
        dks = (ds.T @ qt[i]) * scale
        n = sel.size
        np.add.at(dk, sel, dks.reshape(n, tile_tokens, D))
        np.add.at(dv, sel, dvs.reshape(n, tile_tokens, D))
    return dq.reshape(L, D), dk.reshape(L, D), dv.reshape(L, D)


def coarse_attn(q, k, v, tile_tokens: int = 64):
    """Coarse branch for one (b, h), Eq. 1-3:
    Qc, Kc, Vc = MeanPool_B(Q, K, V)            (Eq. 1), one row per tile, (N, D)
    P_c        = row-softmax(Qc Kc^T / sqrt(D)) (Eq. 2), over all N tiles
    O_c_hat    = P_c Vc                         (Eq. 3)
    Returns (O_c_hat (N, D) fp64, lse_c (N,) fp64 = log of each row's softmax denominator).
    """
    qc = mean_pool(q, tile_tokens)
    kc = mean_pool(k, tile_tokens)
    vc = mean_pool(v, tile_tokens)
    D = qc.shape[1]
    s = (qc @ kc.T) / np.sqrt(D)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ vc) / l, (m + np.log(l))[:, 0]


def gated_merge(o_f, o_c_hat, gate_logits, tile_tokens: int = 64):
    """Output of one (b, h), Eq. 4 and Eq. 13-14:
    O_c = Repeat_B(O_c_hat)       (Eq. 4), every token of tile i gets row i
    G   = tanh(X W_g)             (Eq. 13), gate_logits = X W_g, one per token, shape (L,)
    O   = G * O_c + O_f           (Eq. 14), G broadcast over the D channels
    """
    o_f = np.asarray(o_f, dtype=np.float64)
    o_c = np.repeat(np.asarray(o_c_hat, dtype=np.float64), tile_tokens, axis=0)
    g = np.tanh(np.asarray(gate_logits, dtype=np.float64))[:, None]
    return g * o_c + o_f


def coarse_attn_bwd(q, k, v, d_oc, o_c_hat=None):
    """Gradients of Eq. 1-3 for one (b, h): given d_oc = dLoss/dO_c_hat (N, D), returns
    (dQ, dK, dV), each (L, D). With P_c, O_c_hat from the forward:
    dP   = d_oc Vc^T,  Delta = rowsum(d_oc * O_c_hat),  dS = P_c * (dP - Delta)
    dQc  = dS Kc / sqrt(D),  dKc = dS^T Qc / sqrt(D),  dVc = P_c^T d_oc
    and MeanPool_B spreads each pooled gradient evenly: dQ[t] = dQc[tile(t)] / B, same for K, V.

    `o_c_hat`, when given, is the forward output Delta is formed from, as in a backward pass that
    receives the stored output of the forward; by default the exact output is recomputed.
    """
    qc = mean_pool(q, 64)
    kc = mean_pool(k, 64)
    vc = mean_pool(v, 64)
    d_oc = np.asarray(d_oc, dtype=np.float64)
    D = qc.shape[1]
    s = (qc @ kc.T) / np.sqrt(D)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    o = p @ vc if o_c_hat is None else np.asarray(o_c_hat, dtype=np.float64)
    dp = d_oc @ vc.T
    delta = (d_oc * o).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    dqc = ds @ kc / np.sqrt(D)
    dkc = ds.T @ qc / np.sqrt(D)
    dvc = p.T @ d_oc
    return tuple(np.repeat(x, 64, axis=0) / 64.0 for x in (dqc, dkc, dvc))


def gated_merge_bwd(dout, o_c_hat, gate_logits, tile_tokens: int = 64):
    """Gradients of Eq. 4, 13-14 for one (b, h), given dout = dLoss/dO (L, D):
    dO_f           = dout
    dO_c_hat[i]    = sum over the tokens t of tile i of G[t] * dout[t]   (Repeat_B's adjoint)
    d gate_logits  = (1 - G^2) * rowsum(dout * O_c)                     (tanh' = 1 - tanh^2)
    Returns (dO_f (L, D), dO_c_hat (N, D), d_gate_logits (L,)).
    """
    dout = np.asarray(dout, dtype=np.float64)
    g = np.tanh(np.asarray(gate_logits, dtype=np.float64))
    o_c = np.repeat(np.asarray(o_c_hat, dtype=np.float64), tile_tokens, axis=0)
    L, D = dout.shape
    d_oc = (g[:, None] * dout).reshape(L // tile_tokens, tile_tokens, D).sum(axis=1)
    d_logits = (1.0 - g * g) * (dout * o_c).sum(axis=1)
    return dout.copy(), d_oc, d_logits


def _cube_major_coords(grid, tile, pool):
    """Raster coordinates (t, h, w) of the tokens in cube-major order (§2.2 "Permutation"):
    tiles of `tile` tokens in raster order over the tile grid; inside a tile, its sub-cubes of
    `pool` tokens in raster order; inside a sub-cube, its tokens in raster order."""
    T, H, W = grid
    bt, bh, bw = tile
    rt, rh, rw = pool
    for a in range(T // bt):
        for b in range(H // bh):
            for c in range(W // bw):
                for st in range(bt // rt):
                    for sh in range(bh // rh):
                        for sw in range(bw // rw):
                            for dt in range(rt):
                                for dh in range(rh):
                                    for dw in range(rw):
                                        yield (a * bt + st * rt + dt, b * bh + sh * rh + dh, c * bw + sw * rw + dw)


def permute_to_cube_major(x, tile=(4, 4, 4), pool=(2, 2, 4)):
    """(T, H, W, D) tokens in raster order -> (T*H*W, D) in cube-major order."""
    T, H, W, D = x.shape
    return np.stack([x[t, h, w] for t, h, w in _cube_major_coords((T, H, W), tile, pool)])


def permute_to_raster(y, grid, tile=(4, 4, 4), pool=(2, 2, 4)):
    """Inverse of permute_to_cube_major: (T*H*W, D) cube-major -> (T, H, W, D) raster."""
    T, H, W = grid
    out = np.empty((T, H, W, y.shape[1]), dtype=y.dtype)
    for l, (t, h, w) in enumerate(_cube_major_coords(grid, tile, pool)):
        out[t, h, w] = y[l]
    return out


# ------------------------------------------------------------------------------------------
# grids that the tile does not divide (§2.2 "Kernel Implementation": pad every dimension to a
# multiple of the tile and mask the padding). Readings: pooled means run over real tokens only;
# a sub-cube with no real token is masked as a key and has no query row; Eq. 7 averages the
# real query sub-cubes of a tile; padding keys are masked in both attention branches; rows of
# padding tokens are dropped when the output is cropped back to the grid.
# ------------------------------------------------------------------------------------------

def pad_to_tiles(x, tile=(4, 4, 4)):
    """(T, H, W, D) raster -> ((T', H', W', D) zero-padded to multiples of the tile,
    (T', H', W') bool mask of the real tokens)."""
    T, H, W, D = x.shape
    Tp, Hp, Wp = (-(-n // b) * b for n, b in zip((T, H, W), tile))
    out = np.zeros((Tp, Hp, Wp, D), dtype=np.float64)
    out[:T, :H, :W] = x
    valid = np.zeros((Tp, Hp, Wp), dtype=bool)
    valid[:T, :H, :W] = True
    return out, valid


def _masked_mean_pool(x, valid, group):
    """Mean of the real rows of each group of `group` consecutive rows, and their counts."""
    x = np.asarray(x, dtype=np.float64)
    L, D = x.shape
    w = np.asarray(valid, dtype=np.float64).reshape(L // group, group)
    sums = (x.reshape(L // group, group, D) * w[:, :, None]).sum(axis=1)
    counts = w.sum(axis=1)
    means = np.where(counts[:, None] > 0, sums / np.maximum(counts, 1)[:, None], 0.0)
    return means, counts


def router_scores_padded(q, k, valid, tile_tokens: int = 64, pool_tokens: int = 16):
    """Eq. 5-7 on a padded cube-major sequence; `valid` (L,) marks the real tokens.
    Qr, Kr are means over real tokens; sub-cubes without one are masked keys and have no
    query row; Pr[i, j] = (1 / g_i) sum over the g_i real query sub-cubes a of tile i of
    sum over the real key sub-cubes b of tile j of P_hat[a, b]."""
    qr, cq = _masked_mean_pool(q, valid, pool_tokens)
    kr, ck = _masked_mean_pool(k, valid, pool_tokens)
    G = tile_tokens // pool_tokens
    Lr, D = qr.shape
    N = Lr // G
    s = (qr @ kr.T) / np.sqrt(D)
    s[:, ck == 0] = -np.inf
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    p[cq == 0] = 0.0
    g = (cq > 0).reshape(N, G).sum(axis=1)
    return p.reshape(N, G, N, G).sum(axis=(1, 3)) / g[:, None]


def sparse_attn_fwd_padded(q, k, v, kv_off, kv_idx, valid, tile_tokens: int = 64):
    """Eq. 12 with padding keys masked: for each query token t of tile i, the softmax runs over
    the real tokens of the tiles selected for i. Padding query rows are returned as 0 (they
    are dropped with the padding)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, D = q.shape
    N = L // tile_tokens
    o = np.zeros((L, D))
    for i in range(N):
        sel = np.asarray(kv_idx[kv_off[i]:kv_off[i + 1]])
        if sel.size == 0:
            continue
        keys = np.concatenate([np.arange(j * tile_tokens, (j + 1) * tile_tokens) for j in sel])
        keys = keys[np.asarray(valid)[keys]]
        rows = np.arange(i * tile_tokens, (i + 1) * tile_tokens)
        s = (q[rows] @ k[keys].T) / np.sqrt(D)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        o[rows] = (p @ v[keys]) / p.sum(axis=1, keepdims=True)
    o[~np.asarray(valid)] = 0.0
    return o


def coarse_attn_padded(q, k, v, valid, tile_tokens: int = 64):
    """Eq. 1-3 on a padded sequence: Qc, Kc, Vc are means over the real tokens of each tile
    (every tile of a padded grid holds one), then the dense softmax of Eq. 2 over all tiles."""
    qc, _ = _masked_mean_pool(q, valid, tile_tokens)
    kc, _ = _masked_mean_pool(k, valid, tile_tokens)
    vc, _ = _masked_mean_pool(v, valid, tile_tokens)
    D = qc.shape[1]
    s = (qc @ kc.T) / np.sqrt(D)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ vc) / p.sum(axis=1, keepdims=True)


def vsa2_forward_padded(q, k, v, gate_logits, topk, tile=(4, 4, 4), pool=(2, 2, 4)):
    """Eq. 1-14 for one (b, h) on a raster grid (T, H, W) that the tile need not divide:
    pad, permute to cube-major order, router with masked padding, per-sequence TopK over the
    padded grid's tiles (budget N' * topk), fine and coarse branches with padding keys masked,
    gated merge, then back to raster order, cropped to (T, H, W). Returns (O (T, H, W, D),
    the TopK selection)."""
    T, H, W, D = q.shape
    qp, valid = pad_to_tiles(q, tile)
    kp, _ = pad_to_tiles(k, tile)
    vp, _ = pad_to_tiles(v, tile)
    gp, _ = pad_to_tiles(np.asarray(gate_logits, dtype=np.float64)[..., None], tile)
    grid_p = qp.shape[:3]
    qc, kc, vc, gc = (permute_to_cube_major(x, tile, pool) for x in (qp, kp, vp, gp))
    vm = permute_to_cube_major(valid[..., None].astype(np.float64), tile, pool)[:, 0] > 0
    tile_tokens = int(np.prod(tile))
    pool_tokens = int(np.prod(pool))
    scores = router_scores_padded(qc, kc, vm, tile_tokens, pool_tokens)
    sel = topk_select(scores.astype(np.float32), topk)
    o_f = sparse_attn_fwd_padded(qc, kc, vc, sel["kv_off"], sel["kv_idx"], vm, tile_tokens)
    o_c = coarse_attn_padded(qc, kc, vc, vm, tile_tokens)
    o = gated_merge(o_f, o_c, gc[:, 0], tile_tokens)
    return permute_to_raster(o, grid_p, tile, pool)[:T, :H, :W], sel


def sparse_attn_bwd_padded(q, k, v, do, kv_off, kv_idx, valid, tile_tokens: int = 64, o=None):
    """Gradients (dQ, dK, dV) of `sparse_attn_fwd_padded` for one (b, h), given dO.

    The output of a padding query row is the constant 0 (it is dropped with the padding), so its
    dO reaches no input and its dQ is 0; padding keys take no part in any softmax, so the dK and
    dV of padding tokens are 0. On the real rows of query tile i, with the real tokens of its
    selected tiles as the keys, the textbook backward of `sparse_attn_bwd`:
    dV += P^T dO, dS = P * (dO V^T - rowsum(dO * O)), dQ = dS K / sqrt(D), dK += dS^T Q / sqrt(D).
    `o`, when given, is the stored forward output the rowsum is formed from."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    valid = np.asarray(valid, dtype=bool)
    L, D = q.shape
    N = L // tile_tokens
    scale = 1.0 / np.sqrt(D)
    dq, dk, dv = np.zeros((L, D)), np.zeros((L, D)), np.zeros((L, D))
    for i in range(N):
        sel = np.asarray(kv_idx[kv_off[i]:kv_off[i + 1]])
        rows = np.arange(i * tile_tokens, (i + 1) * tile_tokens)
        rows = rows[valid[rows]]
        if sel.size == 0 or rows.size == 0:
            continue
        keys = np.concatenate([np.arange(j * tile_tokens, (j + 1) * tile_tokens) for j in sel])
        keys = keys[valid[keys]]  # distinct tokens: the selected tiles are distinct
        s = (q[rows] @ k[keys].T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        oi = p @ v[keys] if o is None else np.asarray(o, dtype=np.float64)[rows]
        delta = np.sum(do[rows] * oi, axis=1, keepdims=True)
        dv[keys] += p.T @ do[rows]
        ds = p * (do[rows] @ v[keys].T - delta)
        dq[rows] = (ds @ k[keys]) * scale
        dk[keys] += (ds.T @ q[rows]) * scale
    return dq, dk, dv


def coarse_attn_bwd_padded(q, k, v, d_oc, valid, tile_tokens: int = 64, o_c_hat=None):
    """Gradients of `coarse_attn_padded` for one (b, h), given d_oc = dLoss/dO_c_hat (N, D):
    the pooled-level backward of Eq. 2-3 as in `coarse_attn_bwd`, then the adjoint of the mean
    over a tile's real tokens: each of the n_i real tokens of tile i gets dQc[i] / n_i (same for
    K, V); padding tokens get 0."""
    valid = np.asarray(valid, dtype=bool)
    qc, cnt = _masked_mean_pool(q, valid, tile_tokens)
    kc, _ = _masked_mean_pool(k, valid, tile_tokens)
    vc, _ = _masked_mean_pool(v, valid, tile_tokens)
    d_oc = np.asarray(d_oc, dtype=np.float64)
    D = qc.shape[1]
    s = (qc @ kc.T) / np.sqrt(D)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    o = p @ vc if o_c_hat is None else np.asarray(o_c_hat, dtype=np.float64)
    ds = p * (d_oc @ vc.T - (d_oc * o).sum(axis=1, keepdims=True))
    pooled = (ds @ kc / np.sqrt(D), ds.T @ qc / np.sqrt(D), p.T @ d_oc)
    w = valid[:, None] / np.repeat(np.maximum(cnt, 1), tile_tokens)[:, None]
    return tuple(np.repeat(x, tile_tokens, axis=0) * w for x in pooled)


def gated_merge_bwd_padded(dout, o_c_hat, gate_logits, valid, tile_tokens: int = 64):
    """Gradients of Eq. 4, 13-14 on a padded sequence: the outputs of padding rows are dropped,
    so their dout reaches nothing: `gated_merge_bwd` with dout set to 0 on padding rows (dO_f,
    d gate_logits 0 there; dO_c_hat sums the real tokens of each tile)."""
    valid = np.asarray(valid, dtype=bool)
    dout = np.where(valid[:, None], np.asarray(dout, dtype=np.float64), 0.0)
    return gated_merge_bwd(dout, o_c_hat, gate_logits, tile_tokens)
