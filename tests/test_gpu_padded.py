"""GPU parity on token grids that the 4x4x4 tile does not divide ("Improving Video Sparse
Attention with Fine-grained Router and Sparse Rebasing", §2.2 "Kernel Implementation": every
dimension is padded to a multiple of the tile and the padding is masked).

The raster inputs are permuted to the padded cube-major order by the library (padding rows
become zeros) and every step is compared with the oracle's padded functions, which follow the
same reading: pooled means over real tokens only, sub-cubes without a real token masked as keys
and left out as query rows, Eq. 7 averaged over a tile's real query sub-cubes, padding keys
masked in both attention branches, padding rows dropped on the way back to raster order.
Tolerances are the ones of the whole-tile tests; TopK is bit-exact on the oracle's scores.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import trainable_block_sparse_fine_b200 as V

TILE, POOL = (4, 4, 4), (2, 2, 4)


def _raster(grid, d, heads, dtype, seed):
    """[1, heads, T*H*W, D] smoothed fields in raster order, rounded to the dtype."""
    out = np.stack([S.round_to_dtype(S.smoothed_field(np.random.default_rng([seed, h]), grid, d), dtype)
                    for h in range(heads)])
    return out.reshape(1, heads, -1, d)


def _dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _close(got, want, what, tol_abs=2e-2, tol_rel=5e-3):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= tol_abs and rel <= tol_rel, f"{what}: max abs {err.max():.3e}, rel L2 {rel:.3e}"


def _padded_oracle_inputs(xr, grid, d):
    """Oracle side: raster (T*H*W, D) -> padded cube-major (L', D) and the real-token mask."""
    T, H, W = grid
    xp, valid = O.pad_to_tiles(xr.reshape(T, H, W, d), TILE)
    xc = O.permute_to_cube_major(xp, TILE, POOL)
    vm = O.permute_to_cube_major(valid[..., None].astype(np.float64), TILE, POOL)[:, 0] > 0
    return xc, vm


CASES = {
    "6x7x10_bf16": ((6, 7, 10), 128, "bf16", 3, 2),
    "5x8x5_bf16": ((5, 8, 5), 128, "bf16", 2, 2),
    "6x7x10_fp32_d64": ((6, 7, 10), 64, "fp32", 3, 1),   # the CUDA-core kernels
    "480p_ragged_27x30x50": ((27, 30, 50), 128, "bf16", 64, 2),  # pads to the 480p grid
}


@pytest.mark.parametrize("case", list(CASES))
def test_padded_grid_path_matches_oracle(case):
    grid, d, dtype, topk, heads = CASES[case]
    x = {n: _raster(grid, d, heads, dtype, i) for i, n in enumerate("qkv")}
    e = V.VSA2(1, heads, d, grid, dtype, topk)
    xd = {n: e.to_cube_major(_dev(x[n], dtype)) for n in "qkv"}
    assert xd["q"].shape[2] == e.L and e.L % 64 == 0 and e.L > e.L_real
    N = e.N
    # the router's pooling pass also leaves the coarse branch's Qc, Kc (Eq. 1, over real tokens)
    scores = e.router_scores(xd["q"], xd["k"], coarse_pool=True).cpu().numpy()
    o_sc = np.zeros((1, heads, N, N), np.float32)
    oc_fold = e.coarse_attn(xd["q"], xd["k"], xd["v"], pooled_qk=True)[0].float().cpu().numpy()
    oc_all = e.coarse_attn(xd["q"], xd["k"], xd["v"])[0].float().cpu().numpy()
    sels = []
    for h in range(heads):
        qc, vm = _padded_oracle_inputs(x["q"][0, h], grid, d)
        kc, _ = _padded_oracle_inputs(x["k"][0, h], grid, d)
        vc, _ = _padded_oracle_inputs(x["v"][0, h], grid, d)
        # the permutation: padding rows are zeros, real rows bit-exact
        np.testing.assert_array_equal(xd["q"][0, h].float().cpu().numpy(), qc.astype(np.float32))
        want = O.router_scores_padded(qc, kc, vm)
        g = scores[0, h].astype(np.float64)
        rel = np.linalg.norm(g - want) / np.linalg.norm(want)
        assert rel <= 5e-3 and np.abs(g - want).max() <= 1e-2 * want.max(), (h, rel)
        np.testing.assert_allclose(g.sum(1), 1.0, atol=5e-3)
        o_sc[0, h] = want.astype(np.float32)
        want_c = O.coarse_attn_padded(qc, kc, vc, vm)
        _close(oc_all[0, h], want_c, f"coarse h{h}")
        _close(oc_fold[0, h], want_c, f"coarse, Qc and Kc from the router, h{h}")
        sels.append((qc, kc, vc, vm))
    # TopK over the padded grid's tiles, bit-exact on the oracle's fp32 scores
    kv_off, kv_idx, q_off, q_idx = e.topk_select(torch.from_numpy(o_sc).cuda(), topk, csc=True)
    o, lse = e.attn_fwd(xd["q"], xd["k"], xd["v"], kv_off, kv_idx)
    assert e.device_error() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for h, (qc, kc, vc, vm) in enumerate(sels):
        sel = O.topk_select(o_sc[0, h], topk)
        assert np.array_equal(kv_off[0, h].cpu().numpy(), sel["kv_off"])
        assert np.array_equal(kv_idx[0, h].cpu().numpy(), sel["kv_idx"])
        assert np.array_equal(q_idx[0, h].cpu().numpy(), sel["q_idx"])
        want = O.sparse_attn_fwd_padded(qc, kc, vc, sel["kv_off"], sel["kv_idx"], vm)
        _close(o[0, h][vm], want[vm], f"fine h{h}")
        assert np.all(o[0, h][~vm] == 0) and np.all(np.isneginf(lse[0, h][~vm]))
        assert np.all(np.isfinite(lse[0, h][vm]))


@pytest.mark.parametrize("case", ["6x7x10_bf16", "480p_ragged_27x30x50"])
def test_padded_grid_whole_output_matches_oracle(case):
    """Eq. 14 end to end on the raster grid: permute in, router, TopK, both branches, gated
    merge, permute out (cropped).
    * Against the oracle's exact pieces on the GPU's selection: relative L2 <= 5e-3. (The max
      abs bound is not applied here: both branch outputs are stored in bf16 before the merge
      rounds once more, and above 2 a bf16 half-ulp is already 0.0078; each branch is checked
      against the exact oracle at max abs 2e-2 in the test above.)
    * The merge and the crop composed on the GPU's own branch outputs: max abs <= 2e-2 and
      relative L2 <= 5e-3."""
    grid, d, dtype, topk, heads = CASES[case]
    x = {n: _raster(grid, d, heads, dtype, 10 + i) for i, n in enumerate("qkv")}
    T, H, W = grid
    logits = np.random.default_rng(5).standard_normal((1, heads, T * H * W)).astype(np.float32)
    e = V.VSA2(1, heads, d, grid, dtype, topk)
    xd = {n: e.to_cube_major(_dev(x[n], dtype)) for n in "qkv"}
    # gate logits (X W_g) in the padded cube-major order
    lg_np = np.zeros((1, heads, e.L), np.float32)
    for h in range(heads):
        gp, _ = O.pad_to_tiles(logits[0, h].reshape(T, H, W, 1).astype(np.float64), TILE)
        lg_np[0, h] = O.permute_to_cube_major(gp, TILE, POOL)[:, 0]
    o, _, sel = e.forward(xd["q"], xd["k"], xd["v"])
    oc, _ = e.coarse_attn(xd["q"], xd["k"], xd["v"])
    o_f_gpu, oc_gpu = o.float().cpu().numpy(), oc.float().cpu().numpy()
    out = e.to_raster(e.gated_merge(o, torch.from_numpy(lg_np).cuda(), oc))
    assert e.device_error() == 0
    assert out.shape == (1, heads, T * H * W, d)
    out = out.float().cpu().numpy()
    kv_off, kv_idx = sel[0].cpu().numpy(), sel[1].cpu().numpy()
    for h in range(heads):
        qc, vm = _padded_oracle_inputs(x["q"][0, h], grid, d)
        kc, _ = _padded_oracle_inputs(x["k"][0, h], grid, d)
        vc, _ = _padded_oracle_inputs(x["v"][0, h], grid, d)
        o_f = O.sparse_attn_fwd_padded(qc, kc, vc, kv_off[0, h], kv_idx[0, h], vm)
        o_c = O.coarse_attn_padded(qc, kc, vc, vm)
        merged = O.gated_merge(o_f, o_c, lg_np[0, h])
        want = O.permute_to_raster(merged, e.grid_padded, TILE, POOL)[:T, :H, :W].reshape(-1, d)
        _close(out[0, h], want, f"Eq. 14 h{h}", tol_abs=np.inf)
        comp = O.gated_merge(o_f_gpu[0, h], oc_gpu[0, h], lg_np[0, h])
        want_c = O.permute_to_raster(comp, e.grid_padded, TILE, POOL)[:T, :H, :W].reshape(-1, d)
        _close(out[0, h], want_c, f"merge and crop h{h}")


@pytest.mark.parametrize("case", list(CASES))
def test_padded_grid_backward_matches_oracle(case):
    """Gradients on a grid the tile does not divide, from the GPU's own forward (stored O in the
    dtype and LSE), against the oracle's padded backward given the same stored O (the backward
    forms rowsum(dO * O) from the O it receives): padding keys take no part, the outputs of
    padding rows are dropped (dout there is noise and must not matter), and the gradients of
    padding tokens are exactly 0. The selection is the GPU's own (router, TopK)."""
    grid, d, dtype, topk, heads = CASES[case]
    x = {n: _raster(grid, d, heads, dtype, 20 + i) for i, n in enumerate("qkv")}
    e = V.VSA2(1, heads, d, grid, dtype, topk)
    xd = {n: e.to_cube_major(_dev(x[n], dtype)) for n in "qkv"}
    rng = np.random.default_rng(7)
    sels = [tuple(_padded_oracle_inputs(x[n][0, h], grid, d) for n in "qkv") for h in range(heads)]
    vm = sels[0][0][1]
    do_np = rng.standard_normal((1, heads, e.L, d)).astype(np.float32)
    do_np[:, :, ~vm] = 50.0 * rng.standard_normal((1, heads, int((~vm).sum()), d))  # must not matter
    do_np = S.round_to_dtype(do_np, dtype)
    do = _dev(do_np, dtype)
    o, lse, sel = e.forward(xd["q"], xd["k"], xd["v"], csc=True)
    dq, dk, dv = e.attn_bwd(xd["q"], xd["k"], xd["v"], o, lse, do, *sel)
    assert e.device_error() == 0
    kv_off, kv_idx = sel[0].cpu().numpy(), sel[1].cpu().numpy()
    got = [g.cpu().numpy() for g in (dq, dk, dv)]
    o_np = o.float().cpu().numpy()
    for h in range(heads):
        (qc, vmh), (kc, _), (vc, _) = sels[h]
        want = O.sparse_attn_bwd_padded(qc, kc, vc, do_np[0, h], kv_off[0, h], kv_idx[0, h], vmh, o=o_np[0, h])
        for name, g, w in zip(("dq", "dk", "dv"), got, want):
            assert np.all(g[0, h][~vmh] == 0), f"{name} h{h}: padding tokens"
            _close(g[0, h][vmh], w[vmh], f"{name} h{h}")


@pytest.mark.parametrize("case", ["6x7x10_bf16", "6x7x10_fp32_d64", "480p_ragged_27x30x50"])
def test_padded_grid_coarse_and_merge_backward_match_oracle(case):
    """Gradients of the coarse branch (Eq. 1-3, means over real tokens) and of the gated merge on
    a padded grid against the oracle's padded backward; d_oc comes from the merge backward, whose
    dout is noise on padding rows. Inputs are tile-constant (as in the whole-tile coarse backward
    tests), so the GPU's pooled operands, rounded to the dtype, equal the oracle's exactly."""
    grid, d, dtype, topk, heads = CASES[case]
    # tile-constant inputs with dtype-exact tile values: every real token of a tile holds the
    # tile's vector, so both sides pool to the same (representable) operands
    T, H, W = grid
    rng = np.random.default_rng(8)
    tgrid = tuple(-(-g // 4) for g in grid)
    t, hh, w = np.meshgrid(np.arange(T) // 4, np.arange(H) // 4, np.arange(W) // 4, indexing="ij")
    tile_of = ((t * tgrid[1] + hh) * tgrid[2] + w).reshape(-1)
    x = {}
    for n in "qkv":
        vals = S.round_to_dtype(rng.standard_normal((heads, int(np.prod(tgrid)), d)).astype(np.float32), dtype)
        x[n] = vals[:, tile_of][None].astype(np.float32)
    e = V.VSA2(1, heads, d, grid, dtype, topk)
    xd = {n: e.to_cube_major(_dev(x[n], dtype)) for n in "qkv"}
    vm = _padded_oracle_inputs(x["q"][0, 0], grid, d)[1]
    do_np = rng.standard_normal((1, heads, e.L, d)).astype(np.float32)
    do_np[:, :, ~vm] = 50.0 * rng.standard_normal((1, heads, int((~vm).sum()), d))
    do_np = S.round_to_dtype(do_np, dtype)
    logits = rng.standard_normal((1, heads, e.L)).astype(np.float32)
    oc, lse_c = e.coarse_attn(xd["q"], xd["k"], xd["v"])
    d_logits, d_oc = e.gated_merge_bwd(_dev(do_np, dtype), torch.from_numpy(logits).cuda(), oc)
    grads = [torch.zeros(1, heads, e.L, d, dtype=torch.float32, device="cuda") for _ in range(3)]
    e.coarse_attn_bwd(xd["q"], xd["k"], xd["v"], oc, lse_c, d_oc, *grads)
    assert e.device_error() == 0
    oc_np, d_logits, d_oc_np = oc.float().cpu().numpy(), d_logits.cpu().numpy(), d_oc.cpu().numpy()
    got = [g.cpu().numpy() for g in grads]
    for h in range(heads):
        qc, _ = _padded_oracle_inputs(x["q"][0, h], grid, d)
        kc, _ = _padded_oracle_inputs(x["k"][0, h], grid, d)
        vc, _ = _padded_oracle_inputs(x["v"][0, h], grid, d)
        _, w_doc, w_dlog = O.gated_merge_bwd_padded(do_np[0, h], oc_np[0, h], logits[0, h], vm)
        _close(d_oc_np[0, h], w_doc, f"d_oc h{h}")
        assert np.all(d_logits[0, h][~vm] == 0)
        _close(d_logits[0, h][vm], w_dlog[vm], f"d_logits h{h}")
        # the coarse backward takes d_oc rounded to the dtype (its tensor-core operand)
        d_oc_in = S.round_to_dtype(d_oc_np[0, h], dtype)
        want = O.coarse_attn_bwd_padded(qc, kc, vc, d_oc_in, vm, o_c_hat=oc_np[0, h])
        for name, g, w in zip(("dq", "dk", "dv"), got, want):
            assert np.all(g[0, h][~vm] == 0), f"coarse {name} h{h}: padding tokens"
            _close(g[0, h][vm], w[vm], f"coarse {name} h{h}")
