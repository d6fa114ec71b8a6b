"""The token permutation (§2.2 "Permutation") on the GPU, raster <-> cube-major, against the
oracle's loop construction of the order. It is a copy, so the comparison is bit-exact, in both
directions, for the default 4x4x4 tiles with 2x2x4 sub-cubes and for another tile and pool
shape, in bf16 and fp32, at D = 64 and 128 (three chunk counts per row)."""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from trainable_block_sparse_fine_b200 import _capi as C

# (batch, heads, D, grid, tile, pool, dtype, heads compared against the oracle)
CASES = {
    "bf16_d128": (1, 2, 128, (8, 16, 20), (4, 4, 4), (2, 2, 4), "bf16", None),
    "fp32_d64_other_shape": (2, 1, 64, (4, 8, 16), (2, 4, 8), (1, 2, 8), "fp32", None),
    "bf16_d64": (1, 3, 64, (12, 12, 8), (4, 4, 4), (2, 2, 4), "bf16", None),
    "fp32_d128": (1, 1, 128, (8, 8, 8), (4, 4, 4), (2, 2, 4), "fp32", None),
    "480p_20_heads": (1, 20, 128, (28, 32, 52), (4, 4, 4), (2, 2, 4), "bf16", (0, 19)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_permutation_matches_oracle_both_ways(case):
    B, H, D, grid, tile, pool, dtype, compared = CASES[case]
    L = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(51)
    x = S.round_to_dtype(rng.standard_normal((B, H, *grid, D)).astype(np.float32), dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    src = torch.from_numpy(x.reshape(B, H, L, D)).cuda().to(tdt)
    cube = torch.empty_like(src)
    back = torch.empty_like(src)
    p = C.make_problem(B, H, D, grid, dtype, tile=tile, pool=pool)
    C.vsa2_permute_tokens(p, src, cube, True)
    C.vsa2_permute_tokens(p, cube, back, False)
    torch.cuda.synchronize()
    assert torch.equal(back, src), "raster -> cube-major -> raster is not the identity"
    got = cube.float().cpu().numpy()
    for b in range(B):
        for h in (range(H) if compared is None else compared):
            np.testing.assert_array_equal(got[b, h], O.permute_to_cube_major(x[b, h], tile, pool), err_msg=f"[{b},{h}]")


def test_permutation_rejects_in_place():
    p = C.make_problem(1, 1, 64, (8, 8, 8))
    t = torch.zeros(1, 1, 512, 64, device="cuda")
    with pytest.raises(C.Vsa2Error):
        C.vsa2_permute_tokens(p, t, t, True)
