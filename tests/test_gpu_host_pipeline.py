"""The host-buffer entry point vsa2_forward_host.

It cuts the flat (b, h) range into groups and overlaps each group's PCIe copies with the
kernels of its neighbours. The checks are:
  * its O and LSE are bit-identical to the device-buffer calls (router -> TopK -> forward) on
    the same inputs, for automatic, one-head and ragged groups that cross a batch boundary
    and reuse every staging slot;
  * they hold with pageable host memory too;
  * its O matches the fp64 oracle's attention on the selection the device path made (the
    selection's own parity is covered by the TopK tests).
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import vsa2_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import trainable_block_sparse_fine_b200 as V

# batch 2 x heads 3: groups of 4 flat heads cross the batch boundary, groups of 1 reuse each of
# the three staging slots twice
WL = S.Workload("host_pipeline", 2, 3, 128, (8, 16, 20), 6, "bf16")  # N = 40


def _host_inputs(pin):
    x = {n: torch.from_numpy(S.make_tensor(WL, n)).to(torch.bfloat16) for n in "qkv"}
    return {n: (t.pin_memory() if pin else t) for n, t in x.items()}


def _device_reference(e, x):
    xd = {n: t.cuda() for n, t in x.items()}
    o, lse, sel = e.forward(xd["q"], xd["k"], xd["v"], WL.topk)
    return o.cpu(), lse.cpu(), sel


@pytest.mark.parametrize("pin", [True, False], ids=["pinned", "pageable"])
@pytest.mark.parametrize("per", [0, 1, 4], ids=["auto", "one_head", "ragged"])
def test_host_forward_is_bit_identical_to_device_calls(per, pin):
    e = V.VSA2(WL.batch, WL.heads, WL.head_dim, WL.grid, WL.dtype, WL.topk)
    x = _host_inputs(pin)
    want_o, want_lse, _ = _device_reference(e, x)
    for call in range(2):  # the second call reuses the workspace and the library's streams
        o, lse = e.forward_host(x["q"], x["k"], x["v"], heads_per_group=per, want_lse=True)
        torch.cuda.current_stream().synchronize()
        assert not o.is_cuda and not lse.is_cuda
        assert torch.equal(o, want_o), f"call {call}: O differs"
        assert torch.equal(lse, want_lse), f"call {call}: LSE differs"
    assert e.device_error() == 0


def test_host_forward_matches_oracle_on_its_selection():
    e = V.VSA2(WL.batch, WL.heads, WL.head_dim, WL.grid, WL.dtype, WL.topk)
    x = _host_inputs(True)
    _, _, sel = _device_reference(e, x)
    o, _ = e.forward_host(x["q"], x["k"], x["v"], heads_per_group=1)
    torch.cuda.current_stream().synchronize()
    assert e.device_error() == 0
    o = o.float().numpy()
    kv_off, kv_idx = sel[0].cpu().numpy(), sel[1].cpu().numpy()
    xf = {n: t.float().numpy() for n, t in x.items()}  # the bf16 values both sides compute on
    for b in range(WL.batch):
        for h in range(WL.heads):
            want, _ = O.sparse_attn_fwd(xf["q"][b, h], xf["k"][b, h], xf["v"][b, h], kv_off[b, h], kv_idx[b, h])
            err = np.abs(o[b, h] - want)
            rel = np.linalg.norm(o[b, h] - want) / np.linalg.norm(want)
            assert err.max() <= 2e-2 and rel <= 5e-3, f"o[{b},{h}]: max abs {err.max():.3e}, rel L2 {rel:.3e}"


def test_host_forward_rejects_device_tensors():
    e = V.VSA2(WL.batch, WL.heads, WL.head_dim, WL.grid, WL.dtype, WL.topk)
    q = torch.zeros(WL.batch, WL.heads, WL.tokens, WL.head_dim, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        e.forward_host(q, q, q)
