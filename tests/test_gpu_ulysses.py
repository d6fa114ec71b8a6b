"""Ulysses resharding (App. E of "Improving Video Sparse Attention with Fine-grained Router and
Sparse Rebasing") on a GPU over NCCL, around the real VSA2 engine.

One NCCL rank on one GPU: the two all-to-alls then move every element to itself, so the output
and the gradients through `ulysses_attention` must equal the direct `vsa2_attention` call bit
for bit. This runs the NCCL path of `seq_to_heads` / `heads_to_seq` with CUDA tensors, in their
forward and backward directions, around the kernels of the whole Eq. 14 output. (The exchange
with 2 and 4 ranks is checked on CPU with gloo in tests/test_ulysses_gloo.py.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(port, out):
    import datetime

    import torch.distributed as dist

    import synthetic as S
    import trainable_block_sparse_fine_b200 as V

    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        wl = S.Workload("ulysses", 1, 4, 128, (8, 16, 40), 6, "bf16")  # N = 80 tiles per head
        x = {n: torch.from_numpy(S.make_tensor(wl, n)).cuda().to(torch.bfloat16) for n in ("q", "k", "v", "do")}
        g = torch.randn(1, wl.heads, wl.tokens, generator=torch.Generator().manual_seed(5)).cuda()
        e = V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk)

        def run(through_ulysses):
            t = {n: x[n].clone().requires_grad_(True) for n in ("q", "k", "v")}
            gl = g.clone().requires_grad_(True)
            fn = lambda q, k, v, gg: V.vsa2_attention(q, k, v, gg, e)
            o = V.ulysses_attention(fn, [t["q"], t["k"], t["v"], gl]) if through_ulysses else fn(t["q"], t["k"], t["v"], gl)
            o.backward(x["do"])
            torch.cuda.synchronize()
            return [a.detach().float().cpu().numpy() for a in (o, t["q"].grad, t["k"].grad, t["v"].grad, gl.grad)]

        out["direct"] = run(False)
        out["ulysses"] = run(True)
        out["err"] = e.device_error()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ulysses_nccl_one_rank_equals_direct_call():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    p = ctx.Process(target=_worker, args=(_free_port(), out))
    p.start()
    p.join(timeout=300)
    assert p.exitcode == 0
    assert out["err"] == 0
    for name, a, b in zip(("o", "dq", "dk", "dv", "d_logits"), out["direct"], out["ulysses"]):
        assert np.array_equal(a, b), name
        assert np.isfinite(a).all(), name
