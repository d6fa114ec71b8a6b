"""Ulysses resharding (sequence shards <-> head shards) with gloo ranks on CPU.

Each rank holds a contiguous shard of the cube-major tokens of every head. Through
`ulysses_attention` it runs the whole per-head VSA2 attention (router, per-sequence TopK, fine
branch, coarse branch, gated merge; the oracle stands in for the kernels here) and gets its
shard of the output back. That shard must equal the single-process result on the full tensors,
and the gradient of the resharding must be the inverse resharding of the upstream gradient.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

B, H, GRID, D, TOPK = 1, 4, (8, 8, 16), 8, 3
L = GRID[0] * GRID[1] * GRID[2]


def _inputs():
    rng = np.random.default_rng(91)
    q, k, v = (torch.from_numpy(rng.standard_normal((B, H, L, D))) for _ in range(3))
    g = torch.from_numpy(rng.standard_normal((B, H, L)))
    w = torch.from_numpy(rng.standard_normal((B, H, L, D)))
    return q, k, v, g, w


def _vsa2_heads(q, k, v, g):
    """Eq. 1-14 per head with the fp64 oracle: [B, h, L, D] x3 and [B, h, L] -> [B, h, L, D]."""
    from oracle import vsa2_oracle as O

    out = torch.empty(q.shape, dtype=torch.float64)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            qh, kh, vh = (t[b, h].detach().numpy() for t in (q, k, v))
            sel = O.topk_select(O.router_scores(qh, kh).astype(np.float32), TOPK)
            o_f, _ = O.sparse_attn_fwd(qh, kh, vh, sel["kv_off"], sel["kv_idx"])
            o_c, _ = O.coarse_attn(qh, kh, vh)
            out[b, h] = torch.from_numpy(O.gated_merge(o_f, o_c, g[b, h].detach().numpy()))
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    from trainable_block_sparse_fine_b200.ulysses import heads_to_seq, seq_to_heads, ulysses_attention

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, g, w = _inputs()
        s = slice(rank * L // world, (rank + 1) * L // world)
        o = ulysses_attention(_vsa2_heads, [q[:, :, s], k[:, :, s], v[:, :, s], g[:, :, s]])
        # gradient of the regrouping: a loss on the head-grouped tensor
        x = q[:, :, s].clone().requires_grad_(True)
        hg = H // world
        y = seq_to_heads(x)
        (y * w[:, rank * hg:(rank + 1) * hg]).sum().backward()
        back = heads_to_seq(seq_to_heads(q[:, :, s]))
        out[rank] = (o.numpy(), x.grad.numpy(), y.detach().numpy(), back.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_matches_single_process(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    q, k, v, g, w = _inputs()
    full = _vsa2_heads(q, k, v, g).numpy()
    hg = H // world
    for r in range(world):
        s = slice(r * L // world, (r + 1) * L // world)
        o, grad, y, back = out[r]
        np.testing.assert_array_equal(o, full[:, :, s])
        np.testing.assert_array_equal(y, q[:, r * hg:(r + 1) * hg].numpy())  # head group r, whole sequence
        np.testing.assert_array_equal(grad, w[:, :, s].numpy())  # the adjoint is the inverse regrouping
        np.testing.assert_array_equal(back, q[:, :, s].numpy())
