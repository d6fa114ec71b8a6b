"""Host-side multi-rank logic on CPU: world size 2 over gloo (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from trainable_block_sparse_fine_b200.sharding import shard_units


@pytest.mark.parametrize("batch,heads,world", [(1, 20, 2), (1, 20, 8), (2, 3, 4), (1, 1, 2), (3, 7, 5)])
def test_shards_cover_every_unit_once(batch, heads, world):
    seen = [u for r in range(world) for u in shard_units(batch, heads, r, world)]
    assert sorted(seen) == [(b, h) for b in range(batch) for h in range(heads)]
    sizes = [len(shard_units(batch, heads, r, world)) for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from trainable_block_sparse_fine_b200.sharding import max_over_ranks, shard_units

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard_units(1, 20, rank, world)
        # every rank times its own shard; the job time is the slowest rank
        local_ms = 10.0 + rank * 2.5
        out[rank] = (len(mine), max_over_ranks(local_ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_timing_max_and_shards():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert sorted(out.keys()) == [0, 1]
    assert sum(out[r][0] for r in range(world)) == 20
    assert all(out[r][1] == 12.5 for r in range(world))
