"""A model of the forward kernel's per-slot pipeline and its mbarriers, run under random
schedules on the CPU.

An mbarrier parity wait can only tell the phase in progress from the one just completed: a
waiter two phases behind waits forever, and a waiter one phase ahead passes early. The model
checks, at every poll, that the awaited phase is one of those two, and that every schedule
finishes (no deadlock). The agents follow the kernel's protocol:
  * the producer walks the slot's ops (S0, S1, O0, S2, O1, ... per query tile) and loads K for an
    S op and V for an O op into ring position c % RST, after the release of position c - RST;
  * the MMA issuer waits for the block in the ring, and for an S op also for the S buffer
    (two buffers, freed by the softmax), for an O op also for P (written by the softmax); the
    MMA's completion releases the ring position and signals S (sfull) or P.V done (pvdone);
  * the softmax waits for S, frees its buffer, then waits for the previous P.V before writing P.
The kernel's variant is one producer per slot and a 3-block ring holding K and V in op order.
The model also covers the planned split with two producers (one per d-half, the full barrier
expecting two arrivals).
"""
import random

import pytest


class Barrier:
    def __init__(self, count):
        self.count, self.arrived, self.phases = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.phases += 1

    def poll(self, phase, who):
        """A parity wait for the completion of `phase` (phase -1: a fresh barrier's preceding
        phase). Valid only while `phase` is in progress or has just completed."""
        assert phase - 1 <= self.phases - 1 <= phase, f"{who}: waits for phase {phase}, {self.phases} completed"
        return self.phases >= phase + 1


def ops_of(tiles):
    """The slot's op stream: for a tile of n blocks, S0, S1, O0, S2, O1, ..., O(n-1)."""
    out = []
    for n in tiles:
        s = o = 0
        while o < n:
            if s < n and s <= o + 1:
                out.append(("S", s))
                s += 1
            else:
                out.append(("O", o))
                o += 1
    return out


def run(tiles, rst, producers, rng, mma_latency=3):
    ops = ops_of(tiles)
    full = [Barrier(producers) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    sfull, sfree = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    pfull, pvdone = Barrier(1), Barrier(1)
    prod = [0] * producers            # next ring position per producer
    mma = {"c": 0, "s": 0, "o": 0}    # next op; S and O ops issued
    soft = {"blk": 0, "step": 0}      # next block; 0: wait S, 1: wait previous P.V, then write P
    nblk = sum(tiles)
    pending = []                      # (time, callback): MMA completions
    t = 0

    def producer(p):
        c = prod[p]
        if c >= len(ops):
            return False
        st = c % rst
        if not empty[st].poll(c // rst - 1, f"producer {p} at {c}"):
            return False
        full[st].arrive()
        prod[p] += 1
        return True

    def issuer():
        c = mma["c"]
        if c >= len(ops):
            return False
        st = c % rst
        if not full[st].poll(c // rst, f"issuer at {c}"):
            return False
        kind, _ = ops[c]
        if kind == "S":
            k = mma["s"]
            if not sfree[k % 2].poll(k // 2 - 1, f"issuer S{k}"):
                return False
            done = [empty[st].arrive, sfull[k % 2].arrive]
            mma["s"] += 1
        else:
            k = mma["o"]
            if not pfull.poll(k, f"issuer O{k}"):
                return False
            done = [empty[st].arrive, pvdone.arrive]
            mma["o"] += 1
        pending.append((t + rng.randint(1, mma_latency), done))
        mma["c"] += 1
        return True

    def softmax():
        g = soft["blk"]
        if g >= nblk:
            return False
        if soft["step"] == 0:
            if not sfull[g % 2].poll(g // 2, f"softmax S{g}"):
                return False
            sfree[g % 2].arrive()
            soft["step"] = 1
            return True
        if g > 0 and not pvdone.poll(g - 1, f"softmax P{g}"):
            return False
        pfull.arrive()
        soft["blk"], soft["step"] = g + 1, 0
        return True

    agents = [lambda p=p: producer(p) for p in range(producers)] + [issuer, softmax]
    while mma["c"] < len(ops) or soft["blk"] < nblk or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            for f in done:
                f()
        moved = bool(due)
        for a in rng.sample(agents, len(agents)):
            if rng.random() < 0.7:
                moved |= a()
        assert moved or pending or t < 10_000_000, "deadlock"
        if not moved and not pending and not any(a() for a in agents):
            raise AssertionError(f"deadlock at op {mma['c']} of {len(ops)}, softmax block {soft['blk']}")
    assert pvdone.phases == sum(tiles) and all(p == len(ops) for p in prod)


@pytest.mark.parametrize("producers", [1, 2], ids=["kernel", "two_producers"])
@pytest.mark.parametrize("seed", range(30))
def test_ring_protocol_parity_and_progress(producers, seed):
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run(tiles, rst=3, producers=producers, rng=rng, mma_latency=rng.choice([1, 3, 10]))


def test_op_order_matches_the_kernel_stream():
    assert ops_of([3]) == [("S", 0), ("S", 1), ("O", 0), ("S", 2), ("O", 1), ("O", 2)]
    assert ops_of([1, 2]) == [("S", 0), ("O", 0), ("S", 0), ("S", 1), ("O", 0), ("O", 1)]
