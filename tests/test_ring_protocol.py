"""Models of the tensor-core kernels' pipelines (forward, dQ and dK/dV) with their mbarriers,
run under random schedules on the CPU.

An mbarrier parity wait can only tell the phase in progress from the one just completed: a
waiter two phases behind waits forever, and a waiter one phase ahead passes early. The model
checks, at every poll, that the awaited phase is one of those two, and that every schedule
finishes (no deadlock). The agents follow the kernel's protocol:
  * the producer walks the slot's ops (S0, S1, O0, S2, O1, ... per query tile: S runs one block
    ahead of O; the model also checks a lead of two, S0, S1, S2, O0, S3, O1, ...) and loads K for
    an S op and V for an O op into ring position c % RST, after the release of position c - RST;
  * the MMA issuer waits for the block in the ring, and for an S op also for the S buffer
    (two buffers, freed by the softmax), for an O op also for P (written by the softmax); the
    MMA's completion releases the ring position and signals S (sfull) or P.V done (pvdone);
  * the softmax waits for S, frees its buffer, then waits for the previous P.V before writing P.
The kernel's variant is one producer per slot and a 3-block ring holding K and V in op order.
The model also covers the planned split with two producers (one per d-half, the full barrier
expecting two arrivals). Besides the barrier rules it asserts the data hazards the barriers
exist for: a ring block, an S buffer or P is overwritten only after its last reader finished.
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


def ops_of(tiles, lead=1):
    """The slot's op stream: for a tile of n blocks, S(k) goes before O(k - lead); the kernel's
    lead is 1 (S0, S1, O0, S2, O1, ..., O(n-1)). A lead of 2 (S0, S1, S2, O0, S3, O1, ...) is
    safe too with two S buffers; measured, it was slower (late K blocks held the O ops back)."""
    out = []
    for n in tiles:
        s = o = 0
        while o < n:
            if s < n and s <= o + lead:
                out.append(("S", s))
                s += 1
            else:
                out.append(("O", o))
                o += 1
    return out


def run(tiles, rst, producers, rng, mma_latency=3, lead=1):
    ops = ops_of(tiles, lead)
    full = [Barrier(producers) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    sfull, sfree = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    pfull, pvdone = Barrier(1), Barrier(1)
    prod = [0] * producers            # next ring position per producer
    mma = {"c": 0, "s": 0, "o": 0}    # next op; S and O ops issued
    soft = {"blk": 0, "step": 0}      # next block; 0: wait S, 1: wait previous P.V, then write P
    op_done = set()                   # ring positions whose MMA has completed
    s_read = set()                    # S blocks the softmax has read
    o_done = set()                    # P.V blocks completed
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
        assert c < rst or c - rst in op_done, f"ring position {c} refilled before its MMA finished"
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
            assert k < 2 or k - 2 in s_read, f"S buffer of block {k} overwritten before it was read"
            done = [lambda c=c: op_done.add(c), empty[st].arrive, sfull[k % 2].arrive]
            mma["s"] += 1
        else:
            k = mma["o"]
            if not pfull.poll(k, f"issuer O{k}"):
                return False
            done = [lambda c=c, k=k: (op_done.add(c), o_done.add(k)), empty[st].arrive, pvdone.arrive]
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
            s_read.add(g)
            sfree[g % 2].arrive()
            soft["step"] = 1
            return True
        if g > 0 and not pvdone.poll(g - 1, f"softmax P{g}"):
            return False
        assert g == 0 or g - 1 in o_done, f"P of block {g} written while P.V of block {g - 1} reads P"
        pfull.arrive()
        soft["blk"], soft["step"] = g + 1, 0
        return True

    agents = [lambda p=p: producer(p) for p in range(producers)] + [issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]  # skewed speeds expose races
    while mma["c"] < len(ops) or soft["blk"] < nblk or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            for f in done:
                f()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        assert moved or pending or t < 10_000_000, "deadlock"
        if not moved and not pending and not any(a() for a in agents):
            raise AssertionError(f"deadlock at op {mma['c']} of {len(ops)}, softmax block {soft['blk']}")
    assert pvdone.phases == sum(tiles) and all(p == len(ops) for p in prod)


def run_aliased(tiles, rst, rng, mma_latency=3, rescale_p=0.2, lead=1):
    """The forward kernel's protocol with P written over the S buffer it came from: per slot two
    S/P buffers, pfull and pvdone per block parity, no wait for the previous P.V before writing P;
    the softmax waits for the previous P.V only to rescale O (at random here) and at a tile's end.
    The tensor pipe completes MMAs in issue order. Asserts, besides the parity rule, that S(k)
    overwrites a buffer only after O(k-2) read its P, that P(g) is written only after O(g-2)
    read the previous P of the buffer, and that O is read only after every P.V issued before."""
    ops = ops_of(tiles, lead=lead)
    full = [Barrier(1) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    sfull, sfree = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    pfull, pvdone = [Barrier(4), Barrier(4)], [Barrier(1), Barrier(1)]
    for b in pfull:
        b.count = 1  # one arrival stands for the four softmax warps
    prod = {"c": 0}
    mma = {"c": 0, "s": 0, "o": 0}
    soft = {"blk": 0, "step": 0, "tile": 0, "in_tile": 0}
    done = {"op": set(), "s": set(), "o": set()}
    p_written = set()
    ends = []                      # block index that ends each tile
    acc = 0
    for n in tiles:
        acc += n
        ends.append(acc - 1)
    nblk = acc
    pipe = {"last": 0}
    pending = []
    t = 0

    def producer():
        c = prod["c"]
        if c >= len(ops):
            return False
        st = c % rst
        if not empty[st].poll(c // rst - 1, f"producer at {c}"):
            return False
        assert c < rst or c - rst in done["op"], f"ring position {c} refilled before its MMA finished"
        full[st].arrive()
        prod["c"] += 1
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

            def fin(c=c, k=k, st=st):
                assert k < 2 or k - 2 in done["o"], f"S{k} overwrote P{k - 2} before O{k - 2} read it"
                done["op"].add(c)
                done["s"].add(k)
                empty[st].arrive()
                sfull[k % 2].arrive()
            mma["s"] += 1
        else:
            k = mma["o"]
            if not pfull[k % 2].poll(k // 2, f"issuer O{k}"):
                return False
            assert k in p_written

            def fin(c=c, k=k, st=st):
                done["op"].add(c)
                done["o"].add(k)
                empty[st].arrive()
                pvdone[k % 2].arrive()
            mma["o"] += 1
        pipe["last"] = max(pipe["last"], t) + rng.randint(1, mma_latency)  # in order
        pending.append((pipe["last"], fin))
        mma["c"] += 1
        return True

    def wait_pv(g, who):
        return pvdone[g % 2].poll(g // 2, who)

    def softmax():
        g = soft["blk"]
        if g >= nblk:
            return False
        st = soft["step"]
        if st == 0:                       # wait S, read it, free the buffer
            if not sfull[g % 2].poll(g // 2, f"softmax S{g}"):
                return False
            assert g in done["s"]
            sfree[g % 2].arrive()
            first = g == 0 or (g - 1) in ends
            soft["step"] = 1 if (not first and rng.random() < rescale_p) else 2
            return True
        if st == 1:                       # rescale O: the previous P.V must be done
            if not wait_pv(g - 1, f"softmax rescale at {g}"):
                return False
            assert all(x in done["o"] for x in range(g)), f"O read at block {g} with a P.V pending"
            soft["step"] = 2
            return True
        if st == 2:                       # write P over the S buffer
            assert g < 2 or g - 2 in done["o"], f"P{g} written before O{g - 2} read P{g - 2}"
            p_written.add(g)
            pfull[g % 2].arrive()
            soft["step"] = 3 if g in ends else 0
            if g not in ends:
                soft["blk"] = g + 1
            return True
        if not wait_pv(g, f"softmax epilogue at {g}"):  # st == 3: tile's last P.V, then O
            return False
        assert all(x in done["o"] for x in range(g + 1)), f"epilogue at {g} with a P.V pending"
        soft["blk"], soft["step"] = g + 1, 0
        return True

    agents = [producer, issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while mma["c"] < len(ops) or soft["blk"] < nblk or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, f in sorted(due, key=lambda x: x[0]):
            f()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(a() for a in agents):
            raise AssertionError(f"deadlock at op {mma['c']} of {len(ops)}, softmax block {soft['blk']}")
    assert len(done["o"]) == nblk


@pytest.mark.parametrize("seed", range(80))
def test_forward_protocol_with_p_over_s(seed):
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run_aliased(tiles, rst=3, rng=rng, mma_latency=rng.choice([1, 3, 10, 30]))


def test_forward_protocol_flags_a_single_pfull_barrier():
    """With one pfull barrier instead of one per block parity, the softmax can complete the
    phase of block n+1 before the issuer waited for block n's: the parity rule flags it."""
    with pytest.raises(AssertionError):
        for seed in range(200):
            _run_single_pfull([32, 32, 5], random.Random(seed))


def test_forward_protocol_flags_lead_two_with_p_over_s():
    """S two blocks ahead would overwrite P(k-2) before O(k-2) read it: the model flags it."""
    with pytest.raises(AssertionError):
        for seed in range(50):
            run_aliased([32, 7], rst=3, rng=random.Random(seed), mma_latency=10, lead=2)


def _run_single_pfull(tiles, rng):
    """The kernel's earlier single pfull barrier (count: one per block), with P over S and no
    wait for the previous P.V before writing P."""
    ops = ops_of(tiles, lead=1)
    pf = Barrier(1)
    s_done = set()
    mma_o = 0
    soft_g = 0
    nblk = sum(tiles)
    issued_s = 0
    t = 0
    # a minimal schedule: S ops complete at once; the issuer is slow, the softmax fast
    while soft_g < nblk:
        t += 1
        if issued_s < nblk and issued_s <= mma_o + 1:
            s_done.add(issued_s)
            issued_s += 1
        if soft_g in s_done and rng.random() < 0.9:
            pf.arrive()
            soft_g += 1
        if rng.random() < 0.05 and mma_o < soft_g:
            if pf.poll(mma_o, f"issuer O{mma_o}"):
                mma_o += 1
    return True


@pytest.mark.parametrize("lead", [1, 2], ids=["kernel", "lead2"])
@pytest.mark.parametrize("producers", [1, 2], ids=["one_producer", "two_producers"])
@pytest.mark.parametrize("seed", range(60))
def test_ring_protocol_parity_and_progress(lead, producers, seed):
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run(tiles, rst=3, producers=producers, rng=rng, mma_latency=rng.choice([1, 3, 10]), lead=lead)


def test_op_order_matches_the_kernel_stream():
    assert ops_of([3]) == [("S", 0), ("S", 1), ("O", 0), ("S", 2), ("O", 1), ("O", 2)]
    assert ops_of([1, 2]) == [("S", 0), ("O", 0), ("S", 0), ("S", 1), ("O", 0), ("O", 1)]
    assert ops_of([4], lead=2) == [("S", 0), ("S", 1), ("S", 2), ("O", 0), ("S", 3), ("O", 1), ("O", 2), ("O", 3)]



def run_dkdv(items, rng, rst=6, mma_latency=3):
    """The dK/dV kernel's protocol: per KV tile (item) of n selecting query tiles, op t loads the
    tile's Q / dO stage (producer of the position's parity), the first issuer runs S^T / dP^T
    into the single S buffer, the softmax reads it and writes P / dS into buffer t % 2, the
    second issuer runs dV / dK from that buffer and releases the stage; after the item's last op
    the epilogue waits for every MMA, then the next item's K / V rows go to tensor memory. A KV
    tile that no query tile selected touches no barrier; the per-item phases count non-empty
    items only, as the kernel's do. Data hazards asserted: a stage is refilled only after both
    MMAs and the softmax have read it; S only after the softmax read it; a P / dS buffer only
    after the second MMA two ops back; the K / V rows only after the previous item's MMAs; the
    accumulators are restarted only after the previous item's epilogue."""
    total = sum(items)
    full = [Barrier(1) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    spfull, spfree = Barrier(1), Barrier(1)
    pdsfull, pdsfree = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    itemdone, kvready = Barrier(1), Barrier(1)
    last_of_item = set()
    n = 0
    for k in items:
        n += k
        last_of_item.add(n - 1)
    nonempty = [i for i, k in enumerate(items) if k]
    item_of = [j for j, i in enumerate(nonempty) for _ in range(items[i])]  # non-empty index per op
    prod = [0, 1]                   # producer p fills positions p, p + 2, ...
    a = {"n": 0}
    b = {"n": 0}
    soft = {"item": 0, "it": 0, "n": 0, "step": "kv"}  # item, non-empty items done, op, stage
    a_done, b_done, s_read = set(), set(), set()  # completed first / second MMAs, S blocks read
    epi_done = set()                              # non-empty items whose epilogue has run
    first_op = {sum(items[i] for i in nonempty[:j]): j for j in range(len(nonempty))}
    pending = []
    t = 0

    def producer(p):
        pos = prod[p]
        if pos >= total:
            return False
        st = pos % rst
        if not empty[st].poll(pos // rst - 1, f"producer {p} at {pos}"):
            return False
        old = pos - rst
        assert old < 0 or (old in a_done and old in b_done and old in s_read), f"stage refilled at {pos}"
        full[st].arrive()
        prod[p] += 2
        return True

    def issuer_a():
        c = a["n"]
        if c >= total:
            return False
        first_of_item = c == 0 or (c - 1) in last_of_item
        if first_of_item and not kvready.poll(item_of[c], f"issuer A kv {c}"):
            return False
        if c > 0 and not spfree.poll(c - 1, f"issuer A S {c}"):
            return False
        if not full[c % rst].poll(c // rst, f"issuer A stage {c}"):
            return False
        assert c == 0 or c - 1 in s_read, f"S of op {c} overwrites S of op {c - 1} before it was read"
        pending.append((t + rng.randint(1, mma_latency), [lambda c=c: a_done.add(c), spfull.arrive]))
        a["n"] += 1
        return True

    def issuer_b():
        c = b["n"]
        if c >= total:
            return False
        if not pdsfull[c & 1].poll(c >> 1, f"issuer B {c}"):
            return False
        if c in first_op and first_op[c] > 0:
            assert first_op[c] - 1 in epi_done, f"accumulators restarted at op {c} before the epilogue read them"
        done = [lambda c=c: b_done.add(c), empty[c % rst].arrive, pdsfree[c & 1].arrive]
        if c in last_of_item:
            done.append(itemdone.arrive)
        pending.append((t + rng.randint(1, mma_latency), done))
        b["n"] += 1
        return True

    def softmax():
        if soft["item"] >= len(items):
            return False
        c = soft["n"]
        if soft["step"] == "kv":  # K / V rows of the item into tensor memory
            if items[soft["item"]] == 0:  # zero gradients, no barrier
                soft["item"] += 1
                return True
            prev = [c2 for c2 in range(c) if item_of[c2] == soft["it"] - 1]
            assert all(c2 in a_done for c2 in prev), "K / V rows overwritten under the previous item's MMAs"
            kvready.arrive()
            soft["step"] = "s"
            return True
        if soft["step"] == "s":
            if not spfull.poll(c, f"softmax S {c}") or not full[c % rst].poll(c // rst, f"softmax stage {c}"):
                return False
            s_read.add(c)
            spfree.arrive()
            soft["step"] = "p"
            return True
        if soft["step"] == "p":
            if c >= 2 and not pdsfree[c & 1].poll((c >> 1) - 1, f"softmax P {c}"):
                return False
            assert c < 2 or c - 2 in b_done, f"P / dS buffer of op {c} written under the MMA of op {c - 2}"
            pdsfull[c & 1].arrive()
            soft["n"] += 1
            soft["step"] = "epi" if c in last_of_item else "s"
            return True
        if not itemdone.poll(soft["it"], f"epilogue {soft['item']}"):
            return False
        epi_done.add(soft["it"])
        soft["item"] += 1
        soft["it"] += 1
        soft["step"] = "kv"
        return True

    agents = [lambda: producer(0), lambda: producer(1), issuer_a, issuer_b, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while soft["item"] < len(items) or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            for f in done:
                f()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(ag() for ag in agents):
            raise AssertionError(f"deadlock: issuer A {a['n']}, B {b['n']}, softmax {soft} of {total}")
    assert b["n"] == total and itemdone.phases == len(nonempty)


@pytest.mark.parametrize("seed", range(60))
def test_dkdv_protocol_parity_and_progress(seed):
    rng = random.Random(1000 + seed)
    items = [rng.choice([0, 1, 2, 3, 5, 8, 13, 64]) for _ in range(rng.randint(1, 6))]
    run_dkdv(items, rng, mma_latency=rng.choice([1, 3, 10]))


def run_dq(items, rng, unified, mma_latency=3):
    """The dQ kernel's per-slot protocol: per block n of a query tile, op A(n) runs S = Q K^T
    and dP = dO V^T from block n's K and V, after B(n-1) has finished reading dS (which
    overwrote S); the softmax turns S, dP into dS; op B(n) runs dQ += dS K from the same K block
    and releases it. Op order A0, B0, A1, B1, ... As built, K blocks have a ring of 2 and V
    blocks a ring of 1, V released by A, K by B. With `unified`, K(n), V(n) share one ring of 3
    in load order (the change made in the forward kernel), so a stage's releases must still
    arrive in position order."""
    nblk = sum(items)
    nonempty = [k for k in items if k]
    item_start = set()
    acc = 0
    for k in nonempty:
        item_start.add(acc)
        acc += k
    if unified:
        rings = {"kv": [Barrier(1) for _ in range(3)]}
        emp = {"kv": [Barrier(1) for _ in range(3)]}
        slot = lambda kind, n: ("kv", 2 * n + (kind == "V"), 3)
    else:
        rings = {"K": [Barrier(1) for _ in range(2)], "V": [Barrier(1)]}
        emp = {"K": [Barrier(1) for _ in range(2)], "V": [Barrier(1)]}
        slot = lambda kind, n: (kind, n, 2 if kind == "K" else 1)
    sfull, dsfull, bdone, qready = Barrier(1), Barrier(1), Barrier(1), Barrier(1)
    loads = [(kind, n) for n in range(nblk) for kind in ("K", "V")]
    prod = {"i": 0}
    iss = {"a": 0, "b": 0}
    soft = {"n": 0, "it": 0, "step": "q"}
    a_done, b_done, ds_written, epi_done = set(), set(), set(), set()
    pending = []
    t = 0

    def producer():
        if prod["i"] >= len(loads):
            return False
        kind, n = loads[prod["i"]]
        ring, pos, rst = slot(kind, n)
        if not emp[ring][pos % rst].poll(pos // rst - 1, f"producer {kind}{n}"):
            return False
        # the previous occupant of this stage has been released by its last reader
        if pos >= rst:
            prev_pos = pos - rst
            if unified:
                pk, pn = ("V" if prev_pos % 2 else "K"), prev_pos // 2
            else:
                pk, pn = kind, prev_pos
            assert (pn in b_done) if pk == "K" else (pn in a_done), f"{kind}{n} loaded over {pk}{pn}"
        rings[ring][pos % rst].arrive()
        prod["i"] += 1
        return True

    def issuer():
        a, b = iss["a"], iss["b"]
        if b >= nblk:
            return False
        if a == b:  # A(a)
            if a in item_start and not qready.poll(sorted(item_start).index(a), f"A{a} Q"):
                return False
            if a > 0 and not bdone.poll(a - 1, f"A{a} bdone"):
                return False
            rk, pk, sk = slot("K", a)
            rv, pv, sv = slot("V", a)
            if not rings[rk][pk % sk].poll(pk // sk, f"A{a} K") or not rings[rv][pv % sv].poll(pv // sv, f"A{a} V"):
                return False
            assert a == 0 or a - 1 in b_done, f"S/dP of block {a} overwrite dS of block {a - 1} under its MMA"
            done = [lambda a=a: a_done.add(a), emp[rv][pv % sv].arrive, sfull.arrive]
            pending.append((t + rng.randint(1, mma_latency), done))
            iss["a"] += 1
            return True
        if not dsfull.poll(b, f"B{b}"):
            return False
        assert b in ds_written
        if b in item_start and sorted(item_start).index(b) > 0:
            assert sorted(item_start).index(b) - 1 in epi_done, f"dQ restarted at block {b} before the epilogue"
        rk, pk, sk = slot("K", b)
        done = [lambda b=b: b_done.add(b), emp[rk][pk % sk].arrive, bdone.arrive]
        pending.append((t + rng.randint(1, mma_latency), done))
        iss["b"] += 1
        return True

    def softmax():
        if soft["it"] >= len(nonempty):
            return False
        n = soft["n"]
        if soft["step"] == "q":  # Q and dO rows of the item into tensor memory
            assert all(m in a_done for m in range(n)), "Q / dO overwritten under the previous item's MMAs"
            qready.arrive()
            soft["step"] = "s"
            return True
        if soft["step"] == "s":
            if not sfull.poll(n, f"softmax S{n}"):
                return False
            ds_written.add(n)
            dsfull.arrive()
            soft["n"] += 1
            end = soft["n"] == sum(nonempty[:soft["it"] + 1])
            soft["step"] = "epi" if end else "s"
            return True
        if not bdone.poll(n - 1, f"epilogue {soft['it']}"):
            return False
        epi_done.add(soft["it"])
        soft["it"] += 1
        soft["step"] = "q"
        return True

    agents = [producer, issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while soft["it"] < len(nonempty) or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            for f in done:
                f()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(ag() for ag in agents):
            raise AssertionError(f"deadlock: A {iss['a']}, B {iss['b']}, softmax {soft} of {nblk}")
    assert len(b_done) == nblk


@pytest.mark.parametrize("unified", [False, True], ids=["kernel", "one_ring"])
@pytest.mark.parametrize("seed", range(60))
def test_dq_protocol_parity_and_progress(unified, seed):
    rng = random.Random(2000 + seed)
    items = [rng.choice([0, 1, 2, 3, 5, 8, 32]) for _ in range(rng.randint(1, 6))]
    run_dq(items, rng, unified, mma_latency=rng.choice([1, 3, 10]))
