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
The model also covers splits with two producers per slot (one per d-half, the full barrier
expecting two arrivals; or one per ring-position parity, which with three stages needs the
positions issued in order). Besides the barrier rules it asserts the data hazards the barriers
exist for: a ring block, an S buffer or P is overwritten only after its last reader finished.

Further models: P written over its S buffer and the softmax split over two warps per lane
quarter (`run_aliased`), the dK/dV and dQ kernels (`run_dkdv`, `run_dq`, the latter also with
dS in shared memory), the item queues through which the kernels hand out the items they
draw from a global counter (`run_item_queue`), the forward on 128-token tiles with its
separate K and V rings, P over S and Q rewritten per query tile (`run_b128`), and the dQ kernel
on 128-token tiles with dS over S and K held until dQ has read it (`run_dq_b128`).
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


def run(tiles, rst, producers, rng, mma_latency=3, lead=1, parity=False, ordered=False):
    """`producers` = 2 splits each block between two producers (one per d-half, the full barrier
    expecting both), or with `parity` gives ring position c to producer c % 2 alone; with
    `ordered` a producer loads position c only after position c - 1 was loaded (by the other)."""
    ops = ops_of(tiles, lead)
    full = [Barrier(1 if parity else producers) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    sfull, sfree = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    pfull, pvdone = Barrier(1), Barrier(1)
    prod = [p if parity else 0 for p in range(producers)]  # next ring position per producer
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
        if ordered and c > 0 and prod[1 - p] < c:  # position c - 1 not loaded yet
            return False
        st = c % rst
        if not empty[st].poll(c // rst - 1, f"producer {p} at {c}"):
            return False
        assert c < rst or c - rst in op_done, f"ring position {c} refilled before its MMA finished"
        full[st].arrive()
        prod[p] += producers if parity else 1
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
    assert pvdone.phases == sum(tiles) and all(p >= len(ops) for p in prod)


def run_aliased(tiles, rst, rng, mma_latency=3, rescale_p=0.2, lead=1, halves=1, xch_bufs=2, sfree_count=None):
    """The forward kernel's protocol with P written over the S buffer it came from: per slot two
    S/P buffers, pfull and pvdone per block parity, no wait for the previous P.V before writing P;
    the softmax waits for the previous P.V only to rescale O (at random here) and at a tile's end.
    The tensor pipe completes MMAs in issue order. Asserts, besides the parity rule, that S(k)
    overwrites a buffer only after O(k-2) read its P, that P(g) is written only after O(g-2)
    read the previous P of the buffer, and that O is read only after every P.V issued before.

    `halves` = 2 models the softmax split over two warps per lane quarter, each owning one KV tile
    of the block: each half reads its S columns and writes its P inside them, the halves meet at a
    pair barrier once per block to combine the row max through a shared-memory slot chosen by
    block parity (`xch_bufs` slots), and once at a tile's end to combine the row sums. sfree and
    pfull then expect one arrival per half. The model asserts that an exchange slot is rewritten
    only after the other half read it, and that S(k) overwrites a buffer only after every half
    read S(k-2)."""
    ops = ops_of(tiles, lead=lead)
    full = [Barrier(1) for _ in range(rst)]
    empty = [Barrier(1) for _ in range(rst)]
    sfc = halves if sfree_count is None else sfree_count
    sfull, sfree = [Barrier(1), Barrier(1)], [Barrier(sfc), Barrier(sfc)]
    pfull, pvdone = [Barrier(halves), Barrier(halves)], [Barrier(1), Barrier(1)]
    prod = {"c": 0}
    mma = {"c": 0, "s": 0, "o": 0}
    soft = [{"blk": 0, "step": 0} for _ in range(halves)]
    done = {"op": set(), "s": set(), "o": set()}
    p_written = [set() for _ in range(halves)]
    s_read = [set() for _ in range(halves)]
    gen = [0] * halves               # pair-barrier arrivals per half
    xslot = {}                       # (kind, slot, half) -> [value, halves that have read it]
    rescale = {}                     # block -> rescale decision, the same for every half
    ends = []                        # block index that ends each tile
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
                assert k < 2 or all(k - 2 in r for r in s_read), f"S{k} overwrote S{k - 2} before every half read it"
                done["op"].add(c)
                done["s"].add(k)
                empty[st].arrive()
                sfull[k % 2].arrive()
            mma["s"] += 1
        else:
            k = mma["o"]
            if not pfull[k % 2].poll(k // 2, f"issuer O{k}"):
                return False
            assert all(k in w for w in p_written), f"O{k} issued before every half wrote P{k}"

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

    def put(kind, slot, h, value):
        old = xslot.get((kind, slot, h))
        assert old is None or len(old[1]) == halves - 1, f"{kind} slot {slot} of half {h} rewritten before it was read"
        xslot[(kind, slot, h)] = [value, set()]
        gen[h] += 1

    def take(kind, slot, h, value):
        if any(gen[j] < gen[h] for j in range(halves)):
            return False  # the pair barrier: every half has arrived
        for j in range(halves):
            if j != h:
                v = xslot[(kind, slot, j)]
                assert v[0] == value, f"half {h} read {kind} {v[0]} for {value}"
                v[1].add(h)
        return True

    def softmax(h):
        sm = soft[h]
        g = sm["blk"]
        if g >= nblk:
            return False
        st = sm["step"]
        if st == 0:                       # wait S, read this half's columns, free the buffer
            if not sfull[g % 2].poll(g // 2, f"softmax S{g}"):
                return False
            assert g in done["s"]
            s_read[h].add(g)
            sfree[g % 2].arrive()
            sm["step"] = 1
            return True
        if st == 1:                       # row max of this half into the exchange slot
            put("max", g % xch_bufs, h, g)
            sm["step"] = 2
            return True
        if st == 2:                       # pair barrier, then the other halves' max
            if not take("max", g % xch_bufs, h, g):
                return False
            first = g == 0 or (g - 1) in ends
            r = rescale.setdefault(g, (not first) and rng.random() < rescale_p)
            sm["step"] = 3 if r else 4
            return True
        if st == 3:                       # rescale O: the previous P.V must be done
            if not wait_pv(g - 1, f"softmax rescale at {g}"):
                return False
            assert all(x in done["o"] for x in range(g)), f"O read at block {g} with a P.V pending"
            sm["step"] = 4
            return True
        if st == 4:                       # write P over this half's S columns
            assert g < 2 or g - 2 in done["o"], f"P{g} written before O{g - 2} read P{g - 2}"
            p_written[h].add(g)
            pfull[g % 2].arrive()
            if g in ends:
                sm["step"] = 5
            else:
                sm["blk"], sm["step"] = g + 1, 0
            return True
        if st == 5:                       # tile's last P.V, then this half's row sum
            if not wait_pv(g, f"softmax epilogue at {g}"):
                return False
            assert all(x in done["o"] for x in range(g + 1)), f"epilogue at {g} with a P.V pending"
            put("sum", 0, h, g)
            sm["step"] = 6
            return True
        if not take("sum", 0, h, g):      # st == 6: pair barrier, the other halves' sums
            return False
        sm["blk"], sm["step"] = g + 1, 0
        return True

    agents = [producer, issuer] + [lambda h=h: softmax(h) for h in range(halves)]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while mma["c"] < len(ops) or any(sm["blk"] < nblk for sm in soft) or pending:
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
            raise AssertionError(f"deadlock at op {mma['c']} of {len(ops)}, softmax blocks {[sm['blk'] for sm in soft]}")
    assert len(done["o"]) == nblk


@pytest.mark.parametrize("seed", range(80))
def test_forward_protocol_with_p_over_s(seed):
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run_aliased(tiles, rst=3, rng=rng, mma_latency=rng.choice([1, 3, 10, 30]))


@pytest.mark.parametrize("seed", range(80))
def test_forward_protocol_split_softmax(seed):
    """Two softmax warps per lane quarter (one per KV tile of a block): the split variant of the
    forward, measured and dropped; the protocol stays checked."""
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run_aliased(tiles, rst=3, rng=rng, mma_latency=rng.choice([1, 3, 10, 30]), halves=2)


def test_forward_protocol_split_flags_a_single_exchange_slot():
    """One row-max slot per half instead of one per block parity: a fast half rewrites it for the
    next block before the other half has read it."""
    with pytest.raises(AssertionError):
        for seed in range(200):
            run_aliased([32, 5], rst=3, rng=random.Random(seed), mma_latency=3, halves=2, xch_bufs=1)


def test_forward_protocol_split_flags_one_sfree_arrival():
    """With sfree released by one arrival, S(k+2) can overwrite a buffer the other half has not
    read yet."""
    with pytest.raises(AssertionError):
        for seed in range(200):
            run_aliased([32, 5], rst=3, rng=random.Random(seed), mma_latency=1, halves=2, sfree_count=1)


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


@pytest.mark.parametrize("seed", range(60))
def test_ring_protocol_parity_split_producers_in_order(seed):
    """Two producers per slot on ring-position parity with the kernel's three stages: each loads
    position c only after the other has loaded c - 1, so no stage is waited on two phases ahead."""
    rng = random.Random(5000 + seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
    run(tiles, rst=3, producers=2, rng=rng, mma_latency=rng.choice([1, 3, 10]), parity=True, ordered=True)


def test_ring_protocol_parity_split_without_order_is_flagged():
    """Without that order a producer can wait on a stage two phases ahead (three stages shared by
    two producers): the parity rule flags it."""
    with pytest.raises(AssertionError):
        for seed in range(5000, 5100):
            rng = random.Random(seed)
            tiles = [rng.choice([1, 1, 2, 3, 4, 5, 7, 32]) for _ in range(rng.randint(1, 6))]
            run(tiles, rst=3, producers=2, rng=rng, mma_latency=rng.choice([1, 3, 10]), parity=True)


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


def run_dq(items, rng, unified, mma_latency=3, ds_smem=False, ds_wait=True):
    """The dQ kernel's per-slot protocol: per block n of a query tile, op A(n) runs S = Q K^T
    and dP = dO V^T from block n's K and V; the softmax turns S, dP into dS; op B(n) runs
    dQ += dS K from the same K block and releases it. K blocks have a ring of 2 and V blocks a
    ring of 1, V released by A, K by B. With `unified`, K(n), V(n) share one ring of 3 in load
    order, so a stage's releases must still arrive in position order.

    As built, dS is written over S in tensor memory and the order is A0, B0, A1, B1, ..., A(n)
    after B(n-1) is done. With `ds_smem` (a variant that was measured and dropped) the softmax
    writes dS to shared memory: it frees S/dP (sfree) as soon as both are in registers, and waits
    for B(n-1) before writing dS(n) over the buffer B(n-1) reads; the issuer then runs A(n+1)
    before B(n) (order A0, A1, B0, A2, B1, ...), and the tensor pipe completes MMAs in issue
    order. `ds_wait=False` drops that softmax wait (a seeded mistake)."""
    nblk = sum(items)
    nonempty = [k for k in items if k]
    item_start = set()
    acc = 0
    for k in nonempty:
        item_start.add(acc)
        acc += k
    item_end = {st + k - 1 for st, k in zip(sorted(item_start), nonempty)}
    if unified:
        rings = {"kv": [Barrier(1) for _ in range(3)]}
        emp = {"kv": [Barrier(1) for _ in range(3)]}
        slot = lambda kind, n: ("kv", 2 * n + (kind == "V"), 3)
    else:
        rings = {"K": [Barrier(1) for _ in range(2)], "V": [Barrier(1)]}
        emp = {"K": [Barrier(1) for _ in range(2)], "V": [Barrier(1)]}
        slot = lambda kind, n: (kind, n, 2 if kind == "K" else 1)
    sfull, sfree, dsfull, bdone, qready = Barrier(1), Barrier(1), Barrier(1), Barrier(1), Barrier(1)
    loads = [(kind, n) for n in range(nblk) for kind in ("K", "V")]
    # the issuer's op stream
    ops = []
    for st, k in zip(sorted(item_start), nonempty):
        an = bn = 0
        while bn < k:
            if an < k and an <= bn + (1 if ds_smem else 0):
                ops.append(("A", st + an))
                an += 1
            else:
                ops.append(("B", st + bn))
                bn += 1
    prod = {"i": 0}
    iss = {"c": 0}
    soft = {"n": 0, "it": 0, "step": "q"}
    a_done, b_done, s_read, ds_written, epi_done = set(), set(), set(), set(), set()
    ds_buf = {"block": None}  # which block's dS the shared buffer holds
    pending = []
    pipe = {"last": 0}
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

    def run_mma(done):
        if ds_smem:  # in issue order
            pipe["last"] = max(pipe["last"], t) + rng.randint(1, mma_latency)
            pending.append((pipe["last"], done))
        else:
            pending.append((t + rng.randint(1, mma_latency), done))

    def issuer():
        if iss["c"] >= len(ops):
            return False
        kind, n = ops[iss["c"]]
        if kind == "A":
            if n in item_start and not qready.poll(sorted(item_start).index(n), f"A{n} Q"):
                return False
            if ds_smem:
                if n > 0 and not sfree.poll(n - 1, f"A{n} sfree"):
                    return False
            elif n > 0 and not bdone.poll(n - 1, f"A{n} bdone"):
                return False
            rk, pk, sk = slot("K", n)
            rv, pv, sv = slot("V", n)
            if not rings[rk][pk % sk].poll(pk // sk, f"A{n} K") or not rings[rv][pv % sv].poll(pv // sv, f"A{n} V"):
                return False
            if ds_smem:
                assert n == 0 or n - 1 in s_read, f"S/dP of block {n} overwrite block {n - 1} before the softmax read it"
            else:
                assert n == 0 or n - 1 in b_done, f"S/dP of block {n} overwrite dS of block {n - 1} under its MMA"
            run_mma([lambda n=n: a_done.add(n), emp[rv][pv % sv].arrive, sfull.arrive])
        else:
            if not dsfull.poll(n, f"B{n}"):
                return False
            assert n in ds_written
            if n in item_start and sorted(item_start).index(n) > 0:
                assert sorted(item_start).index(n) - 1 in epi_done, f"dQ restarted at block {n} before the epilogue"
            rk, pk, sk = slot("K", n)

            def fin(n=n):
                assert not ds_smem or ds_buf["block"] == n, f"B{n} read dS of block {ds_buf['block']}"
                b_done.add(n)
            run_mma([fin, emp[rk][pk % sk].arrive, bdone.arrive])
        iss["c"] += 1
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
            assert n in a_done
            s_read.add(n)
            if ds_smem:
                sfree.arrive()
                soft["step"] = "w"
                return True
            ds_written.add(n)
            dsfull.arrive()
            return advance(n)
        if soft["step"] == "w":  # dS into shared memory once B(n-1) has read the previous dS
            if ds_wait and n > 0 and not bdone.poll(n - 1, f"softmax dS{n}"):
                return False
            assert n == 0 or (n - 1) in b_done or (n - 1) not in ds_written, f"dS{n} written under B{n - 1}"
            ds_buf["block"] = n
            ds_written.add(n)
            dsfull.arrive()
            return advance(n)
        if not bdone.poll(n - 1, f"epilogue {soft['it']}"):
            return False
        epi_done.add(soft["it"])
        soft["it"] += 1
        soft["step"] = "q"
        return True

    def advance(n):
        soft["n"] += 1
        soft["step"] = "epi" if n in item_end else "s"
        return True

    agents = [producer, issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while soft["it"] < len(nonempty) or pending:
        t += 1
        due = [x for x in pending if x[0] <= t]
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in sorted(due, key=lambda x: x[0]):
            for f in done:
                f()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(ag() for ag in agents):
            raise AssertionError(f"deadlock: op {iss['c']} of {len(ops)}, softmax {soft} of {nblk}")
    assert len(b_done) == nblk


@pytest.mark.parametrize("layout", ["kernel", "one_ring", "smem_ds"])
@pytest.mark.parametrize("seed", range(60))
def test_dq_protocol_parity_and_progress(layout, seed):
    rng = random.Random(2000 + seed)
    items = [rng.choice([0, 1, 2, 3, 5, 8, 32]) for _ in range(rng.randint(1, 6))]
    run_dq(items, rng, unified=layout == "one_ring", mma_latency=rng.choice([1, 3, 10]),
           ds_smem=layout == "smem_ds")


def test_dq_protocol_flags_a_missing_ds_wait():
    """Without the softmax's wait for B(n-1), dS(n) can land in shared memory while the previous
    dQ MMA still reads it."""
    with pytest.raises(AssertionError):
        for seed in range(200):
            run_dq([32, 5], random.Random(seed), unified=False, mma_latency=10, ds_smem=True, ds_wait=False)


def test_dq_protocol_one_ring_deadlocks_with_a_ahead():
    """A single K/V ring in load order cannot serve A(n+1) before B(n): V(n+1) would wait for the
    release of K(n) by B(n), which the in-order issuer holds behind A(n+1)."""
    with pytest.raises(AssertionError, match="deadlock"):
        run_dq([8], random.Random(0), unified=True, mma_latency=3, ds_smem=True)


def run_item_queue(n_items, qd, rng, empty_count=None, ahead=2, consumers=2):
    """The forward kernel's per-slot item queue: the producer warp takes items from a global
    counter and writes each into entry k % qd (after the entry's release, iqempty), `ahead`
    items before it loads the item's blocks, then -1 at the end. The MMA issuer and the
    softmax's first warp each read every entry in order (after iqfull) and release it; a
    consumer can finish item k only once the producer has reached item k's loads. Asserts the
    parity rule, that no entry is rewritten before both consumers read it, that both read the
    producer's sequence exactly, and progress."""
    ids = list(range(n_items)) + [-1]
    full = [Barrier(1) for _ in range(qd)]
    empty = [Barrier(consumers if empty_count is None else empty_count) for _ in range(qd)]
    slots = [None] * qd
    readers = [set() for _ in range(qd)]
    prod = {"k": 0}
    cons = [{"k": 0, "got": [], "working": None} for _ in range(consumers)]

    def loads_reached():  # items whose blocks the producer has issued
        return max(0, prod["k"] - ahead)

    def producer():
        k = prod["k"]
        if k >= len(ids):
            return False
        e = k % qd
        if not empty[e].poll(k // qd - 1, f"producer entry {k}"):
            return False
        assert slots[e] is None or readers[e] == set(range(consumers)), f"entry {k} rewritten before every consumer read it"
        slots[e] = ids[k]
        readers[e] = set()
        full[e].arrive()
        prod["k"] += 1
        return True

    def consumer(c):
        st = cons[c]
        if st["working"] is not None:  # finish the current item once its loads were issued
            if st["working"] < loads_reached() or prod["k"] == len(ids):
                st["working"] = None
                return True
            return False
        k = st["k"]
        if st["got"] and st["got"][-1] == -1:
            return False
        e = k % qd
        if not full[e].poll(k // qd, f"consumer {c} entry {k}"):
            return False
        v = slots[e]
        readers[e].add(c)
        empty[e].arrive()
        st["got"].append(v)
        st["k"] += 1
        if v >= 0:
            st["working"] = v
        return True

    agents = [producer] + [lambda c=c: consumer(c) for c in range(consumers)]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while not all(st["got"] and st["got"][-1] == -1 for st in cons):
        moved = False
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not any(a() for a in agents):
            raise AssertionError(f"deadlock: producer at {prod['k']}, consumers at {[st['k'] for st in cons]}")
    for st in cons:
        assert st["got"] == ids


@pytest.mark.parametrize("seed", range(60))
def test_item_queue_parity_and_progress(seed):
    rng = random.Random(seed)
    run_item_queue(rng.randint(0, 40), qd=4, rng=rng)


@pytest.mark.parametrize("seed", range(40))
def test_item_queue_backward_kernels(seed):
    """The backward kernels' queues: the drawing producer writes an item when it reaches it (no
    lookahead); the dQ kernel has two takers per slot, the dK/dV kernel four."""
    rng = random.Random(300 + seed)
    run_item_queue(rng.randint(0, 40), qd=4, rng=rng, ahead=0, consumers=2)
    run_item_queue(rng.randint(0, 40), qd=4, rng=rng, ahead=0, consumers=4)


def test_item_queue_flags_a_single_release():
    """iqempty completing on one consumer's release lets the producer rewrite an entry the other
    consumer has not read."""
    with pytest.raises(AssertionError):
        for seed in range(200):
            run_item_queue(30, qd=4, rng=random.Random(seed), empty_count=1)


def test_item_queue_needs_as_many_entries_as_the_lookahead():
    """With qd < ahead the producer waits for a release that needs its own loads: deadlock (the
    kernel has qd = 4, ahead = 2)."""
    run_item_queue(10, qd=2, rng=random.Random(0), ahead=2)
    with pytest.raises(AssertionError, match="deadlock"):
        run_item_queue(10, qd=1, rng=random.Random(0), ahead=2)


def run_b128(items, rng, kst=3, vst=3, mma_latency=3, rescale_p=0.2, lead=1, qready_count=True):
    """The forward on 128-token tiles: a K ring and a V ring, each with its own producer (in the
    item's block order); one MMA issuer walking S0, S1, O0, S2, O1, ... per item; S(n) and P(n)
    share TMEM buffer n % 2 (P written over S by the softmax), so S(n + 2) may overwrite it only
    after O(n) has read P(n), which the in-order tensor pipe gives because S(n + 2) is issued
    after O(n). Per item the softmax writes Q (after reading the item's last S) and signals
    qready, which the first S MMA of the item waits for; O(0) of an item starts a fresh
    accumulation, after the softmax's epilogue of the previous item read O (ordered through
    pfull). A raise (random here) waits for O(n - 1) before rescaling O. `qready_count=False`
    lets the first S of an item skip its wait (a seeded mistake)."""
    tiles = [n for n in items]
    ops = []  # (kind, item, block, global block index)
    gb = 0
    for it, n in enumerate(tiles):
        for kind, k in ops_of([n], lead):
            ops.append((kind, it, k, gb + k))
        gb += n
    nblk = gb
    kfull, kempty = [Barrier(1) for _ in range(kst)], [Barrier(1) for _ in range(kst)]
    vfull, vempty = [Barrier(1) for _ in range(vst)], [Barrier(1) for _ in range(vst)]
    sfull, pfull, pvdone = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    qready = Barrier(1)
    prod = {"k": 0, "v": 0}
    mma = {"c": 0, "s": 0, "o": 0, "tile": 0}
    soft = {"item": 0, "blk": 0, "g": 0, "step": 0}
    s_done, o_done, s_read, p_written, o_issued = set(), set(), set(), set(), set()
    q_written = set()       # items whose Q is in TMEM
    epi_done = set()        # items whose epilogue has read O
    k_read, v_read = set(), set()
    pipe = {"free": 0}      # the tensor pipe completes in issue order
    pending = []
    t = 0
    nonempty = [i for i, n in enumerate(tiles) if n > 0]

    def producer(kind):
        c = prod[kind]
        if c >= nblk:
            return False
        nst, empty, full, read = (kst, kempty, kfull, k_read) if kind == "k" else (vst, vempty, vfull, v_read)
        st = c % nst
        if not empty[st].poll(c // nst - 1, f"{kind} producer at {c}"):
            return False
        assert c < nst or c - nst in read, f"{kind} ring position {c} refilled before its MMA finished"
        full[st].arrive()
        prod[kind] += 1
        return True

    def issue(done):
        pipe["free"] = max(pipe["free"], t) + rng.randint(1, mma_latency)
        pending.append((pipe["free"], done))

    def issuer():
        c = mma["c"]
        if c >= len(ops):
            return False
        kind, it, k, g = ops[c]
        if kind == "S":
            if k == 0:
                tl = nonempty.index(it)
                if qready_count and not qready.poll(tl, f"issuer Q of item {it}"):
                    return False
            if not kfull[g % kst].poll(g // kst, f"issuer S{g}"):
                return False
            # the pipe runs one thread's MMAs in order: O(g - 2) issued means it reads P(g - 2) first
            assert g < 2 or g - 2 in o_issued, f"S{g} issued before O{g - 2}"
            assert g < 2 or g - 2 in s_read, f"S{g} overwrites S{g - 2} before the softmax read it"

            def done(g=g, it=it):
                assert it in q_written, f"S{g} read Q of item {it} before it was written"
                assert (g - 2 < 0) or (g - 2 in o_done) or (g - 2 not in p_written), f"S{g} overwrote P{g - 2}"
                s_done.add(g)
                k_read.add(g)
                kempty[g % kst].arrive()
                sfull[g % 2].arrive()
            issue(done)
            mma["s"] += 1
        else:
            if not vfull[g % vst].poll(g // vst, f"issuer O{g} V"):
                return False
            if not pfull[g % 2].poll(g // 2, f"issuer O{g} P"):
                return False
            if k == 0:
                assert it == 0 or (it - 1) in epi_done or all(tiles[j] == 0 for j in range(it)), \
                    f"O(0) of item {it} would reset O before the previous epilogue read it"

            o_issued.add(g)

            def done(g=g):
                assert g in p_written
                o_done.add(g)
                v_read.add(g)
                vempty[g % vst].arrive()
                pvdone[g % 2].arrive()
            issue(done)
            mma["o"] += 1
        mma["c"] += 1
        return True

    def softmax():
        it = soft["item"]
        if it >= len(tiles):
            return False
        n = tiles[it]
        if soft["step"] == 0:  # item start: write Q (the previous item's S are all read)
            if n > 0:
                assert all(x in s_done for x in range(soft["g"])), "Q rewritten before the last S finished"
                q_written.discard(it - 1)
                q_written.add(it)
                qready.arrive()
            soft["step"] = 1
            return True
        b = soft["blk"]
        g = soft["g"]
        if b < n:
            if soft["step"] == 1:
                if not sfull[g % 2].poll(g // 2, f"softmax S{g}"):
                    return False
                s_read.add(g)
                soft["step"] = 2 if (b > 0 and rng.random() < rescale_p) else 3
                return True
            if soft["step"] == 2:  # raise: rescale O once O(g - 1) is done
                if not pvdone[(g - 1) % 2].poll((g - 1) // 2, f"softmax rescale at {g}"):
                    return False
                assert g - 1 in o_done
                soft["step"] = 3
                return True
            p_written.add(g)  # P over its own S buffer: nothing to wait for
            pfull[g % 2].arrive()
            soft["blk"], soft["g"], soft["step"] = b + 1, g + 1, 1
            return True
        if n > 0:  # epilogue: O of the item complete
            if not pvdone[(g - 1) % 2].poll((g - 1) // 2, f"softmax epilogue of item {it}"):
                return False
            assert g - 1 in o_done
        epi_done.add(it)
        soft["item"], soft["blk"], soft["step"] = it + 1, 0, 0
        return True

    agents = [lambda: producer("k"), lambda: producer("v"), issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while mma["c"] < len(ops) or soft["item"] < len(tiles) or pending:
        t += 1
        due = sorted([x for x in pending if x[0] <= t], key=lambda x: x[0])
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            done()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(a() for a in agents):
            raise AssertionError(f"deadlock at op {mma['c']} of {len(ops)}, softmax item {soft['item']}")
    assert len(o_done) == nblk and prod["k"] == nblk and prod["v"] == nblk


@pytest.mark.parametrize("seed", range(30))
def test_b128_forward_protocol(seed):
    rng = random.Random(seed)
    items = [rng.choice([0, 1, 2, 3, 5, 8]) for _ in range(rng.randint(2, 8))]
    run_b128(items, rng)


def test_b128_forward_protocol_flags_a_skipped_qready_wait():
    hits = 0
    for seed in range(60):
        rng = random.Random(seed)
        try:
            run_b128([3, 4, 2, 5], rng, qready_count=False)
        except AssertionError:
            hits += 1
    assert hits > 0


def test_b128_forward_protocol_flags_lead_two_with_p_over_s():
    """With S two blocks ahead (S0, S1, S2, O0, ...), S(n + 2) would be issued before O(n) has
    read P(n) from the buffer it overwrites."""
    hits = 0
    for seed in range(30):
        try:
            run_b128([4, 3, 5], random.Random(seed), lead=2)
        except AssertionError:
            hits += 1
    assert hits == 30


def run_dq_b128(items, rng, kst=3, vst=2, mma_latency=3, skip_dsfull=False, skip_qready=False):
    """The dQ kernel on 128-token tiles: a K ring (a tile held until dQ(n) has read it) and a V
    ring (released after S/dP(n)), each with its own producer; one MMA issuer walking
    S/dP(0), dQ(0), S/dP(1), dQ(1), ... with one S and one dP buffer, reused for block n once
    dQ(n - 1) is done (bdone); the softmax reads S and dP of block n, writes dS over S and signals
    dsfull; per item it writes Q and dO (after the item before has had all its S/dP read) and
    signals qready, and its epilogue reads dQ after the item's last dQ MMA. The tensor pipe
    completes one thread's MMAs in issue order. `skip_dsfull` / `skip_qready` drop a wait (seeded
    mistakes)."""
    tiles = list(items)
    nblk = sum(tiles)
    kfull, kempty = [Barrier(1) for _ in range(kst)], [Barrier(1) for _ in range(kst)]
    vfull, vempty = [Barrier(1) for _ in range(vst)], [Barrier(1) for _ in range(vst)]
    sfull, dsfull, bdone, qready = Barrier(1), Barrier(1), Barrier(1), Barrier(1)
    prod = {"k": 0, "v": 0}
    mma = {"c": 0, "phase": 0, "item": 0, "blk": 0}  # phase 0: S/dP of block c, 1: dQ of block c
    soft = {"item": 0, "blk": 0, "g": 0, "step": 0}
    sp_done, dq_done, sp_read, ds_written = set(), set(), set(), set()
    k_read, v_read = set(), set()
    q_items, epi_done = set(), set()
    pipe = {"free": 0}
    pending = []
    t = 0
    nonempty = [i for i, n in enumerate(tiles) if n > 0]
    blocks = [(it, b) for it, n in enumerate(tiles) for b in range(n)]  # block c -> (item, index)

    def producer(kind):
        c = prod[kind]
        if c >= nblk:
            return False
        nst, empty, full, read = (kst, kempty, kfull, k_read) if kind == "k" else (vst, vempty, vfull, v_read)
        st = c % nst
        if not empty[st].poll(c // nst - 1, f"{kind} producer at {c}"):
            return False
        assert c < nst or c - nst in read, f"{kind} ring position {c} refilled before its last MMA"
        full[st].arrive()
        prod[kind] += 1
        return True

    def issue(done):
        pipe["free"] = max(pipe["free"], t) + rng.randint(1, mma_latency)
        pending.append((pipe["free"], done))

    def issuer():
        c = mma["c"]
        if c >= nblk:
            return False
        it, b = blocks[c]
        if mma["phase"] == 0:
            if b == 0 and not skip_qready and not qready.poll(nonempty.index(it), f"issuer Q of item {it}"):
                return False
            if c > 0 and not bdone.poll(c - 1, f"issuer S/dP{c}"):
                return False
            if not kfull[c % kst].poll(c // kst, f"issuer K{c}") or not vfull[c % vst].poll(c // vst, f"issuer V{c}"):
                return False

            def done(c=c, it=it):
                assert it in q_items, f"S/dP{c} read Q/dO of item {it} before they were written"
                assert c == 0 or (c - 1 in dq_done and c - 1 in sp_read), f"S/dP{c} overwrote block {c - 1}"
                sp_done.add(c)
                v_read.add(c)
                vempty[c % vst].arrive()
                sfull.arrive()
            issue(done)
            mma["phase"] = 1
            return True
        if not skip_dsfull and not dsfull.poll(c, f"issuer dQ{c}"):
            return False
        if b == 0:
            assert it == 0 or all(j in epi_done for j in range(it)), f"dQ(0) of item {it} before the epilogue"

        def done(c=c):
            assert c in ds_written, f"dQ{c} read dS before it was written"
            dq_done.add(c)
            k_read.add(c)
            kempty[c % kst].arrive()
            bdone.arrive()
        issue(done)
        mma["phase"], mma["c"] = 0, c + 1
        return True

    def softmax():
        it = soft["item"]
        if it >= len(tiles):
            return False
        n, g = tiles[it], soft["g"]
        if soft["step"] == 0:  # item start: Q and dO into TMEM
            if n > 0:
                assert all(x in sp_done for x in range(g)), "Q/dO rewritten before the last S/dP finished"
                q_items.add(it)
                qready.arrive()
            soft["step"] = 1
            return True
        if soft["blk"] < n:
            if soft["step"] == 1:
                if not sfull.poll(g, f"softmax S/dP{g}"):
                    return False
                sp_read.add(g)
                soft["step"] = 2
                return True
            ds_written.add(g)  # dS over S
            dsfull.arrive()
            soft["blk"], soft["g"], soft["step"] = soft["blk"] + 1, g + 1, 1
            return True
        if n > 0:
            if not bdone.poll(g - 1, f"softmax epilogue of item {it}"):
                return False
            assert all(x in dq_done for x in range(g - n, g))
        epi_done.add(it)
        soft["item"], soft["blk"], soft["step"] = it + 1, 0, 0
        return True

    agents = [lambda: producer("k"), lambda: producer("v"), issuer, softmax]
    speed = [rng.uniform(0.05, 1.0) for _ in agents]
    while mma["c"] < nblk or soft["item"] < len(tiles) or pending:
        t += 1
        due = sorted([x for x in pending if x[0] <= t], key=lambda x: x[0])
        pending[:] = [x for x in pending if x[0] > t]
        for _, done in due:
            done()
        moved = bool(due)
        for i in rng.sample(range(len(agents)), len(agents)):
            if rng.random() < speed[i]:
                moved |= agents[i]()
        if not moved and not pending and not any(a() for a in agents):
            raise AssertionError(f"deadlock at block {mma['c']} of {nblk}, softmax item {soft['item']}")
    assert len(dq_done) == nblk and prod["k"] == nblk and prod["v"] == nblk


@pytest.mark.parametrize("seed", range(30))
def test_dq_b128_protocol(seed):
    rng = random.Random(seed)
    run_dq_b128([rng.choice([0, 1, 2, 3, 5, 8]) for _ in range(rng.randint(2, 8))], rng)


@pytest.mark.parametrize("mistake", ["skip_dsfull", "skip_qready"])
def test_dq_b128_protocol_flags_a_skipped_wait(mistake):
    hits = 0
    for seed in range(60):
        try:
            run_dq_b128([3, 4, 2, 5], random.Random(seed), **{mistake: True})
        except AssertionError:
            hits += 1
    assert hits > 0
