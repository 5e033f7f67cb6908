"""Discrete-event model of the backward kernel's barrier schedule (fa_bwd_kernel.cuh).

The roles of one CTA -- the TMA producer, the MMA issuer with the tensor core
executing its MMAs in order, and the eight compute warps -- are re-stated as
generators over mbarriers with the hardware's parity rule (a wait on parity p
returns once the barrier's current, incomplete phase has the other parity).  Random
latencies are drawn for copies, MMAs and compute.  Checked for every schedule:
  * every role finishes (no deadlock);
  * every wait is released by exactly the phase it was written for (a waiter that
    fell two phases behind would be released by the wrong phase -- parity aliasing);
  * the data each role consumes is the data of its own tile (Q/dO slot contents,
    S/dP contents, the dS^T buffer and the dQ columns), so no buffer is overwritten
    while still in use.
At d = 64 the compute warps first copy the block's K and V rows into TMEM and arrive on
kv_tmem, which the issuer waits for before the first S^T.
An alternative issue order -- dP^T of tile t + 1 right after dQ_t, ahead of the wait for
the compute warps to read dQ_t out of the S columns -- is checked as well.
Geometry as in the kernel: warp w serves TMEM lane quadrant qd and query half g; the
tile's 128 queries are four blocks cb of 32.  A warp computes its blocks cb = 2g + pass
in two passes and hands each pass over on p_full[pass]; the issuer runs dV and dK of
pass h (blocks h and 2 + h) while the next pass is computed.  dS^T of block cb goes to
shared-memory box cb // 2, rows of quadrant qd -- the region where warp (qd, g = box)
stages its dQ for the tensor reduce.  S/dP columns are tracked per (block, quadrant),
shared-memory regions per (box, quadrant).
This checks the protocol as designed; the kernel is checked by the GPU parity tests.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: more arrivals than expected"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.completed & 1) != parity


def fill(cols, v):
    for half in cols:
        half[:] = [v] * len(half)


def holds(cols, v):
    return all(x == v for half in cols for x in half)


def kernel_cb(pass_, g):
    """Query block a warp of query half g computes in pass pass_."""
    return 2 * g + pass_


def kernel_pass_blocks(h):
    """Query blocks the issuer's dV / dK of pass h read (kk = 2h, 2h+1, 2h+4, 2h+5)."""
    return (h, 2 + h)


BLOCKS = [(cb, qd) for cb in range(4) for qd in range(4)]
REGIONS = [(box, qd) for box in range(2) for qd in range(4)]


class Sim:
    def __init__(self, n_t, stages, seed, warps=8, stages_o=None, kv_in_tmem=False):
        self.rng = random.Random(seed)
        self.kv_in_tmem = kv_in_tmem
        self.n_t, self.S, self.W = n_t, stages, warps
        self.SO = stages if stages_o is None else stages_o
        self.now = 0
        self.events = []          # (time, seq, callable)
        self.seq = 0
        b = Barrier
        self.kv = b("kv_full", 1)
        self.q_full = [b(f"q_full{s}", 1) for s in range(stages)]
        self.q_empty = [b(f"q_empty{s}", 1) for s in range(stages)]
        self.o_full = [b(f"o_full{s}", 1) for s in range(self.SO)]
        self.o_empty = [b(f"o_empty{s}", 1) for s in range(self.SO)]
        self.s_full = b("s_full", 1)
        self.p_full = [b(f"p_full{h}", warps) for h in range(2)]
        self.dq_full, self.s_free = b("dq_full", 1), b("s_free", warps)
        self.drain = b("drain", 1)
        self.kv_tmem = b("kv_tmem", warps)   # K and V rows copied into TMEM (d = 64)
        self.k_tmem = None                   # what the TMEM copy of K / V was taken from
        self.kv_landed = False
        # buffer contents: which tile's data they hold
        self.slot = [None] * stages           # Q slot -> tile
        self.oslot = [None] * self.SO         # dO slot -> tile
        # per (block, quadrant): S^T / P^T / dQ columns ("S", t) / ("P", t) / ("dQ", t)
        # and dP^T / dS^T columns ("dP", t) / ("dS", t)
        self.s_cols = {k: None for k in BLOCKS}
        self.dp_cols = {k: None for k in BLOCKS}
        # per (box, quadrant) of the dS^T buffer: ("dS", t) / ("dQ", t), and whether a
        # tensor reduce is still reading the dQ staged there
        self.region = {k: None for k in REGIONS}
        self.reading = {k: False for k in REGIONS}
        self.tc_free_at = 0                   # tensor core busy until
        self.errors = []

    def fill_s(self, v):
        for k in BLOCKS:
            self.s_cols[k] = v

    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.now + dt, self.seq, fn))

    def lat(self, lo, hi):
        return self.rng.randint(lo, hi)

    # ---- tensor core: MMAs run in issue order; a commit fires after the last one
    def mma(self, dur, effect):
        start = max(self.now, self.tc_free_at)
        self.tc_free_at = start + dur
        self.seq += 1
        self.events.append((self.tc_free_at, self.seq, effect))

    def commit(self, bar):
        self.seq += 1
        self.events.append((max(self.now, self.tc_free_at), self.seq, bar.arrive))

    def run(self, roles):
        waiting = []   # (gen, bar, parity, want_completed)
        ready = [(r, None) for r in roles]
        done = 0
        steps = 0
        while True:
            steps += 1
            assert steps < 10 ** 6
            progressed = True
            while progressed:
                progressed = False
                for gen, _ in list(ready):
                    ready.remove((gen, _))
                    try:
                        op = gen.send(None)
                    except StopIteration:
                        done += 1
                        continue
                    kind = op[0]
                    if kind == "wait":
                        waiting.append((gen, op[1], op[2], op[3]))
                    elif kind == "delay":
                        self.at(op[1], lambda g=gen: ready.append((g, None)))
                    progressed = True
                still = []
                for gen, bar, par, want in waiting:
                    if bar.passes(par):
                        if bar.completed != want:
                            self.errors.append(f"{bar.name}: released at {bar.completed} completions, "
                                               f"written for {want}")
                        ready.append((gen, None))
                        progressed = True
                    else:
                        still.append((gen, bar, par, want))
                waiting = still
            if done == len(roles):
                return True
            if not self.events:
                return False   # deadlock
            self.events.sort()
            t, _, fn = self.events.pop(0)
            self.now = max(self.now, t)
            fn()


def wait(bar, k):
    """Wait for the (k+1)-th completion of bar (k = -1: the fresh barrier's 'previous' phase)."""
    parity = (k & 1) if k >= 0 else 1
    return ("wait", bar, parity, k + 1)


def producer(sim):
    def land_kv():
        sim.kv_landed = True
        sim.kv.arrive()
    sim.at(sim.lat(50, 400), land_kv)
    for t in range(sim.n_t):
        s = t % sim.S
        yield wait(sim.q_empty[s], t // sim.S - 1)

        def land(s=s, t=t):
            sim.slot[s] = t
            sim.q_full[s].arrive()
        sim.at(sim.lat(50, 600), land)
        so = t % sim.SO
        yield wait(sim.o_empty[so], t // sim.SO - 1)

        def land_o(so=so, t=t):
            sim.oslot[so] = t
            sim.o_full[so].arrive()
        sim.at(sim.lat(50, 600), land_o)
        yield ("delay", 1)


def issuer(sim, pass_blocks=kernel_pass_blocks, dp_ahead=False, dp_too_early=False):
    """The kernel's order: S^T_t, then dP^T_t once dO_t has landed.  dp_ahead: dP^T of
    tile t + 1 right after dQ_t instead, before the wait for s_free (also safe; measured
    slower).  dp_too_early (a planted mistake): dP^T of tile t + 1 right after tile t's
    s_full commit."""
    def issue_dp(t):
        so = t % sim.SO
        yield wait(sim.o_full[so], t // sim.SO)

        def mma2(t=t, so=so):
            if sim.oslot[so] != t:
                sim.errors.append(f"dP of tile {t} read dO slot holding {sim.oslot[so]}")
            for k in BLOCKS:
                if sim.dp_cols[k] not in (None, ("dS", t - 1)):
                    sim.errors.append(f"dP of tile {t} overwrote {sim.dp_cols[k]}")
                sim.dp_cols[k] = ("dP", t)
        sim.mma(sim.lat(50, 150), mma2)

    yield wait(sim.kv, 0)
    if sim.kv_in_tmem:
        yield wait(sim.kv_tmem, 0)
        if sim.k_tmem != "copied":
            sim.errors.append("S^T issued before K and V were copied into TMEM")
    dp_ahead = dp_ahead and not dp_too_early
    if dp_ahead and sim.n_t > 0:
        yield from issue_dp(0)
    for t in range(sim.n_t):
        s = t % sim.S
        so = t % sim.SO
        yield wait(sim.q_full[s], t // sim.S)
        if t > 0:
            yield wait(sim.s_free, t - 1)

        def mma1(t=t, s=s):
            if sim.slot[s] != t:
                sim.errors.append(f"S of tile {t} read Q slot holding {sim.slot[s]}")
            sim.fill_s(("S", t))
        sim.mma(sim.lat(50, 150), mma1)
        if not dp_ahead:
            yield from issue_dp(t)
        sim.commit(sim.s_full)
        if dp_too_early and t + 1 < sim.n_t:
            yield from issue_dp(t + 1)
        for h in range(2):
            yield wait(sim.p_full[h], t)
            keys = [(cb, qd) for cb in pass_blocks(h) for qd in range(4)]

            def mma3(t=t, so=so, keys=keys):
                if sim.oslot[so] != t or any(sim.s_cols[k] != ("P", t) for k in keys):
                    sim.errors.append(f"dV of tile {t} read dO {sim.oslot[so]}, P^T {[sim.s_cols[k] for k in keys]}")
            sim.mma(sim.lat(25, 75), mma3)
            if h == 1:
                sim.commit(sim.o_empty[so])

            def mma4(t=t, s=s, keys=keys):
                if sim.slot[s] != t or any(sim.dp_cols[k] != ("dS", t) for k in keys):
                    sim.errors.append(f"dK of tile {t} read Q {sim.slot[s]}, dS^T {[sim.dp_cols[k] for k in keys]}")
            sim.mma(sim.lat(25, 75), mma4)
        sim.commit(sim.q_empty[s])

        def mma5(t=t):
            if any(sim.region[k] != ("dS", t) for k in REGIONS):
                sim.errors.append(f"dQ of tile {t} read dS^T {sim.region}")
            sim.fill_s(("dQ", t))
        sim.mma(sim.lat(50, 200), mma5)
        sim.commit(sim.dq_full)
        if dp_ahead and t + 1 < sim.n_t:
            yield from issue_dp(t + 1)
        yield ("delay", 1)
    sim.commit(sim.drain)


def compute_warp(sim, w, rows_barrier, cb_of=kernel_cb):
    qd, g = w % 4, w // 4
    own = (g, qd)                       # where this warp stages dQ
    if sim.kv_in_tmem and sim.n_t > 0:
        yield wait(sim.kv, 0)
        if not sim.kv_landed:
            sim.errors.append(f"warp {w} copied K/V into TMEM before they landed")
        yield ("delay", sim.lat(20, 200))
        sim.copies = getattr(sim, "copies", 0) + 1
        if sim.copies == sim.W:
            sim.k_tmem = "copied"
        sim.kv_tmem.arrive()
    for t in range(sim.n_t):
        yield from rows_barrier(t)
        yield wait(sim.s_full, t)
        # the warp waits for its own dQ reduce to finish reading before any dS^T store
        while sim.reading[own]:
            yield ("delay", 10)
        for pass_ in range(2):
            cb = cb_of(pass_, g)
            blk, reg = (cb, qd), (cb // 2, qd)

            def ok():
                return sim.s_cols[blk] == ("S", t) and sim.dp_cols[blk] == ("dP", t)
            if not ok():
                sim.errors.append(f"warp {w} tile {t} block {cb} read {sim.s_cols[blk]} {sim.dp_cols[blk]}")
            yield ("delay", sim.lat(50, 400))
            # the block's columns must still hold this tile's S / dP when the reads end
            if not ok():
                sim.errors.append(f"warp {w} tile {t} block {cb}: S/dP overwritten during the read")
            sim.s_cols[blk], sim.dp_cols[blk] = ("P", t), ("dS", t)
            if sim.reading[reg]:
                sim.errors.append(f"warp {w} tile {t}: dS^T written over dQ staging {reg} under a reduce")
            sim.region[reg] = ("dS", t)
            sim.p_full[pass_].arrive()
        yield wait(sim.dq_full, t)
        if any(sim.s_cols[k] != ("dQ", t) for k in BLOCKS):
            sim.errors.append(f"warp {w} tile {t} read dQ from {sim.s_cols}")
        yield ("delay", sim.lat(50, 500))
        if any(sim.s_cols[k] != ("dQ", t) for k in BLOCKS):
            sim.errors.append(f"warp {w} tile {t}: dQ overwritten during the read")
        sim.s_free.arrive()
        # dQ staged in this warp's region of the dS^T buffer (the dQ product, its last
        # reader, is done), then a tensor reduce reads it asynchronously
        yield ("delay", sim.lat(20, 200))
        sim.region[own] = ("dQ", t)
        sim.reading[own] = True

        def read_done(t=t):
            if sim.region[own] != ("dQ", t):
                sim.errors.append(f"warp {w}: dQ staging of tile {t} overwritten during the reduce")
            sim.reading[own] = False
        sim.at(sim.lat(100, 3000), read_done)
    if sim.n_t > 0:
        yield wait(sim.drain, 0)


def make_named_barrier(sim):
    """bar.red over the compute warps at the top of each tile."""
    state = {"arrived": 0, "gen": 0}

    def barrier(t):
        my = state["gen"]
        state["arrived"] += 1
        if state["arrived"] == sim.W:
            state["arrived"] = 0
            state["gen"] += 1
        while state["gen"] == my:
            yield ("delay", 1)
    return barrier


@pytest.mark.parametrize("n_t", [1, 2, 3, 7])
@pytest.mark.parametrize("stages", [(1, 1), (2, 2), (2, 1)])
@pytest.mark.parametrize("dp_ahead", [True, False])
def test_backward_schedule_finishes_without_aliasing(n_t, stages, dp_ahead):
    for seed in range(25):
        # d = 64 (two Q and dO slots) keeps K and V in TMEM as well
        sim = Sim(n_t, stages[0], seed, stages_o=stages[1], kv_in_tmem=stages == (2, 2))
        nb = make_named_barrier(sim)
        roles = [producer(sim), issuer(sim, dp_ahead=dp_ahead)] + [compute_warp(sim, w, nb) for w in range(sim.W)]
        assert sim.run(roles), f"deadlock (n_t={n_t}, stages={stages}, seed={seed})"
        assert not sim.errors, sim.errors[:3]


def test_each_pass_reaches_every_block_once():
    # the compute passes and the issuer's halves name the same blocks, and each warp's
    # dS^T stays inside the box where it alone stages dQ
    for h in range(2):
        assert sorted(kernel_cb(h, g) for g in range(2)) == sorted(kernel_pass_blocks(h))
    assert sorted(kernel_cb(p, g) for p in range(2) for g in range(2)) == [0, 1, 2, 3]
    assert all(kernel_cb(p, g) // 2 == g for p in range(2) for g in range(2))
    kk = lambda h: [4 * (k4 // 2) + 2 * h + k4 % 2 for k4 in range(4)]   # the kernel's MMA steps
    assert sorted({k // 2 for k in kk(0)}) == sorted(kernel_pass_blocks(0))
    assert sorted(kk(0) + kk(1)) == list(range(8))


def team(sim, issuer_role, compute_role):
    nb = make_named_barrier(sim)   # one named barrier shared by the compute warps
    return [producer(sim), issuer_role] + [compute_role(sim, w, nb) for w in range(sim.W)]


def _finds_a_mistake(make_roles, n_t=4, stages=2, seeds=25):
    for seed in range(seeds):
        sim = Sim(n_t, stages, seed)
        if not sim.run(make_roles(sim)) or sim.errors:
            return True
    return False


def test_model_detects_a_planted_mistake():
    # the issuer no longer waits for s_free: the next tile's S overwrites dQ before it is read
    def bad_issuer(sim):
        yield wait(sim.kv, 0)
        for t in range(sim.n_t):
            s = t % sim.S
            yield wait(sim.q_full[s], t // sim.S)

            def mma12(t=t):
                sim.fill_s(("S", t))
                for k in BLOCKS:
                    sim.dp_cols[k] = ("dP", t)
            sim.mma(50, mma12)
            sim.commit(sim.s_full)
            yield wait(sim.p_full[0], t)
            yield wait(sim.p_full[1], t)
            so = t % sim.SO
            yield wait(sim.o_full[so], t // sim.SO)
            sim.mma(50, lambda: None)
            sim.commit(sim.o_empty[so])
            sim.commit(sim.q_empty[s])

            def mma5(t=t):
                sim.fill_s(("dQ", t))
            sim.mma(50, mma5)
            sim.commit(sim.dq_full)
        sim.commit(sim.drain)

    assert _finds_a_mistake(lambda sim: team(sim, bad_issuer(sim), compute_warp))


def test_model_detects_a_missing_reduce_wait():
    # a compute warp writes dS^T without waiting for its own dQ reduce to read the staging
    def bad_compute(sim, w, rows_barrier):
        qd, g = w % 4, w // 4
        own = (g, qd)
        for t in range(sim.n_t):
            yield from rows_barrier(t)
            yield wait(sim.s_full, t)
            yield ("delay", sim.lat(100, 800))
            for pass_ in range(2):
                cb = kernel_cb(pass_, g)
                sim.s_cols[(cb, qd)], sim.dp_cols[(cb, qd)] = ("P", t), ("dS", t)
                sim.region[(cb // 2, qd)] = ("dS", t)
                sim.p_full[pass_].arrive()
            yield wait(sim.dq_full, t)
            yield ("delay", sim.lat(50, 500))
            sim.s_free.arrive()
            sim.region[own] = ("dQ", t)
            sim.reading[own] = True

            def read_done(t=t):
                if sim.region[own] != ("dQ", t):
                    sim.errors.append("staging overwritten")
                sim.reading[own] = False
            sim.at(sim.lat(1000, 5000), read_done)
        if sim.n_t > 0:
            yield wait(sim.drain, 0)

    assert _finds_a_mistake(lambda sim: team(sim, issuer(sim), bad_compute), n_t=5)


def test_model_detects_a_pass_split_across_the_warps_boxes():
    # passes that split the tile into query halves 0-63 / 64-127 instead: the warp of
    # half 1 writes dS^T into box 0, where warp 0's dQ reduce may still be reading
    bad_cb = lambda p, g: 2 * p + g
    bad_blocks = lambda h: (2 * h, 2 * h + 1)

    def roles(sim):
        nb = make_named_barrier(sim)
        return [producer(sim), issuer(sim, bad_blocks)] + \
            [compute_warp(sim, w, nb, bad_cb) for w in range(sim.W)]
    assert _finds_a_mistake(roles, n_t=5)


def test_model_detects_a_second_pass_issued_early():
    # the issuer runs dV/dK of both passes after the first pass's arrivals only
    def early_issuer(sim):
        yield wait(sim.kv, 0)
        for t in range(sim.n_t):
            s = t % sim.S
            yield wait(sim.q_full[s], t // sim.S)
            if t > 0:
                yield wait(sim.s_free, t - 1)

            def mma1(t=t):
                sim.fill_s(("S", t))
                for k in BLOCKS:
                    sim.dp_cols[k] = ("dP", t)
            sim.mma(50, mma1)
            so = t % sim.SO
            yield wait(sim.o_full[so], t // sim.SO)
            sim.commit(sim.s_full)
            yield wait(sim.p_full[0], t)

            def mma3(t=t):
                if any(sim.s_cols[k] != ("P", t) for k in BLOCKS):
                    sim.errors.append(f"a block of tile {t} read before it was written")
            sim.mma(20, mma3)
            sim.commit(sim.o_empty[so])
            sim.commit(sim.q_empty[s])
            yield wait(sim.p_full[1], t)

            def mma5(t=t):
                sim.fill_s(("dQ", t))
            sim.mma(50, mma5)
            sim.commit(sim.dq_full)
        sim.commit(sim.drain)

    assert _finds_a_mistake(lambda sim: team(sim, early_issuer(sim), compute_warp), n_t=3)


def test_model_detects_the_next_dp_issued_before_dp_is_read():
    def roles(sim):
        nb = make_named_barrier(sim)
        return [producer(sim), issuer(sim, dp_too_early=True)] + \
            [compute_warp(sim, w, nb) for w in range(sim.W)]
    assert _finds_a_mistake(roles, n_t=4, stages=2)
