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


class Sim:
    def __init__(self, n_t, stages, seed, warps=8, stages_o=None):
        self.rng = random.Random(seed)
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
        self.s_full, self.p_full = b("s_full", 1), b("p_full", warps)
        self.dq_full, self.s_free = b("dq_full", 1), b("s_free", warps)
        self.drain = b("drain", 1)
        # buffer contents: which tile's data they hold
        self.slot = [None] * stages           # Q slot -> tile
        self.oslot = [None] * self.SO         # dO slot -> tile
        self.s_cols = None                    # S^T / P^T / dQ columns: ("S", t) / ("dQ", t)
        self.dp_cols = None                   # dP^T / dS^T columns
        self.ds_smem = None                   # dS^T in shared memory
        self.stage = [None] * warps           # each warp's part of that buffer: ("dS", t) / ("dQ", t)
        self.reading = [False] * warps        # a tensor reduce is still reading the warp's dQ staging
        self.tc_free_at = 0                   # tensor core busy until
        self.errors = []

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
    sim.at(sim.lat(50, 400), sim.kv.arrive)
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


def issuer(sim):
    yield wait(sim.kv, 0)
    for t in range(sim.n_t):
        s = t % sim.S
        yield wait(sim.q_full[s], t // sim.S)
        if t > 0:
            yield wait(sim.s_free, t - 1)

        def mma1(t=t, s=s):
            if sim.slot[s] != t:
                sim.errors.append(f"S of tile {t} read Q slot holding {sim.slot[s]}")
            sim.s_cols = ("S", t)
        sim.mma(sim.lat(50, 150), mma1)
        so = t % sim.SO
        yield wait(sim.o_full[so], t // sim.SO)

        def mma2(t=t, so=so):
            if sim.oslot[so] != t:
                sim.errors.append(f"dP of tile {t} read dO slot holding {sim.oslot[so]}")
            sim.dp_cols = ("dP", t)
        sim.mma(sim.lat(50, 150), mma2)
        sim.commit(sim.s_full)
        yield wait(sim.p_full, t)

        def mma3(t=t, so=so):
            if sim.oslot[so] != t or sim.s_cols != ("P", t):
                sim.errors.append(f"dV of tile {t} read dO {sim.oslot[so]}, {sim.s_cols}")
        sim.mma(sim.lat(50, 150), mma3)
        sim.commit(sim.o_empty[so])

        def mma4(t=t, s=s):
            if sim.slot[s] != t or sim.dp_cols != ("dS", t):
                sim.errors.append(f"dK of tile {t} read Q {sim.slot[s]}, {sim.dp_cols}")
        sim.mma(sim.lat(50, 150), mma4)
        sim.commit(sim.q_empty[s])

        def mma5(t=t):
            if sim.ds_smem != t or any(st != ("dS", t) for st in sim.stage):
                sim.errors.append(f"dQ of tile {t} read dS^T of {sim.ds_smem} / {sim.stage}")
            sim.s_cols = ("dQ", t)
        sim.mma(sim.lat(50, 200), mma5)
        sim.commit(sim.dq_full)
        yield ("delay", 1)
    sim.commit(sim.drain)


def compute_warp(sim, w, rows_barrier):
    for t in range(sim.n_t):
        yield from rows_barrier(t)
        yield wait(sim.s_full, t)
        if sim.s_cols not in (("S", t), ("P", t)) or sim.dp_cols not in (("dP", t), ("dS", t)):
            sim.errors.append(f"warp {w} tile {t} read {sim.s_cols} {sim.dp_cols}")
        yield ("delay", sim.lat(100, 800))
        # the columns must still hold this tile's S / dP (or the other warps' P / dS)
        # when the reads end
        if sim.s_cols not in (("S", t), ("P", t)) or sim.dp_cols not in (("dP", t), ("dS", t)):
            sim.errors.append(f"warp {w} tile {t}: S/dP overwritten during the read")
        # dS^T goes where this warp staged the previous tile's dQ: its reduce must be done reading
        while sim.reading[w]:
            yield ("delay", 10)
        sim.stage[w] = ("dS", t)
        sim.s_cols, sim.dp_cols, sim.ds_smem = ("P", t), ("dS", t), t
        sim.p_full.arrive()
        yield wait(sim.dq_full, t)
        if sim.s_cols != ("dQ", t):
            sim.errors.append(f"warp {w} tile {t} read dQ from {sim.s_cols}")
        yield ("delay", sim.lat(50, 500))
        if sim.s_cols != ("dQ", t):
            sim.errors.append(f"warp {w} tile {t}: dQ overwritten during the read")
        sim.s_free.arrive()
        # dQ staged in this warp's part of the dS^T buffer (the dQ product, its last
        # reader, is done), then a tensor reduce reads it asynchronously
        yield ("delay", sim.lat(20, 200))
        sim.stage[w] = ("dQ", t)
        sim.reading[w] = True

        def read_done(w=w, t=t):
            if sim.stage[w] != ("dQ", t):
                sim.errors.append(f"warp {w}: dQ staging of tile {t} overwritten during the reduce")
            sim.reading[w] = False
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
def test_backward_schedule_finishes_without_aliasing(n_t, stages):
    for seed in range(25):
        sim = Sim(n_t, stages[0], seed, stages_o=stages[1])
        nb = make_named_barrier(sim)
        roles = [producer(sim), issuer(sim)] + [compute_warp(sim, w, nb) for w in range(sim.W)]
        assert sim.run(roles), f"deadlock (n_t={n_t}, stages={stages}, seed={seed})"
        assert not sim.errors, sim.errors[:3]


def test_model_detects_a_planted_mistake():
    # the issuer no longer waits for s_free: the next tile's S overwrites dQ before it is read
    def bad_issuer(sim):
        yield wait(sim.kv, 0)
        for t in range(sim.n_t):
            s = t % sim.S
            yield wait(sim.q_full[s], t // sim.S)

            def mma12(t=t):
                sim.s_cols, sim.dp_cols = ("S", t), ("dP", t)
            sim.mma(50, mma12)
            sim.commit(sim.s_full)
            yield wait(sim.p_full, t)
            so = t % sim.SO
            yield wait(sim.o_full[so], t // sim.SO)
            sim.mma(50, lambda: None)
            sim.commit(sim.o_empty[so])
            sim.commit(sim.q_empty[s])

            def mma5(t=t):
                sim.s_cols = ("dQ", t)
            sim.mma(50, mma5)
            sim.commit(sim.dq_full)
        sim.commit(sim.drain)

    found = False
    for seed in range(25):
        sim = Sim(4, 2, seed)
        nb = make_named_barrier(sim)
        roles = [producer(sim), bad_issuer(sim)] + [compute_warp(sim, w, nb) for w in range(sim.W)]
        ok = sim.run(roles)
        if not ok or sim.errors:
            found = True
            break
    assert found


def test_model_detects_a_missing_reduce_wait():
    # a compute warp writes dS^T without waiting for its dQ reduce to read the staging
    def bad_compute(sim, w, rows_barrier):
        for t in range(sim.n_t):
            yield from rows_barrier(t)
            yield wait(sim.s_full, t)
            yield ("delay", sim.lat(100, 800))
            sim.stage[w] = ("dS", t)
            sim.s_cols, sim.dp_cols, sim.ds_smem = ("P", t), ("dS", t), t
            sim.p_full.arrive()
            yield wait(sim.dq_full, t)
            yield ("delay", sim.lat(50, 500))
            sim.s_free.arrive()
            sim.stage[w] = ("dQ", t)
            sim.reading[w] = True

            def read_done(w=w, t=t):
                if sim.stage[w] != ("dQ", t):
                    sim.errors.append("staging overwritten")
                sim.reading[w] = False
            sim.at(sim.lat(1000, 5000), read_done)
        if sim.n_t > 0:
            yield wait(sim.drain, 0)

    found = False
    for seed in range(25):
        sim = Sim(5, 2, seed)
        nb = make_named_barrier(sim)
        roles = [producer(sim), issuer(sim)] + [bad_compute(sim, w, nb) for w in range(sim.W)]
        if not sim.run(roles) or sim.errors:
            found = True
            break
    assert found
