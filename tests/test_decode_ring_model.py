"""Discrete-event model of the single-row decode kernel's K/V ring
(fa_decode_kernel.cuh).

Roles of one CTA: the producer lane copies K/V tile j into ring slot j % S once
all eight compute warps have released that slot (empty barrier, eight arrivals),
the copy landing after a random latency completes the slot's full barrier; each
compute warp waits for tile j's full phase, reads the slot for a random time,
and arrives on the slot's empty barrier.  Waits follow the mbarrier parity rule
(the Barrier class of the backward model).  Checked for every schedule: no
deadlock, every wait released by exactly the phase it was written for, and every
warp reads tile j from its slot while the slot still holds tile j (no copy lands
over a tile a warp is still reading).  Planted mistakes are caught: a producer
that waits for only one warp's release, and a warp that never releases a slot.
"""
import random

import pytest

from test_bwd_protocol_model import Barrier

WARPS = 8


def wait(bar, k):
    """Wait for the (k+1)-th completion of bar (k = -1: the fresh barrier's 'previous' phase)."""
    parity = (k & 1) if k >= 0 else 1
    return ("wait", bar, parity, k + 1)


class Ring:
    def __init__(self, n_t, stages, seed, empty_count=WARPS):
        self.rng = random.Random(seed)
        self.n_t, self.S = n_t, stages
        self.full = [Barrier(f"full{s}", 1) for s in range(stages)]
        self.empty = [Barrier(f"empty{s}", empty_count) for s in range(stages)]
        self.slot = [None] * stages          # tile a slot holds
        self.now, self.seq, self.events = 0.0, 0, []
        self.errors = []

    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.now + dt, self.seq, fn))

    def run(self, roles):
        waiting, ready, done = [], [(r, None) for r in roles], 0
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
                    if op[0] == "wait":
                        waiting.append((gen, op[1], op[2], op[3]))
                    else:
                        self.at(op[1], lambda g=gen: ready.append((g, None)))
                    progressed = True
                still = []
                for gen, bar, par, want in waiting:
                    if bar.passes(par):
                        if bar.completed != want:
                            self.errors.append(f"{bar.name}: released at {bar.completed}, written for {want}")
                        ready.append((gen, None))
                        progressed = True
                    else:
                        still.append((gen, bar, par, want))
                waiting = still
            if done == len(roles):
                return True
            if not self.events:
                return False
            self.events.sort()
            t, _, fn = self.events.pop(0)
            self.now = max(self.now, t)
            fn()


def producer(m):
    for j in range(m.n_t):
        s = j % m.S
        yield wait(m.empty[s], j // m.S - 1)

        def land(s=s, j=j):
            m.slot[s] = j
            m.full[s].arrive()
        m.at(m.rng.uniform(50, 3000), land)
        yield ("delay", 1)


def compute(m, w, release=True):
    for j in range(m.n_t):
        s = j % m.S
        yield wait(m.full[s], j // m.S)
        if m.slot[s] != j:
            m.errors.append(f"warp {w} tile {j}: slot {s} holds {m.slot[s]}")
        yield ("delay", m.rng.uniform(20, 400))
        if m.slot[s] != j:
            m.errors.append(f"warp {w} tile {j}: slot {s} overwritten by {m.slot[s]} during the read")
        if release:
            m.empty[s].arrive()


@pytest.mark.parametrize("stages", [1, 2, 3, 6])
@pytest.mark.parametrize("n_t", [0, 1, 2, 5, 29])
def test_decode_ring_finishes_without_aliasing(n_t, stages):
    for seed in range(30):
        m = Ring(n_t, stages, seed)
        assert m.run([producer(m)] + [compute(m, w) for w in range(WARPS)]), (n_t, stages, seed)
        assert not m.errors, m.errors[:3]


def test_model_catches_a_producer_that_waits_for_one_warp():
    caught = False
    for seed in range(30):
        m = Ring(9, 2, seed, empty_count=1)
        # every warp still arrives: the empty barrier now completes once per arrival
        ok = m.run([producer(m)] + [compute(m, w) for w in range(WARPS)])
        if not ok or m.errors:
            caught = True
            break
    assert caught


def test_model_catches_a_warp_that_never_releases_its_slot():
    m = Ring(7, 3, 0)
    roles = [producer(m)] + [compute(m, w, release=(w != 5)) for w in range(WARPS)]
    assert not m.run(roles)   # the producer waits for slot 0 forever: a deadlock
