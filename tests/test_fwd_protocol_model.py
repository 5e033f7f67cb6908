"""Discrete-event model of the forward kernel's barrier schedule (fa_fwd_kernel.cuh,
dense single-pass mode).

Roles of one CTA, re-stated as generators over mbarriers with the hardware's parity
rule: the K producer (Q once, then the K ring), the V producer (V ring), the QK^T
issuer and the PV issuer sharing one in-order tensor core, and the eight softmax
warps (lane quadrant q, group g = the tiles j with j % 2 == g).  Random latencies for
copies, MMAs and softmax work; a random subset of tiles takes the O-rescale branch.
Checked for every schedule:
  * no deadlock;
  * every wait is released by exactly the phase it was written for (no parity
    aliasing);
  * data: QK^T(i) reads K_i and PV(j) reads V_j from their ring slots; a score buffer
    is overwritten only after all four warps of its group read it; P(j) is written
    only after PV(j-3) finished reading that P buffer and PV(j) reads P(j) complete;
    an O rescale at tile j runs after PV(j-1) and before PV(j); the epilogue reads O
    after every PV.
The reference max of tile j goes from warp (q, g) to warp (q, g ^ 1) in a shared word
tagged with j, written in one store; the reader polls until the tag names the tile it
needs.  Checked as well: the reader gets that tile's max, and no word is overwritten
before its reader took it (a warp reads the other's word for tile j - 1 before it
publishes tile j).  A planted writer that publishes before it reads is caught.
"""
import random

import pytest

from test_bwd_protocol_model import Barrier


class Fwd:
    def __init__(self, n, ns_k, ns_v, seed, p_rescale=0.3, slow=1.0, v_lat=(200, 3000), n_s=1, n_p=3):
        self.rng = random.Random(seed)
        self.n_s, self.n_p = n_s, n_p    # TMEM score buffers, P buffers
        self.v_lat = v_lat
        self.n, self.nsk, self.nsv, self.p_rescale, self.slow = n, ns_k, ns_v, p_rescale, slow
        self.now, self.seq, self.events, self.tc_free = 0.0, 0, [], 0.0
        b = Barrier
        self.q_full = b("q_full", 1)
        self.kf = [b(f"k_full{s}", 1) for s in range(ns_k)]
        self.ke = [b(f"k_empty{s}", 1) for s in range(ns_k)]
        self.vf = [b(f"v_full{s}", 1) for s in range(ns_v)]
        self.ve = [b(f"v_empty{s}", 1) for s in range(ns_v)]
        self.s_full = [b(f"s_full{g}", 1) for g in range(2)]
        self.s_free = [b(f"s_free{i}", 4) for i in range(n_s)]
        self.p_full = [b(f"p_full{i}", 4) for i in range(n_p)]
        self.pv_done = [b(f"pv_done{i}", 1) for i in range(n_p)]
        self.drain = b("drain", 2)
        self.kslot, self.vslot = [None] * ns_k, [None] * ns_v
        self.s_buf = [None] * n_s        # tile held by each score buffer
        self.s_reads = [0] * n_s         # quadrants that have read it
        self.p_buf = [None] * n_p        # (tile, quadrants written)
        self.pv_done_count = 0           # PVs finished
        self.pv_started = -1             # last PV started
        self.word = {}                   # (q, g) -> tile tag of the published max
        self.word_read = {}              # (q, g) -> last tag the other warp took
        self.errors = []

    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.now + dt, self.seq, fn))

    def lat(self, lo, hi):
        return self.rng.uniform(lo, hi)

    def mma(self, dur, start_fn, end_fn):
        start = max(self.now, self.tc_free)
        self.tc_free = start + dur
        self.seq += 1
        self.events.append((start, self.seq, start_fn))
        self.seq += 1
        self.events.append((self.tc_free, self.seq, end_fn))

    def commit(self, bar):
        self.seq += 1
        self.events.append((max(self.now, self.tc_free) + 1e-6, self.seq, bar.arrive))

    def run(self, roles):
        waiting, ready, done = [], list(roles), 0
        while True:
            progressed = True
            while progressed:
                progressed = False
                for gen in list(ready):
                    ready.remove(gen)
                    try:
                        op = gen.send(None)
                    except StopIteration:
                        done += 1
                        continue
                    if op[0] == "wait":
                        waiting.append((gen,) + op[1:])
                    else:
                        self.at(op[1], lambda g=gen: ready.append(g))
                    progressed = True
                still = []
                for gen, bar, par, want in waiting:
                    if bar.passes(par):
                        if bar.completed != want:
                            self.errors.append(f"{bar.name}: released at {bar.completed}, written for {want}")
                        ready.append(gen)
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


def wait(bar, k):
    return ("wait", bar, (k & 1) if k >= 0 else 1, k + 1)


def k_producer(m):
    m.at(m.lat(100, 800), m.q_full.arrive)
    for j in range(m.n):
        s = j % m.nsk
        yield wait(m.ke[s], j // m.nsk - 1)

        def land(s=s, j=j):
            m.kslot[s] = j
            m.kf[s].arrive()
        m.at(m.lat(200, 3000), land)
        yield ("delay", 1)


def v_producer(m):
    for j in range(m.n):
        s = j % m.nsv
        yield wait(m.ve[s], j // m.nsv - 1)

        def land(s=s, j=j):
            m.vslot[s] = j
            m.vf[s].arrive()
        m.at(m.lat(*m.v_lat), land)
        yield ("delay", 1)


def qk_issuer(m):
    if m.n == 0:
        return
    yield wait(m.q_full, 0)
    for i in range(m.n):
        sb = i % m.n_s
        if i >= m.n_s:
            yield wait(m.s_free[sb], (i - m.n_s) // m.n_s)
        s = i % m.nsk
        yield wait(m.kf[s], i // m.nsk)

        def start(i=i, s=s, sb=sb):
            if m.kslot[s] != i:
                m.errors.append(f"QK{i} read K slot holding {m.kslot[s]}")
            if i >= m.n_s and not (m.s_buf[sb] == i - m.n_s and m.s_reads[sb] == 4):
                m.errors.append(f"QK{i} overwrote S{m.s_buf[sb]} after {m.s_reads[sb]} reads")

        def end(i=i, s=s, sb=sb):
            if m.kslot[s] != i:
                m.errors.append(f"QK{i}: K slot changed under it ({m.kslot[s]})")
            m.s_buf[sb], m.s_reads[sb] = i, 0
        m.mma(m.lat(300, 600), start, end)
        m.commit(m.s_full[i & 1])
        m.commit(m.ke[s])
    m.commit(m.drain)


def pv_issuer(m):
    if m.n == 0:
        return
    for j in range(m.n):
        pb = j % m.n_p
        yield wait(m.p_full[pb], j // m.n_p)
        s = j % m.nsv
        yield wait(m.vf[s], j // m.nsv)

        def start(j=j, s=s, pb=pb):
            if m.vslot[s] != j:
                m.errors.append(f"PV{j} read V slot holding {m.vslot[s]}")
            if m.p_buf[pb] != (j, 4):
                m.errors.append(f"PV{j} read P buffer holding {m.p_buf[pb]}")
            m.pv_started = j

        def end(j=j, s=s, pb=pb):
            # the operands must still be there when the product finishes reading them
            if m.p_buf[pb] != (j, 4) or m.vslot[s] != j:
                m.errors.append(f"PV{j}: P buffer {m.p_buf[pb]} / V slot {m.vslot[s]} changed under it")
            m.pv_done_count += 1
        m.mma(m.lat(300, 700), start, end)
        m.commit(m.pv_done[pb])
        m.commit(m.ve[s])
    m.commit(m.drain)


def take_max(m, q, g, j):
    # poll the other warp's word until it carries tile j - 1
    polls = 0
    while m.word.get((q, g ^ 1)) != j - 1:
        polls += 1
        assert polls < 10 ** 5, "poll never satisfied"
        yield ("delay", m.lat(5, 40))
    m.word_read[(q, g ^ 1)] = j - 1


def publish_max(m, q, g, j):
    prev = m.word.get((q, g))
    if prev is not None and m.word_read.get((q, g)) != prev:
        m.errors.append(f"q{q}: max of tile {prev} overwritten by tile {j} before it was read")
    m.word[(q, g)] = j


def exchange_max(m, q, g, j, publish_first=False):
    if publish_first and j + 1 < m.n:
        publish_max(m, q, g, j)
    if j > 0:
        yield from take_max(m, q, g, j)
    if not publish_first and j + 1 < m.n:
        publish_max(m, q, g, j)


def softmax(m, q, g, publish_first=False):
    for j in range(g, m.n, 2):
        yield wait(m.s_full[g], j >> 1)
        sb = j % m.n_s
        if m.s_buf[sb] != j:
            m.errors.append(f"softmax q{q} read S{m.s_buf[sb]} for tile {j}")
        yield ("delay", m.lat(100, 300) * m.slow)
        m.s_reads[sb] += 1
        m.s_free[sb].arrive()
        yield ("delay", m.lat(20, 600) * m.slow)   # mask and row max of the scores
        yield from exchange_max(m, q, g, j, publish_first)
        pb = j % m.n_p
        if j >= m.n_p:
            yield wait(m.pv_done[pb], (j - m.n_p) // m.n_p)
            if m.pv_done_count < j - m.n_p + 1:
                m.errors.append(f"P{j} written before PV{j - m.n_p} finished")
        yield ("delay", m.lat(400, 2000) * m.slow)
        cur = m.p_buf[pb]
        m.p_buf[pb] = (j, (cur[1] + 1) if cur and cur[0] == j else 1)
        if j > 0 and m.rng.random() < m.p_rescale:
            yield wait(m.pv_done[(j - 1) % m.n_p], (j - 1) // m.n_p)
            if m.pv_done_count < j or m.pv_started >= j:
                m.errors.append(f"O rescale at tile {j}: PV done {m.pv_done_count}, started {m.pv_started}")
            yield ("delay", m.lat(100, 400))
        m.p_full[pb].arrive()
    if m.n > 0:
        yield wait(m.drain, 0)
        if m.pv_done_count != m.n:
            m.errors.append(f"epilogue after {m.pv_done_count} of {m.n} PVs")


# K / V ring slots, TMEM score buffers, TMEM P buffers
CONFIGS = [(4, 4, 1, 3), (2, 2, 1, 3), (4, 4, 2, 2), (2, 2, 2, 2), (4, 4, 1, 2)]


@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 5, 8, 13])
@pytest.mark.parametrize("slots", CONFIGS)
def test_forward_schedule_finishes_without_aliasing(n, slots):
    for seed in range(20):
        for slow, v_lat in ((0.3, (200, 3000)), (1.0, (200, 3000)), (3.0, (200, 3000)),
                            (1.0, (3000, 9000))):
            m = Fwd(n, slots[0], slots[1], seed, slow=slow, v_lat=v_lat, n_s=slots[2], n_p=slots[3])
            roles = [k_producer(m), v_producer(m), qk_issuer(m), pv_issuer(m)]
            roles += [softmax(m, q, g) for q in range(4) for g in range(2)]
            assert m.run(roles), f"deadlock n={n} slots={slots} seed={seed}"
            assert not m.errors, m.errors[:3]


def test_model_detects_a_planted_mistake():
    # the softmax no longer waits for PV(j-3) before writing P(j) into its buffer
    def bad_softmax(m, q, g):
        for j in range(g, m.n, 2):
            yield wait(m.s_full[g], j >> 1)
            yield ("delay", m.lat(100, 300))
            m.s_reads[0] += 1
            m.s_free[0].arrive()
            yield from exchange_max(m, q, g, j)
            pb = j % 3
            yield ("delay", m.lat(50, 200))
            cur = m.p_buf[pb]
            m.p_buf[pb] = (j, (cur[1] + 1) if cur and cur[0] == j else 1)
            m.p_full[pb].arrive()
        if m.n > 0:
            yield wait(m.drain, 0)

    caught = False
    for seed in range(40):
        m = Fwd(9, 2, 2, seed, v_lat=(3000, 9000))   # slow V: PV lags the softmax
        roles = [k_producer(m), v_producer(m), qk_issuer(m), pv_issuer(m)]
        roles += [bad_softmax(m, q, g) for q in range(4) for g in range(2)]
        if not m.run(roles) or m.errors:
            caught = True
            break
    assert caught


def test_model_detects_a_max_published_before_the_other_is_read():
    # a warp that publishes tile j's max before taking the other warp's tile j - 1:
    # the other warp can then publish j + 1 over the word this one has not read yet
    caught = False
    for seed in range(40):
        m = Fwd(9, 2, 2, seed, slow=3.0)
        roles = [k_producer(m), v_producer(m), qk_issuer(m), pv_issuer(m)]
        roles += [softmax(m, q, g, publish_first=True) for q in range(4) for g in range(2)]
        try:
            ok = m.run(roles)
        except AssertionError:
            ok = False
        if not ok or m.errors:
            caught = True
            break
    assert caught
