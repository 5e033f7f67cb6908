"""Discrete-event model of the persistent forward kernel's barrier schedule
(fa_fwd_persist.cuh).

The roles of one persistent CTA, re-stated as generators over mbarriers with the
hardware's parity rule (the Barrier class and the event loop of the single-block model
are reused): the K producer (Q per block, the K ring, and the scheduler that claims the
next block after the block's last K copy and publishes it through a two-slot mailbox),
the V producer, the QK^T and PV issuers on one in-order tensor core, and the eight
softmax warps (lane quadrant q, group g = the tiles j of a block with j % 2 == g).  A
CTA takes a random sequence of blocks, some of them with no K/V tile.  Every barrier
phase is counted over all the blocks taken, as in the kernel.

Checked for every schedule:
  * no deadlock, and every wait released by exactly the phase it was written for;
  * data: QK^T reads the Q of its own block and the K tile of its global index; a
    block's Q copy lands only after every QK^T of the previous block finished; a score
    buffer is overwritten only after all four warps of its group read it; P(t) is
    written only after PV(t-3) read that buffer; an O rescale runs between PV(t-1) and
    PV(t); the first PV of a block (which starts O afresh) runs only after all eight
    softmax warps read the previous block's O; the epilogue reads O after every PV of
    its block; the epilogue exchange buffer is not overwritten before the partner
    warp read it; every mailbox reader gets the item of its own block; the reference
    max travels between the two warps of a quadrant in a word tagged with the tile's
    index over all blocks, which is read before it is overwritten.
"""
import random

import pytest

from test_bwd_protocol_model import Barrier
from test_fwd_protocol_model import Fwd, publish_max, take_max, wait


class Persist(Fwd):
    def __init__(self, blocks, ns_k, ns_v, seed, slow=1.0, v_lat=(200, 3000), n_s=1, n_p=3, p_rescale=0.3):
        super().__init__(0, ns_k, ns_v, seed, p_rescale=p_rescale, slow=slow, v_lat=v_lat, n_s=n_s, n_p=n_p)
        self.blocks = blocks             # K/V tiles of each block this CTA takes, in order
        b = Barrier
        self.q_free = b("q_free", 1)
        self.o_free = b("o_free", 8)
        self.drain = b("drain", 1)
        self.fin = b("fin", 2)
        self.clc = b("clc", 1)
        self.item_ready = [b(f"item_ready{s}", 1) for s in range(2)]
        self.item_used = [b(f"item_used{s}", 11) for s in range(2)]
        self.quad = [b(f"quad{q}", 2) for q in range(4)]   # the epilogue's named barrier
        self.go = {}                     # (q, block) -> the two warps' next-item answers
        self.mail = [None, None]
        self.q_block = None              # block whose Q is in the Q buffer
        self.qk_block_done = {}          # block -> QK^T products finished
        self.o_block = None              # block whose products O holds
        self.o_reads = {}                # block -> softmax warps that read its O
        self.pv_block = {}               # block -> PV products finished
        self.epi = {}                    # (parity, q, g) -> block written

    def n_of(self, k):
        return self.blocks[k]


def take_next(m, k):
    """A mailbox reader's next item: the block index k + 1, or None."""
    s = k & 1
    yield wait(m.item_ready[s], k >> 1)
    item = m.mail[s]
    if item is None or item[0] != k + 1:
        m.errors.append(f"mailbox slot {s} held {item} for the successor of block {k}")
    yield ("delay", m.lat(5, 40))
    m.item_used[s].arrive()
    return k + 1 if item is not None and item[1] else None


def k_producer(m):
    k, jr, nq = 0, 0, 0
    while True:
        n = m.n_of(k)
        if n > 0:
            if nq > 0:
                yield wait(m.q_free, nq - 1)
                if m.qk_block_done.get(m.q_block, 0) != m.n_of(m.q_block):
                    m.errors.append(f"Q of block {k} copied while block {m.q_block}'s QK^T ran")

            def land_q(k=k):
                m.q_block = k
                m.q_full.arrive()
            m.at(m.lat(100, 800), land_q)
            nq += 1
            for j in range(n):
                s = jr % m.nsk
                yield wait(m.ke[s], jr // m.nsk - 1)

                def land(s=s, t=jr):
                    m.kslot[s] = t
                    m.kf[s].arrive()
                m.at(m.lat(200, 3000), land)
                jr += 1
                yield ("delay", 1)
        # scheduler: claim the next block now, one request at a time
        m.at(m.lat(100, 2500), m.clc.arrive)
        yield wait(m.clc, k)
        got = k + 1 < len(m.blocks)
        s = k & 1
        if k >= 2:
            yield wait(m.item_used[s], (k - 2) >> 1)
        m.mail[s] = (k + 1, got)
        m.item_ready[s].arrive()
        if not got:
            return
        k += 1


def v_producer(m):
    k, jr = 0, 0
    while True:
        for j in range(m.n_of(k)):
            s = jr % m.nsv
            yield wait(m.ve[s], jr // m.nsv - 1)

            def land(s=s, t=jr):
                m.vslot[s] = t
                m.vf[s].arrive()
            m.at(m.lat(*m.v_lat), land)
            jr += 1
            yield ("delay", 1)
        nxt = yield from take_next(m, k)
        if nxt is None:
            return
        k = nxt


def qk_issuer(m):
    k, tt, nq = 0, 0, 0
    while True:
        n = m.n_of(k)
        if n > 0:
            yield wait(m.q_full, nq)
            for i in range(n):
                sb = tt % m.n_s
                if tt >= m.n_s:
                    yield wait(m.s_free[sb], (tt - m.n_s) // m.n_s)
                s = tt % m.nsk
                yield wait(m.kf[s], tt // m.nsk)

                def start(t=tt, s=s, sb=sb, k=k):
                    if m.kslot[s] != t:
                        m.errors.append(f"QK{t} read K slot holding {m.kslot[s]}")
                    if m.q_block != k:
                        m.errors.append(f"QK{t} of block {k} read the Q of block {m.q_block}")
                    if t >= m.n_s and not (m.s_buf[sb] == t - m.n_s and m.s_reads[sb] == 4):
                        m.errors.append(f"QK{t} overwrote S{m.s_buf[sb]} after {m.s_reads[sb]} reads")

                def end(t=tt, s=s, sb=sb, k=k):
                    if m.kslot[s] != t or m.q_block != k:
                        m.errors.append(f"QK{t}: K slot ({m.kslot[s]}) or Q ({m.q_block}) changed under it")
                    m.s_buf[sb], m.s_reads[sb] = t, 0
                    m.qk_block_done[k] = m.qk_block_done.get(k, 0) + 1
                m.mma(m.lat(300, 600), start, end)
                m.commit(m.s_full[i & 1])
                m.commit(m.ke[s])
                tt += 1
            m.commit(m.q_free)
            nq += 1
        nxt = yield from take_next(m, k)
        if nxt is None:
            break
        k = nxt
    m.commit(m.fin)
    yield wait(m.fin, 0)


def pv_issuer(m):
    k, tt, nq, prev = 0, 0, 0, None
    while True:
        n = m.n_of(k)
        if n > 0:
            if nq > 0:
                yield wait(m.o_free, nq - 1)
            for j in range(n):
                pb = tt % m.n_p
                yield wait(m.p_full[pb], tt // m.n_p)
                s = tt % m.nsv
                yield wait(m.vf[s], tt // m.nsv)

                def start(t=tt, s=s, pb=pb, j=j, k=k, prev=prev):
                    if m.vslot[s] != t:
                        m.errors.append(f"PV{t} read V slot holding {m.vslot[s]}")
                    if m.p_buf[pb] != (t, 4):
                        m.errors.append(f"PV{t} read P buffer holding {m.p_buf[pb]}")
                    if j == 0:
                        if prev is not None and m.o_reads.get(prev, 0) != 8:
                            m.errors.append(f"block {k} restarted O after {m.o_reads.get(prev, 0)} reads of "
                                            f"block {prev}'s O")
                        m.o_block = k
                    elif m.o_block != k:
                        m.errors.append(f"PV{t} of block {k} accumulates into O of block {m.o_block}")
                    m.pv_started = t

                def end(t=tt, s=s, pb=pb, k=k):
                    if m.p_buf[pb] != (t, 4) or m.vslot[s] != t:
                        m.errors.append(f"PV{t}: P buffer {m.p_buf[pb]} / V slot {m.vslot[s]} changed under it")
                    m.pv_done_count += 1
                    m.pv_block[k] = m.pv_block.get(k, 0) + 1
                m.mma(m.lat(300, 700), start, end)
                m.commit(m.pv_done[pb])
                m.commit(m.ve[s])
                tt += 1
            m.commit(m.drain)
            nq += 1
            prev = k
        nxt = yield from take_next(m, k)
        if nxt is None:
            break
        k = nxt
    m.commit(m.fin)
    yield wait(m.fin, 0)


def softmax(m, q, g):
    k, tt0, nq, sf_own, n_epi = 0, 0, 0, 0, 0
    while True:
        n = m.n_of(k)
        for j in range(g, n, 2):
            tt = tt0 + j
            yield wait(m.s_full[g], sf_own + (j >> 1))
            sb = tt % m.n_s
            if m.s_buf[sb] != tt:
                m.errors.append(f"softmax q{q} read S{m.s_buf[sb]} for tile {tt}")
            yield ("delay", m.lat(100, 300) * m.slow)
            m.s_reads[sb] += 1
            m.s_free[sb].arrive()
            yield ("delay", m.lat(20, 600) * m.slow)   # mask and row max of the scores
            if j > 0:
                yield from take_max(m, q, g, tt)   # the other warp's tile tt - 1 (same block)
            if j + 1 < n:
                publish_max(m, q, g, tt)
            pb = tt % m.n_p
            if tt >= m.n_p:
                yield wait(m.pv_done[pb], (tt - m.n_p) // m.n_p)
                if m.pv_done_count < tt - m.n_p + 1:
                    m.errors.append(f"P{tt} written before PV{tt - m.n_p} finished")
            yield ("delay", m.lat(400, 2000) * m.slow)
            cur = m.p_buf[pb]
            m.p_buf[pb] = (tt, (cur[1] + 1) if cur and cur[0] == tt else 1)
            if j > 0 and m.rng.random() < m.p_rescale:
                yield wait(m.pv_done[(tt - 1) % m.n_p], (tt - 1) // m.n_p)
                if m.pv_done_count < tt or m.pv_started >= tt:
                    m.errors.append(f"O rescale at tile {tt}: PV done {m.pv_done_count}, started {m.pv_started}")
                yield ("delay", m.lat(100, 400))
            m.p_full[pb].arrive()
        # epilogue of block k
        if n > 0:
            yield wait(m.drain, nq)
            if m.pv_block.get(k, 0) != n or m.o_block != k:
                m.errors.append(f"epilogue of block {k} after {m.pv_block.get(k, 0)} of {n} PVs (O of {m.o_block})")
        m.epi[(k & 1, q, g)] = k
        # the next block's item is read before the quadrant's barrier, so the two warps
        # take the decision to go on together (the kernel folds a read that ran out
        # into the barrier's failure flag)
        nxt = yield from take_next(m, k)
        m.go.setdefault((q, k), []).append(nxt)
        m.quad[q].arrive()
        yield wait(m.quad[q], n_epi)
        answers = m.go[(q, k)]
        if len(answers) != 2 or answers[0] != answers[1]:
            m.errors.append(f"q{q}: the warps of a quadrant disagree after block {k}: {answers}")
        n_epi += 1
        yield ("delay", m.lat(1, 300))
        if m.epi.get((k & 1, q, g ^ 1)) != k:
            m.errors.append(f"q{q} g{g}: epilogue exchange of block {k} holds {m.epi.get((k & 1, q, g ^ 1))}")
        if n > 0:
            yield ("delay", m.lat(50, 400))
            if m.o_block != k:
                m.errors.append(f"block {k}'s O overwritten by block {m.o_block} before it was read")
            m.o_reads[k] = m.o_reads.get(k, 0) + 1
            m.o_free.arrive()
            tt0 += n
            sf_own += (n + 1) // 2 if g == 0 else n // 2
            nq += 1
        if nxt is None:
            return
        k = nxt


def roles(m, kp=k_producer, vp=v_producer, qk=qk_issuer, pv=pv_issuer, sm=softmax):
    r = [kp(m), vp(m), qk(m), pv(m)]
    return r + [sm(m, q, g) for q in range(4) for g in range(2)]


def random_blocks(rng):
    return [rng.choice([0, 1, 1, 2, 3, 4, 5, 7]) for _ in range(rng.randint(1, 6))]


# K / V ring slots, TMEM score buffers, TMEM P buffers (the kernel: 4/4 or 2/2, 1, 3)
CONFIGS = [(4, 4, 1, 3), (2, 2, 1, 3), (4, 4, 1, 2)]


@pytest.mark.parametrize("slots", CONFIGS)
def test_persistent_schedule_finishes_without_aliasing(slots):
    for seed in range(60):
        rng = random.Random(1000 + seed)
        blocks = random_blocks(rng)
        for slow, v_lat in ((0.3, (200, 3000)), (1.0, (200, 3000)), (3.0, (200, 3000)), (1.0, (3000, 9000))):
            m = Persist(blocks, slots[0], slots[1], seed, slow=slow, v_lat=v_lat, n_s=slots[2], n_p=slots[3])
            assert m.run(roles(m)), f"deadlock blocks={blocks} slots={slots} seed={seed}"
            assert not m.errors, (blocks, m.errors[:3])


def test_edge_sequences():
    for blocks in ([0], [1], [0, 0, 0], [0, 3, 0, 1], [1, 1, 1, 1, 1, 1, 1], [9, 0, 9], [2, 13, 1]):
        for seed in range(10):
            m = Persist(blocks, 2, 2, seed)
            assert m.run(roles(m)), f"deadlock {blocks}"
            assert not m.errors, (blocks, m.errors[:3])


def test_two_score_buffers_are_unsafe_across_blocks():
    # With two score buffers the QK^T issuer may run two tiles ahead; at a block
    # boundary the block-local parity of s_full and the global score buffer no longer
    # match, and s_full(g) can complete twice before group g waits once.  The kernel
    # therefore keeps a single score buffer (static_assert in fa_fwd_persist.cuh).
    bad = False
    for seed in range(60):
        rng = random.Random(1000 + seed)
        blocks = random_blocks(rng)
        m = Persist(blocks, 2, 2, seed, n_s=2, n_p=2)
        if not m.run(roles(m)) or m.errors:
            bad = True
            break
    assert bad


def test_model_detects_missing_o_free_wait():
    # the PV issuer starts a block's O without waiting for the softmax warps to read
    # the previous block's O out of TMEM
    def bad_pv(m):
        k, tt, prev = 0, 0, None
        while True:
            n = m.n_of(k)
            for j in range(n):
                pb = tt % m.n_p
                yield wait(m.p_full[pb], tt // m.n_p)
                s = tt % m.nsv
                yield wait(m.vf[s], tt // m.nsv)

                def start(j=j, k=k, prev=prev):
                    if j == 0:
                        if prev is not None and m.o_reads.get(prev, 0) != 8:
                            m.errors.append("O restarted early")
                        m.o_block = k
                    m.pv_started = tt

                def end(k=k):
                    m.pv_done_count += 1
                    m.pv_block[k] = m.pv_block.get(k, 0) + 1
                m.mma(m.lat(300, 700), start, end)
                m.commit(m.pv_done[pb])
                m.commit(m.ve[s])
                tt += 1
            if n > 0:
                m.commit(m.drain)
                prev = k
            nxt = yield from take_next(m, k)
            if nxt is None:
                break
            k = nxt
        m.commit(m.fin)
        yield wait(m.fin, 0)

    caught = False
    for seed in range(60):
        m = Persist([1, 1, 2, 1, 1], 4, 4, seed, slow=3.0)
        if not m.run(roles(m, pv=bad_pv)) or m.errors:
            caught = True
            break
    assert caught


def test_model_detects_missing_q_free_wait():
    # the K producer copies the next block's Q without waiting for q_free
    def bad_k(m):
        k, jr = 0, 0
        while True:
            n = m.n_of(k)
            if n > 0:
                def land_q(k=k):
                    m.q_block = k
                    m.q_full.arrive()
                m.at(m.lat(100, 800), land_q)
                for j in range(n):
                    s = jr % m.nsk
                    yield wait(m.ke[s], jr // m.nsk - 1)

                    def land(s=s, t=jr):
                        m.kslot[s] = t
                        m.kf[s].arrive()
                    m.at(m.lat(200, 3000), land)
                    jr += 1
                    yield ("delay", 1)
            m.at(m.lat(10, 50), m.clc.arrive)
            yield wait(m.clc, k)
            got = k + 1 < len(m.blocks)
            s = k & 1
            if k >= 2:
                yield wait(m.item_used[s], (k - 2) >> 1)
            m.mail[s] = (k + 1, got)
            m.item_ready[s].arrive()
            if not got:
                return
            k += 1

    caught = False
    for seed in range(60):
        m = Persist([3, 3, 3, 3], 4, 4, seed)
        if not m.run(roles(m, kp=bad_k)) or m.errors:
            caught = True
            break
    assert caught
