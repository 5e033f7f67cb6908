"""Model of the backward kernel's wind-down after a bounded wait ran out
(fa_bwd_kernel.cuh, producer and MMA issuer).

The producer copies tile t into ring slot t % S once the consumer (the MMA
issuer) has freed that slot; each copy lands after a random latency.  At a
random point the consumer's wait runs out: it raises the CTA's abort flag and
stops, and the CTA releases its shared memory once every role has finished.  A
producer that sees the abort while it waits for a free slot stops too.  The rule
in the kernel: before finishing, the producer waits for the newest copy of every
slot, always -- also when it had already issued its last copy and never saw the
abort itself.  Checked: no copy lands after the CTA has released its memory.
A planted producer that waits only when it gave up itself is caught.
"""
import random

import pytest


def simulate(n_t, S, seed, always=True):
    rng = random.Random(seed)
    land = {}                                    # copy -> time it lands
    free = {}                                    # copy -> time its slot was freed
    abort_at = None
    fail_tile = rng.choice([None] + list(range(n_t)))
    t_prod = 0.0                                 # producer clock
    t_cons = 0.0                                 # consumer clock
    issued = 0
    own_fail = False
    # the two roles, stepped in time order: the producer issues copy `issued` when
    # its slot is free; the consumer takes copy `c` when it has landed
    c = 0
    while True:
        # next producer action time
        p_next = None
        if issued < n_t and not own_fail:
            need = free.get(issued - S, 0.0) if issued >= S else 0.0
            if issued >= S and (issued - S) not in free:
                need = None                      # slot not freed yet
            if need is not None:
                p_next = max(t_prod, need) + 1.0
        # next consumer action time
        q_next = None
        if abort_at is None and c < n_t and c in land:
            q_next = max(t_cons, land[c])
        if abort_at is None and c < n_t and fail_tile == c:
            # this wait runs out a little before the copy lands (or right away)
            give_up = t_cons + rng.uniform(1.0, 50.0)
            if c not in land or give_up < land[c]:
                q_next = None
                if p_next is None or give_up <= p_next:
                    abort_at = give_up
                    t_cons = give_up
                    continue
        if p_next is None and q_next is None:
            if issued < n_t and not own_fail and abort_at is not None:
                # the producer waits for a slot nobody will free: its bounded wait
                # sees the abort flag and it gives up too
                own_fail = True
                t_prod = max(t_prod, abort_at)
            break
        if q_next is not None and (p_next is None or q_next <= p_next):
            t_cons = q_next + rng.uniform(20.0, 200.0)   # the products of tile c
            free[c] = t_cons
            c += 1
        else:
            if abort_at is not None and p_next > abort_at:
                own_fail = True                  # the slot wait sees the abort
                t_prod = max(t_prod, abort_at)
                continue
            t_prod = p_next
            land[issued] = t_prod + rng.uniform(50.0, 3000.0)
            issued += 1
        if abort_at is None and c >= n_t:
            break
    # wind-down
    prod_exit = t_prod
    if always or own_fail:
        newest = range(max(0, issued - S), issued)
        prod_exit = max([prod_exit] + [land[i] for i in newest])
    cons_exit = abort_at if abort_at is not None else t_cons
    release = max(prod_exit, cons_exit)
    late = [i for i in range(issued) if land[i] > release]
    return late, abort_at is not None


@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("n_t", [1, 2, 3, 5, 9])
def test_no_copy_lands_after_release(S, n_t):
    aborts = 0
    for seed in range(300):
        late, aborted = simulate(n_t, S, seed)
        aborts += aborted
        assert not late, (n_t, S, seed, late)
    assert aborts > 0                            # the abort path was exercised


def test_model_catches_a_producer_that_waits_only_after_its_own_give_up():
    caught = False
    for seed in range(300):
        late, _ = simulate(3, 2, seed, always=False)
        if late:
            caught = True
            break
    assert caught
