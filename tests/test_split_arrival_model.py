"""Model of the split-KV arrival words (split_arrive_last in fa_fwd_kernel.cuh).

Each of the n CTAs of a query block, after writing its partial, runs three atomic
steps on the block's 64-bit word: read it; if it carries another call's ticket,
compare-and-swap it to (ticket << 16) | 0 (once, no retry); add 1 and take the old
value.  The CTA whose add returns count n - 1 merges.  Here the three steps of every
CTA are interleaved in random orders (each step atomic, as on the device), starting
from random leftover contents, leftovers of an earlier call, or zero.  Checked: exactly
one CTA sees itself last, it is the last to add, and the word ends as
(ticket << 16) | n.  A planted variant that adds without claiming first fails.
"""
import random

import pytest

MASK48 = (1 << 48) - 1


def run(n, ticket, initial, order_rng, claim=True):
    word = [initial]
    state = [dict(step=0, cur=None, last=None) for _ in range(n)]
    done = []
    while len(done) < n:
        live = [i for i in range(n) if state[i]["step"] < 3]
        i = order_rng.choice(live)
        st = state[i]
        if st["step"] == 0:                       # read (atomicAdd(word, 0))
            st["cur"] = word[0]
            st["step"] = 1 if claim else 2
        elif st["step"] == 1:                     # claim once if the ticket is another call's
            if (st["cur"] >> 16) != ticket and word[0] == st["cur"]:
                word[0] = ticket << 16
            st["step"] = 2
        else:                                     # add 1, old value back
            old = word[0]
            word[0] = (old + 1) & ((1 << 64) - 1)
            st["last"] = (old & 0xFFFF) + 1 == n
            st["step"] = 3
            done.append(i)
    return word[0], [i for i in range(n) if state[i]["last"]], done


@pytest.mark.parametrize("n", [1, 2, 3, 18, 64, 256])
def test_exactly_one_last_arrival(n):
    rng = random.Random(n)
    for trial in range(300):
        ticket = rng.getrandbits(48)
        kind = trial % 3
        if kind == 0:
            initial = rng.getrandbits(64)                       # whatever the workspace held
            if (initial >> 16) == ticket:
                continue                                        # the 2^-48 collision the design accepts
        elif kind == 1:
            initial = (((ticket - 1) & MASK48) << 16) | rng.randrange(0, 257)   # an earlier call
        else:
            initial = 0                                         # zero-filled memory
        final, last, done = run(n, ticket, initial, random.Random(trial))
        assert len(last) == 1, (n, trial, last)
        assert last[0] == done[-1]
        assert final == (ticket << 16) | n


def test_zero_filled_word_and_ticket_zero():
    # a zero word already "carries" ticket 0 with count 0: still exactly one last arrival
    final, last, _ = run(5, 0, 0, random.Random(1))
    assert len(last) == 1 and final == 5


def test_model_catches_adding_without_a_claim():
    rng = random.Random(7)
    caught = False
    for trial in range(50):
        ticket = rng.getrandbits(48)
        initial = (((ticket + 3) & MASK48) << 16) | 7     # leftovers of another call
        final, last, done = run(18, ticket, initial, random.Random(trial), claim=False)
        if len(last) != 1 or last[0] != done[-1] or final != (ticket << 16) | 18:
            caught = True
            break
    assert caught
