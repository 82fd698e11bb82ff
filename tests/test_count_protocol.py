"""The segment counters' count-in protocol, modelled on the host.

A segment cut into n pieces is merged by the CTA that stores its last piece:
every piece counts itself in on the segment's 64-bit counter, tagged with the
launch's epoch (epoch << 16 | pieces counted), and the one that brings the
count to n merges. The decode kernel reads the counter early (a guess), then:
a counter already tagged with this launch's epoch takes a plain atomic add; one
an older launch left is re-tagged to (epoch << 16 | 1) by a CAS, retried with
what the CAS returns. This models that loop over atomic operations on one
shared word, with every interleaving of the pieces' steps drawn at random, and
checks what the merge relies on: the counts the pieces see are exactly 1 .. n
(so exactly one piece sees n), whatever the counter held before the launch,
and the counter ends at (epoch << 16 | n).
"""
import random

import pytest

MASK48 = (1 << 48) - 1


class Word:
    """One 64-bit word with the two atomics the protocol uses."""

    def __init__(self, v):
        self.v = v & ((1 << 64) - 1)

    def add(self, x):
        old = self.v
        self.v = (self.v + x) & ((1 << 64) - 1)
        return old

    def cas(self, expect, new):
        old = self.v
        if old == expect:
            self.v = new
        return old


def piece(word, ep, out):
    """One piece's count-in as a generator: each yield is one atomic step."""
    guess = word.v  # the early read (a plain load; may be stale by the time it is used)
    yield
    old = guess
    while True:
        if (old >> 16) == ep:
            now = word.add(1) + 1
            yield
            break
        prev = word.cas(old, (ep << 16) | 1)
        yield
        if prev == old:
            now = (ep << 16) | 1
            break
        old = prev
    out.append(now)


def run(n, ep, start, rng):
    word = Word(start)
    out = []
    live = [piece(word, ep, out) for _ in range(n)]
    while live:
        g = rng.choice(live)
        try:
            next(g)
        except StopIteration:
            live.remove(g)
    return word.v, out


@pytest.mark.parametrize("n", [1, 2, 3, 27, 74])
def test_counts_are_one_to_n_from_any_previous_state(n):
    rng = random.Random(1000 + n)
    for trial in range(300):
        ep = rng.randrange(1, MASK48)
        kind = trial % 4
        if kind == 0:      # left by the previous launch, fully counted
            start = ((ep - 1) << 16) | rng.randrange(1, 1025)
        elif kind == 1:    # left by an aborted launch long ago
            start = (rng.randrange(0, ep) << 16) | rng.randrange(0, 1 << 16)
        elif kind == 2:    # never written (a zeroed workspace: epoch 0)
            start = 0
        else:              # anything at all (a workspace never zeroed)
            start = rng.getrandbits(64)
            if (start >> 16) == ep:  # a garbage word that carries this launch's tag is out of contract
                start ^= 1 << 40
        final, seen = run(n, ep, start, rng)
        counts = sorted(v & 0xFFFF for v in seen)
        assert counts == list(range(1, n + 1)), (n, kind, hex(start), counts)
        assert all(v >> 16 == ep for v in seen)
        assert final == (ep << 16) | n


def test_a_counter_tagged_with_this_launch_only_adds():
    # pieces that read a current counter never re-tag it (no CAS, no retries)
    rng = random.Random(7)
    ep = 12345
    final, seen = run(50, ep, (ep << 16) | 0, rng)
    assert sorted(v & 0xFFFF for v in seen) == list(range(1, 51))
    assert final == (ep << 16) | 50


def test_the_model_catches_a_lost_count():
    # a mutant that re-tags a stale counter with a plain store instead of a CAS:
    # two pieces that both read the stale value overwrite each other's count,
    # and some interleaving shows it
    def store_piece(word, ep, out):
        old = word.v
        yield
        if (old >> 16) == ep:
            now = word.add(1) + 1
        else:
            word.v = (ep << 16) | 1
            now = (ep << 16) | 1
        yield
        out.append(now)

    rng = random.Random(3)
    caught = False
    for _ in range(200):
        ep = 99
        word = Word((98 << 16) | 5)
        out = []
        live = [store_piece(word, ep, out) for _ in range(8)]
        while live:
            g = rng.choice(live)
            try:
                next(g)
            except StopIteration:
                live.remove(g)
        caught |= sorted(v & 0xFFFF for v in out) != list(range(1, 9))
    assert caught
