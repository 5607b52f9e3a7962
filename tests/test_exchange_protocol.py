"""A model of the one-kernel Ulysses exchange across ranks (dist.ulysses_seq2head_p2p /
ulysses_head2seq_p2p with dist.PeerBuffers), run under random interleavings on the CPU.

Every rank r of P repeats, step after step, in stream order: the first barrier (no rank is
still reading its buffer), its scatter kernel (one store into every rank's buffer: share r
of that step), the second barrier (every share has landed), then the consumer of its own
buffer (the attention kernel), which reads all P shares.  A barrier lets a rank through once
every rank has reached it.  The stores of one scatter land in any order and at any time
before the rank's next barrier, and the reads of one consumer in any order.

Checked: every read sees the share of its own step (no stale share from the step before,
no share of the next step written under it), and no schedule deadlocks.  The protocol with
either barrier removed must be flagged, which shows the checks can fail."""
import random

import pytest


class Violation(AssertionError):
    pass


def run(P, steps, seed, drop=None):
    rng = random.Random(seed)
    buf = [[None] * P for _ in range(P)]  # buf[d][s]: the share of rank s in rank d's buffer
    arrived = {}                           # barrier name -> ranks that reached it

    def rank(r):
        for k in range(steps):
            if drop != "first":
                yield ("barrier", ("free", k))
            for d in rng.sample(range(P), P):  # the kernel's stores, in any order
                buf[d][r] = (k, r)
                yield None
            if drop != "second":
                yield ("barrier", ("landed", k))
            for s in rng.sample(range(P), P):  # the consumer's reads, in any order
                got = buf[r][s]
                if got != (k, s):
                    raise Violation(f"rank {r} step {k} read {got} for share {s}")
                yield None

    gens = {r: rank(r) for r in range(P)}
    waiting = {}  # rank -> barrier name it waits at
    while gens:
        ready = [r for r in gens if r not in waiting or
                 len(arrived.get(waiting[r], ())) == P]
        if not ready:
            raise Violation("deadlock")
        r = rng.choice(ready)
        waiting.pop(r, None)
        try:
            ev = next(gens[r])
        except StopIteration:
            del gens[r]
            continue
        if ev is not None and ev[0] == "barrier":
            arrived.setdefault(ev[1], set()).add(r)
            waiting[r] = ev[1]


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
def test_exchange_protocol_holds_under_random_interleavings(P):
    for seed in range(300):
        run(P, 4, seed * 31 + P)


@pytest.mark.parametrize("drop", ["first", "second"])
def test_exchange_without_a_barrier_is_caught(drop):
    caught = 0
    for seed in range(300):
        try:
            run(4, 4, seed, drop)
        except Violation:
            caught += 1
    assert caught > 0, f"dropping the {drop} barrier was never flagged"
