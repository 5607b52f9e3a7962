"""A model of the shared-memory ring of the Ulysses transforms' TMA kernel
(permute_tma_kernel in sequence_parallelism_attn_b200/csrc/permute.cu), run under random
latencies on the CPU with the simulator of tests/_protocol_sim.py.

One thread per CTA: NS stages, loads of blocks 0 .. NS-2 issued up front; then per block n:
wait for its load (the stage's mbarrier, phase n / NS), issue its stores (one per GQA
replica) as one bulk group, and -- while loads remain -- wait until every bulk group but the
most recent has read its source (cp.async.bulk.wait_group.read 1) before refilling the stage
that held block n - 1 with block n + NS - 1.  Checked: every store reads the block it must,
no stage is refilled under a pending store, no mbarrier phase is overrun, no deadlock.  A
ring that refills without the read wait, or that waits for the wrong group count, must be
flagged."""
import pytest

from _protocol_sim import Sim, Violation


def permute_role(sim, n_blocks, NS, rep, mutation=None):
    for i in range(NS):
        sim.bar(f"b{i}", 1)

    def issue_load(i):
        sim.bars[f"b{i % NS}"].arrive(tx=1)
        sim.tma_load(f"b{i % NS}", f"stage{i % NS}", ("blk", i))

    def thread():
        issued = 0
        while issued < NS - 1 and issued < n_blocks:
            issue_load(issued)
            issued += 1
        n = 0
        while n < n_blocks:
            if not (yield ("wait", f"b{n % NS}", n // NS)):
                break  # the bounded wait gave up
            sim.bulk_group([(f"stage{n % NS}", ("blk", n))] * rep, f"stores of block {n}")
            if issued < n_blocks:
                if mutation == "no_read_wait":
                    pass
                else:
                    k = 2 if mutation == "wait_read_2" else 1
                    yield ("until", lambda k=k: sim.bulk_read_done_but(k))
                issue_load(issued)
                issued += 1
            n += 1
            yield None
        yield ("until", lambda: sim.bulk_read_done_but(0))  # bulk_wait_all
        if mutation != "no_load_drain":
            for i in range(n, issued):  # loads issued but never consumed land before exit
                yield ("drain", f"b{i % NS}", i // NS)

    return {"thread": thread()}


@pytest.mark.parametrize("NS", [2, 3])
@pytest.mark.parametrize("n_blocks,rep", [(1, 1), (2, 2), (3, 1), (7, 1), (9, 8)])
def test_permute_ring_holds_under_random_latencies(NS, n_blocks, rep):
    for seed in range(300):
        sim = Sim(seed * 97 + n_blocks)
        sim.run(permute_role(sim, n_blocks, NS, rep))


@pytest.mark.parametrize("mutation", ["no_read_wait", "wait_read_2"])
def test_permute_ring_mutations_are_caught(mutation):
    caught = 0
    for seed in range(300):
        sim = Sim(seed)
        try:
            sim.run(permute_role(sim, 8, 3, 2, mutation))
        except Violation:
            caught += 1
    assert caught > 0, f"{mutation} was never flagged"


@pytest.mark.parametrize("n_blocks", [2, 5, 9])
def test_permute_ring_abort_tears_down_cleanly(n_blocks):
    """A wait that gives up at any step: the thread waits for its stores and the loads it
    issued, so the CTA ends with nothing in flight; without the load drain it may not."""
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (12 * n_blocks))
        sim.run(permute_role(sim, n_blocks, 3, 2))
    caught = 0
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (12 * n_blocks))
        try:
            sim.run(permute_role(sim, n_blocks, 3, 2, "no_load_drain"))
        except Violation:
            caught += 1
    assert caught > 0
