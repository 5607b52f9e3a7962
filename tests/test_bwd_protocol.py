"""A model of the synchronisation protocol of the tensor-core backward kernels (bwd_sm100,
and bwd_dq_sm100 of the deterministic mode, in
sequence_parallelism_attn_b200/csrc/attn_bwd_sm100.cu), run under random latencies on the
CPU.

Each role of a CTA -- the loader, the three MMA-issuing threads, the two compute
warpgroups, the four dQ reduce warps -- is a generator that performs, in the kernel's
order, its mbarrier waits and arrivals, its MMA issues and commits, its TMA loads, its
tensor-memory and shared-memory loads and stores, and its bulk reduce groups.  The model
executes:
  * mbarriers with the hardware's parity rule (a wait for phase k succeeds while the phase
    count differs from k in its low bit), arrival counts and TMA transaction counts;
  * MMAs per issuing thread in issue order (tcgen05 operations of one thread complete in
    order), interleaved at random across threads, and a commit arriving once everything
    its thread issued before it has completed;
  * TMA loads completing at random times, and bulk reduce groups reading their staging
    buffers at random times (cp.async.bulk.wait_group.read counts a thread's own groups).
Every read of a tensor-memory region half, a shared-memory stage or dS^T block, or a
staging buffer names the data it must see (which item's S^T, P^T, dP^T, dQ, Q, dO, dS^T);
the model flags a read that sees anything else, a barrier that completes a phase twice
before one of its waiters has seen the first (the parity hazard), and a schedule in which
no role can proceed.  Mutated protocols (one wait removed) must be flagged, which shows the
checks can fail."""
import pytest

from _protocol_sim import Sim, Violation


# One CTA per key tile computes dK, dV and its contributions to dQ.  Tensor memory: S^T
# (R_S, one region, P^T of each 64-query half written over it), dP^T (R_dP, one N = 64 MMA
# per query half), dQ of the tile over R_dP once both halves of dP^T have been read, and the
# dV / dK accumulators.  Per query tile i:
#   A: dV per half once its P^T is published (p0 / p1), commit dvdone and the stage's
#      empty (the stage is refilled once A and B have both released it); once dV(i) has
#      completed (its own dvdone) and tile i+1 has landed, S^T(i+1) into R_S, sready.
#   C: dP^T(i+1) per half once the reduce warps have read that half of dQ(i) (rfree0 /
#      rfree1), dpready0 / dpready1.
#   B: dK over each half once its dS^T is in shared memory (ds0 / ds1); after the second,
#      dQ(i) = dS K into R_dP, dqready, then the second dK half and the stage's empty.
#   compute warpgroup c: S^T(i) -> P^T over it (p_c); dP^T half c -> dS^T, stored to
#      shared memory (over dO(i) when the head dimension is 128, so only after dV(i) and
#      both dP^T halves have read dO(i): dvdone, dpready of the other half), ds_c.
#   reduce warps (one per TMEM lane quarter): dqready; per 64-column half of dQ(i): load
#      it, rfree of that half, then 16-column chunks through three staging buffers per warp
#      into bulk reduce-adds (wait_group.read 2 before a buffer is reused).
# In the deterministic mode (skip_dq) B issues no dQ MMA but still commits dqready, and the
# reduce warps only arrive on rfree0 / rfree1 after it: the same barriers in the same order.
def fused_roles(sim, n, ds_in_do=True, mutation=None, skip_dq=False):
    NS, NRED = 2, 4
    for name, count in (("fixed", 1), ("sready", 1), ("dpready0", 1), ("dpready1", 1),
                        ("dvdone", 1), ("p0", 1), ("p1", 1), ("ds0", 1), ("ds1", 1),
                        ("dqready", 1), ("rfree0", NRED), ("rfree1", NRED), ("acc", 2),
                        ("drain", 3)):
        sim.bar(name, count)
    for s in range(NS):
        sim.bar(f"full{s}", 2)
        sim.bar(f"empty{s}", 2)  # A after dV, B after dK: both read the stage
    do_blocks = lambda s: [f"dO{s}b0", f"dO{s}b1"]
    ds_block = lambda s, c: f"dO{s}b{c}" if ds_in_do else f"dS{s}b{c}"

    def loader():
        sim.bars["fixed"].arrive(tx=1)
        sim.tma_load("fixed", "KV", "KV")
        yield None
        armed = {}
        for it in range(n):
            slot = it % NS
            if it >= NS and not (yield ("wait", f"empty{slot}", it // NS - 1)):
                break
            sim.bars[f"full{slot}"].arrive(tx=3)       # expect_tx, then Q and dO
            sim.tma_load(f"full{slot}", f"Q{slot}", ("Q", it))
            for blk in do_blocks(slot):
                sim.tma_load(f"full{slot}", blk, ("dO", it))
            sim.write(f"rows{slot}", ("rows", it))      # LSE, Delta, positions: plain stores
            yield None
            sim.bars[f"full{slot}"].arrive()
            armed[slot] = it
        if mutation != "no_load_drain":
            yield ("drain", "fixed", 0)                 # every copy it started has landed
            for slot, it in armed.items():
                yield ("drain", f"full{slot}", it // NS)

    q = lambda i: (f"Q{i % NS}", ("Q", i))
    do = lambda i: [(blk, ("dO", i)) for blk in do_blocks(i % NS)]

    def mma_a():  # S^T and dV
        if (yield ("wait", "fixed", 0)) and n > 0 and (yield ("wait", "full0", 0)):
            sim.mma("A", [("KV", "KV"), q(0)], [("RSh0", ("S", 0)), ("RSh1", ("S", 0))], "S^T(0)")
            sim.commit("A", "sready")
            for it in range(n):
                ok = True
                for c in (0, 1):
                    if not (yield ("wait", f"p{c}", it)):
                        ok = False
                        break
                    sim.mma("A", [(f"RSh{c}", ("P", it))] + do(it), [], f"dV h{c}({it})")
                if not ok:
                    break
                sim.commit("A", "dvdone")
                if mutation != "no_a_release":
                    sim.commit("A", f"empty{it % NS}")
                if it + 1 < n:
                    # the kernel waits for its own dV(i) before S^T(i+1) overwrites the P^T
                    # that dV(i) reads; with one thread's MMAs executed in order (as modelled)
                    # the wait is a margin, not a requirement
                    if not (yield ("wait", "dvdone", it)):
                        break
                    if not (yield ("wait", f"full{(it + 1) % NS}", (it + 1) // NS)):
                        break
                    sim.mma("A", [("KV", "KV"), q(it + 1)],
                            [("RSh0", ("S", it + 1)), ("RSh1", ("S", it + 1))], f"S^T({it + 1})")
                    sim.commit("A", "sready")
        if n > 0:
            sim.commit("A", "acc")
            sim.commit("A", "drain")
            if mutation != "no_mma_drain":
                yield ("drain", "drain", 0)

    def mma_c():  # dP^T, one half at a time
        if (yield ("wait", "fixed", 0)) and n > 0 and (yield ("wait", "full0", 0)):
            for h in (0, 1):
                sim.mma("C", [("KV", "KV")] + do(0), [(f"RdPh{h}", ("dP", 0))], f"dP^T h{h}(0)")
                sim.commit("C", f"dpready{h}")
            for it in range(n - 1):
                if not (yield ("wait", f"full{(it + 1) % NS}", (it + 1) // NS)):
                    break
                ok = True
                for h in (0, 1):
                    if mutation != "no_rfree_wait" and not (yield ("wait", f"rfree{h}", it)):
                        ok = False
                        break
                    sim.mma("C", [("KV", "KV")] + do(it + 1), [(f"RdPh{h}", ("dP", it + 1))],
                            f"dP^T h{h}({it + 1})")
                    sim.commit("C", f"dpready{h}")
                if not ok:
                    break
        if n > 0:
            sim.commit("C", "drain")
            if mutation != "no_mma_drain":
                yield ("drain", "drain", 0)

    def mma_b():  # dK and dQ
        if (yield ("wait", "fixed", 0)) and n > 0:
            for it in range(n):
                s = it % NS
                if not (yield ("wait", "ds0", it)):
                    break
                sim.mma("B", [(ds_block(s, 0), ("dS", it)), q(it)], [], f"dK h0({it})")
                if mutation != "no_ds1_wait" and not (yield ("wait", "ds1", it)):
                    break
                if not skip_dq:
                    sim.mma("B", [(ds_block(s, 0), ("dS", it)), (ds_block(s, 1), ("dS", it)),
                                  ("KV", "KV")], [("RdPh0", ("dQ", it)), ("RdPh1", ("dQ", it))],
                            f"dQ({it})")
                sim.commit("B", "dqready")
                sim.mma("B", [(ds_block(s, 1), ("dS", it)), q(it)], [], f"dK h1({it})")
                sim.commit("B", f"empty{s}")
        if n > 0:
            sim.commit("B", "acc")
            sim.commit("B", "drain")
            if mutation != "no_mma_drain":
                yield ("drain", "drain", 0)

    def compute(c):
        ok = True
        for it in range(n):
            s = it % NS
            if not (yield ("wait", "sready", it)):
                ok = False
                break
            sim.read(f"RSh{c}", ("S", it), f"WG{c} S^T({it})")
            sim.read(f"rows{s}", ("rows", it), f"WG{c} rows({it})")
            yield None
            sim.write(f"RSh{c}", ("P", it))
            yield None
            sim.bars[f"p{c}"].arrive()
            if not (yield ("wait", f"dpready{c}", it)):
                ok = False
                break
            sim.read(f"RdPh{c}", ("dP", it), f"WG{c} dP^T({it})")
            yield None
            if ds_in_do and mutation != "no_do_wait":
                if not (yield ("wait", "dvdone", it)):
                    ok = False
                    break
                if not (yield ("wait", f"dpready{1 - c}", it)):
                    ok = False
                    break
            sim.write(ds_block(s, c), ("dS", it))
            yield None
            sim.bars[f"ds{c}"].arrive()
        if ok and n > 0:
            yield ("wait", "acc", 0)

    def reduce(w):
        k = 0
        for it in range(n):
            if not (yield ("wait", "dqready", it)):
                break
            for h in (0, 1):
                if skip_dq:
                    sim.bars[f"rfree{h}"].arrive()
                    continue
                sim.read(f"RdPh{h}", ("dQ", it), f"RED{w} dQ h{h}({it})")
                yield None
                sim.bars[f"rfree{h}"].arrive()
                for ch in range(4):
                    buf = f"stg{w}{k % 3}"
                    if mutation != "no_stage_wait":
                        yield ("until", lambda: sim.bulk_read_done_but(2, w))
                    sim.write(buf, ("dQc", it, h, ch))
                    yield None
                    sim.bulk_group([(buf, ("dQc", it, h, ch))], f"RED{w} reduce", owner=w)
                    k += 1
        if mutation != "no_reduce_drain":
            yield ("until", lambda: sim.bulk_read_done_but(0, w))  # bulk_wait_all

    roles = {"load": loader(), "A": mma_a(), "B": mma_b(), "C": mma_c(),
             "WG0": compute(0), "WG1": compute(1)}
    for w in range(NRED):
        roles[f"RED{w}"] = reduce(w)
    return roles


# The deterministic mode's dQ kernel (bwd_dq_sm100, one CTA per query tile).  Per key tile
# j: S(j) (thread A) into one of two S regions, dP(j) (thread B).  The compute warps wait
# S(j) (sready) and dP(j) (dpready), read both (dpfree), and store dS over their half of
# S(j) (ds0 / ds1).  A issues S(j+1) as soon as K(j+1) has landed and commits sready once
# every compute warp has read tile j (dpfree), so that the commit waits for S(j+1) alone and
# never for dQ(j); then dQ per half after ds0 / ds1.  B issues dP(j+1) once dP(j) has been
# read.  The compute warps may then finish tile j+1 before A has waited for tile j's dS, so
# ds0 / ds1 alternate between two barriers each by tile parity.
def dq_roles(sim, n, mutation=None):
    NS = 2
    s_col = lambda j: "S1" if j & 1 else "S0"
    for name, count in (("fixed", 1), ("sready", 1), ("dpready", 1), ("ds00", 1), ("ds01", 1),
                        ("ds10", 1), ("ds11", 1), ("acc", 1), ("drain", 2), ("dpfree", 2)):
        sim.bar(name, count)
    for s in range(NS):
        sim.bar(f"full{s}", 1)
        sim.bar(f"empty{s}", 1)

    def loader():
        sim.bars["fixed"].arrive(tx=1)
        sim.tma_load("fixed", "QdO", "QdO")
        yield None
        armed = {}
        for jt in range(n):
            slot = jt % NS
            if jt >= NS and not (yield ("wait", f"empty{slot}", jt // NS - 1)):
                break
            sim.bars[f"full{slot}"].arrive(tx=1)
            sim.tma_load(f"full{slot}", f"stage{slot}", ("KV", jt))
            armed[slot] = jt
            yield None
        yield ("drain", "fixed", 0)
        for slot, jt in armed.items():
            yield ("drain", f"full{slot}", jt // NS)

    kv = lambda j: [(f"stage{j % NS}", ("KV", j)), ("QdO", "QdO")]
    ds = lambda c, j: f"ds{c}{j & 1}"

    def mma_a():  # S and dQ
        if (yield ("wait", "fixed", 0)) and (yield ("wait", "full0", 0)):
            sim.mma("A", kv(0), [(s_col(0) + "h0", ("S", 0)), (s_col(0) + "h1", ("S", 0))],
                    "S(0)")
            sim.commit("A", "sready")
            for jt in range(n):
                more = jt + 1 < n
                if more:
                    if not (yield ("wait", f"full{(jt + 1) % NS}", (jt + 1) // NS)):
                        break
                    sim.mma("A", kv(jt + 1), [(s_col(jt + 1) + "h0", ("S", jt + 1)),
                                              (s_col(jt + 1) + "h1", ("S", jt + 1))],
                            f"S({jt + 1})")
                    if mutation != "no_sready_gate" and not (yield ("wait", "dpfree", jt)):
                        break
                    sim.commit("A", "sready")
                if not (yield ("wait", ds(0, jt), jt // 2)):
                    break
                sim.mma("A", [(s_col(jt) + "h0", ("dS", jt))] + kv(jt), [], f"dQ h0({jt})")
                if mutation != "no_ds1_wait" and not (yield ("wait", ds(1, jt), jt // 2)):
                    break
                sim.mma("A", [(s_col(jt) + "h1", ("dS", jt))] + kv(jt), [], f"dQ h1({jt})")
                sim.commit("A", f"empty{jt % NS}")
        sim.commit("A", "acc")
        sim.commit("A", "drain")
        if mutation != "no_mma_drain":
            yield ("drain", "drain", 0)

    def mma_b():  # dP
        if (yield ("wait", "fixed", 0)) and (yield ("wait", "full0", 0)):
            sim.mma("B", kv(0), [("dPh0", ("dP", 0)), ("dPh1", ("dP", 0))], "dP(0)")
            sim.commit("B", "dpready")
            for jt in range(n - 1):
                if mutation != "no_dpfree_wait" and not (yield ("wait", "dpfree", jt)):
                    break
                if not (yield ("wait", f"full{(jt + 1) % NS}", (jt + 1) // NS)):
                    break
                sim.mma("B", kv(jt + 1), [("dPh0", ("dP", jt + 1)), ("dPh1", ("dP", jt + 1))],
                        f"dP({jt + 1})")
                sim.commit("B", "dpready")
        sim.commit("B", "drain")
        if mutation != "no_mma_drain":
            yield ("drain", "drain", 0)

    def compute(c):
        ok = True
        for jt in range(n):
            if not (yield ("wait", "sready", jt)):
                ok = False
                break
            if not (yield ("wait", "dpready", jt)):
                ok = False
                break
            sim.read(f"{s_col(jt)}h{c}", ("S", jt), f"WG{c} S({jt})")
            sim.read(f"dPh{c}", ("dP", jt), f"WG{c} dP({jt})")
            yield None
            sim.bars["dpfree"].arrive()
            yield None
            sim.write(f"{s_col(jt)}h{c}", ("dS", jt))
            yield None
            sim.bars[ds(c, jt)].arrive()
        if ok and n > 0:
            yield ("wait", "acc", 0)

    return {"load": loader(), "A": mma_a(), "B": mma_b(), "WG0": compute(0), "WG1": compute(1)}


KERNELS = {"d128": lambda sim, n, mutation=None: fused_roles(sim, n, True, mutation),
           "d64": lambda sim, n, mutation=None: fused_roles(sim, n, False, mutation),
           "d128_skip_dq": lambda sim, n, mutation=None: fused_roles(sim, n, True, mutation,
                                                                     skip_dq=True),
           "d64_skip_dq": lambda sim, n, mutation=None: fused_roles(sim, n, False, mutation,
                                                                    skip_dq=True),
           "dq": dq_roles}
ALL = ["d128", "d64", "d128_skip_dq", "d64_skip_dq", "dq"]


@pytest.mark.parametrize("kernel", ALL)
@pytest.mark.parametrize("n", [1, 2, 3, 4, 7])
def test_protocol_holds_under_random_latencies(kernel, n):
    for seed in range(300):
        sim = Sim(seed * 1000 + n)
        sim.run(KERNELS[kernel](sim, n))


@pytest.mark.parametrize("kernel,mutation", [("d128", "no_rfree_wait"),
                                             ("d128", "no_do_wait"),
                                             ("d128", "no_ds1_wait"),
                                             ("d128", "no_stage_wait"),
                                             ("d64", "no_a_release"),
                                             ("d64", "no_rfree_wait"),
                                             ("d128_skip_dq", "no_do_wait"),
                                             ("d128_skip_dq", "no_ds1_wait"),
                                             ("d64_skip_dq", "no_a_release"),
                                             ("dq", "no_dpfree_wait"),
                                             ("dq", "no_ds1_wait"),
                                             ("dq", "no_sready_gate")])
def test_mutated_protocols_are_caught(kernel, mutation):
    caught = 0
    for seed in range(300):
        sim = Sim(seed)
        try:
            sim.run(KERNELS[kernel](sim, 4, mutation))
        except Violation:
            caught += 1
    assert caught > 0, f"{kernel} with {mutation} was never flagged"


@pytest.mark.parametrize("kernel", ALL)
@pytest.mark.parametrize("n", [1, 3, 6])
def test_abort_at_any_point_tears_down_cleanly(kernel, n):
    """A bounded wait that gives up at any step: every role stops, drains only its own
    work, and the CTA ends with no MMA, TMA load or bulk reduce in flight (tensor memory and
    shared memory may then be released), without deadlock."""
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (60 * n))
        sim.run(KERNELS[kernel](sim, n))


@pytest.mark.parametrize("mutation", ["no_mma_drain", "no_load_drain", "no_reduce_drain"])
def test_teardown_without_a_drain_is_caught(mutation):
    """The MMA threads skipping their drain wait (any one alone is covered by the others',
    since the drain barrier counts all three commits), the loader skipping its own, or the
    reduce warps ending with bulk reduces still reading their staging buffers."""
    caught = 0
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % 300)
        try:
            sim.run(fused_roles(sim, 5, True, mutation))
        except Violation:
            caught += 1
    assert caught > 0, f"{mutation} was never flagged"


def test_dq_kernel_teardown_without_a_drain_is_caught():
    """The deterministic mode's dQ kernel: both MMA threads skipping their drain wait."""
    caught = 0
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % 200)
        try:
            sim.run(dq_roles(sim, 5, "no_mma_drain"))
        except Violation:
            caught += 1
    assert caught > 0
