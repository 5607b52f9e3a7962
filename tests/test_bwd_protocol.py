"""A model of the synchronisation protocol of the two tensor-core backward kernels
(bwd_dq_sm100 and bwd_dkdv_sm100 in sequence_parallelism_attn_b200/csrc/attn_bwd_sm100.cu),
run under random latencies on the CPU.

Each role of a CTA -- the loader, the two MMA-issuing threads, the two compute warpgroups --
is a generator that performs, in the kernel's order, its mbarrier waits and arrivals, its
MMA issues and commits, its TMA loads and its tensor-memory loads and stores.  The model
executes:
  * mbarriers with the hardware's parity rule (a wait for phase k succeeds while the phase
    count differs from k in its low bit), arrival counts and TMA transaction counts;
  * MMAs per issuing thread in issue order (tcgen05 operations of one thread complete in
    order), interleaved at random across threads, and a commit arriving once everything
    its thread issued before it has completed;
  * TMA loads completing at random times.
Every read of a tensor-memory region half or a shared-memory stage names the data it must
see (which tile's S, dP, P/dS, or which tile's Q/dO, K/V); the model flags a read that sees
anything else, a barrier that completes a phase twice before one of its waiters has seen
the first (the parity hazard), and a schedule in which no role can proceed.  Mutated
protocols (one wait removed) must be flagged, which shows the checks can fail."""
import pytest

from _protocol_sim import Sim, Violation


# ------------------------------------------------------------------ the dK/dV kernel
# Per query tile i: S^T(i) (thread B) into one region and dP^T(i) (thread A) into the other.
# A compute warpgroup waits S^T(i) alone, forms P^T of its 64-query half and stores it over
# the S^T columns it read (pready), then waits dP^T(i), reads it (dpfree), forms dS^T and
# stores it beside P^T (dsready).  A issues dV per half after pready, then -- once B's dK(i)
# is done (xfree) -- dP^T(i+1) over the region of P^T / dS^T(i); B issues S^T(i+1) into the
# dP^T(i) region once every compute warp has read it, and dK per half after dsready.  So
# the exponentials of tile i+1 overlap the chain dK(i) -> dP^T(i+1).  pready alternates
# between two barriers per half (tile parity): A's wait for tile i may otherwise come after
# the warpgroup's arrival for tile i+1.
def dkdv_roles(sim, n, mutation=None):
    NS = 2
    st_col = lambda i: "R1" if i & 1 else "R0"   # S^T region of query tile i
    dpt_col = lambda i: "R0" if i & 1 else "R1"  # dP^T region of query tile i
    for name, count in (("fixed", 1), ("sready", 1), ("dpready", 1), ("ds0", 1), ("ds1", 1),
                        ("p00", 1), ("p01", 1), ("p10", 1), ("p11", 1), ("acc", 2),
                        ("drain", 2), ("xfree", 1), ("dpfree", 2)):
        sim.bar(name, count)
    for s in range(NS):
        sim.bar(f"full{s}", 2)
        sim.bar(f"empty{s}", 1)
    pready = lambda c, i: f"p{c}{i & 1}"

    def loader():
        sim.bars["fixed"].arrive(tx=1)
        sim.tma_load("fixed", "KV", "KV")
        yield None
        armed = {}
        for it in range(n):
            slot = it % NS
            if it >= NS and not (yield ("wait", f"empty{slot}", it // NS - 1)):
                break
            sim.bars[f"full{slot}"].arrive(tx=1)       # expect_tx, then Q and dO
            sim.tma_load(f"full{slot}", f"stage{slot}", ("QdO", it))
            sim.write(f"rows{slot}", ("rows", it))      # LSE, Delta, positions: plain stores
            yield None
            sim.bars[f"full{slot}"].arrive()
            armed[slot] = it
        if mutation != "no_load_drain":
            yield ("drain", "fixed", 0)                 # every copy it started has landed
            for slot, it in armed.items():
                yield ("drain", f"full{slot}", it // NS)

    def stage_reads(i):
        return [(f"stage{i % NS}", ("QdO", i))]

    def half_regions(region):
        return [region + "h0P", region + "h0D", region + "h1P", region + "h1D"]

    def mma_a():  # dP^T and dV
        if (yield ("wait", "fixed", 0)) and (yield ("wait", "full0", 0)):
            sim.mma("A", [("KV", "KV")] + stage_reads(0),
                    [(r, ("dP", 0)) for r in half_regions(dpt_col(0))], "dP^T(0)")
            sim.commit("A", "dpready")
            for it in range(n):
                more = it + 1 < n
                if mutation != "no_pready_wait" and not (yield ("wait", pready(0, it), it // 2)):
                    break
                sim.mma("A", [(st_col(it) + "h0P", ("P", it))] + stage_reads(it), [],
                        f"dV h0({it})")
                if not (yield ("wait", pready(1, it), it // 2)):
                    break
                sim.mma("A", [(st_col(it) + "h1P", ("P", it))] + stage_reads(it), [],
                        f"dV h1({it})")
                if more and mutation != "no_xfree_wait" and not (yield ("wait", "xfree", it)):
                    break
                sim.commit("A", f"empty{it % NS}")
                if more:
                    sim.mma("A", [("KV", "KV")] + stage_reads(it + 1),
                            [(r, ("dP", it + 1)) for r in half_regions(dpt_col(it + 1))],
                            f"dP^T({it + 1})")
                    sim.commit("A", "dpready")
        sim.commit("A", "acc")  # unconditional (n > 0): a commit with nothing pending arrives
        sim.commit("A", "drain")
        if mutation != "no_mma_drain":
            yield ("drain", "drain", 0)

    def mma_b():  # S^T and dK
        if (yield ("wait", "fixed", 0)) and (yield ("wait", "full0", 0)):
            sim.mma("B", [("KV", "KV")] + stage_reads(0),
                    [(r, ("S", 0)) for r in half_regions(st_col(0))], "S^T(0)")
            sim.commit("B", "sready")
            for it in range(n):
                if it + 1 < n:
                    if mutation != "no_dpfree_wait" and not (yield ("wait", "dpfree", it)):
                        break
                    if not (yield ("wait", f"full{(it + 1) % NS}", (it + 1) // NS)):
                        break
                    sim.mma("B", [("KV", "KV")] + stage_reads(it + 1),
                            [(r, ("S", it + 1)) for r in half_regions(st_col(it + 1))],
                            f"S^T({it + 1})")
                    sim.commit("B", "sready")
                if not (yield ("wait", "ds0", it)):
                    break
                sim.mma("B", [(st_col(it) + "h0D", ("dS", it))] + stage_reads(it), [],
                        f"dK h0({it})")
                if not (yield ("wait", "ds1", it)):
                    break
                sim.mma("B", [(st_col(it) + "h1D", ("dS", it))] + stage_reads(it), [],
                        f"dK h1({it})")
                sim.commit("B", "xfree")
        sim.commit("B", "acc")
        sim.commit("B", "drain")
        if mutation != "no_mma_drain":
            yield ("drain", "drain", 0)

    def compute(c):
        ok = True
        for it in range(n):
            if not (yield ("wait", "sready", it)):
                ok = False
                break
            sim.read(f"{st_col(it)}h{c}P", ("S", it), f"WG{c} S({it})")
            sim.read(f"{st_col(it)}h{c}D", ("S", it), f"WG{c} S({it})")
            sim.read(f"rows{it % NS}", ("rows", it), f"WG{c} rows({it})")
            yield None
            if mutation == "store_before_read" and c == 1:
                sim.write(f"{st_col(it)}h0P", ("P", it))  # a half it does not own
            sim.write(f"{st_col(it)}h{c}P", ("P", it))
            yield None
            sim.bars[pready(c, it)].arrive()
            if mutation != "no_dpready_wait" and not (yield ("wait", "dpready", it)):
                ok = False
                break
            sim.read(f"{dpt_col(it)}h{c}P", ("dP", it), f"WG{c} dP({it})")
            sim.read(f"{dpt_col(it)}h{c}D", ("dP", it), f"WG{c} dP({it})")
            yield None
            sim.bars["dpfree"].arrive()
            yield None
            sim.write(f"{st_col(it)}h{c}D", ("dS", it))
            yield None
            sim.bars[f"ds{c}"].arrive()
        if ok and n > 0:
            yield ("wait", "acc", 0)

    return {"load": loader(), "A": mma_a(), "B": mma_b(), "WG0": compute(0), "WG1": compute(1)}


# ------------------------------------------------------------------ the dQ kernel
# Per key tile j: S(j) (thread A) into one of two S regions, dP(j) (thread B).  The compute
# warps wait S(j) (sready) and dP(j) (dpready), read both (dpfree), and store dS over their
# half of S(j) (ds0 / ds1).  A issues S(j+1) as soon as K(j+1) has landed and commits
# sready once every compute warp has read tile j (dpfree), so that the commit waits for
# S(j+1) alone and never for dQ(j); then dQ per half after ds0 / ds1.  B issues dP(j+1) once
# dP(j) has been read.  The compute warps may then finish tile j+1 before A has waited for
# tile j's dS, so ds0 / ds1 alternate between two barriers each by tile parity.
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


KERNELS = {"dkdv": dkdv_roles, "dq": dq_roles}


@pytest.mark.parametrize("kernel", ["dkdv", "dq"])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 7])
def test_protocol_holds_under_random_latencies(kernel, n):
    for seed in range(300):
        sim = Sim(seed * 1000 + n)
        sim.run(KERNELS[kernel](sim, n))


@pytest.mark.parametrize("kernel,mutation", [("dkdv", "no_xfree_wait"),
                                             ("dkdv", "no_dpfree_wait"),
                                             ("dkdv", "store_before_read"),
                                             ("dkdv", "no_pready_wait"),
                                             ("dkdv", "no_dpready_wait"),
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


@pytest.mark.parametrize("kernel", ["dkdv", "dq"])
@pytest.mark.parametrize("n", [1, 3, 6])
def test_abort_at_any_point_tears_down_cleanly(kernel, n):
    """A bounded wait that gives up at any step: every role stops, drains only its own
    work, and the CTA ends with no MMA or TMA load in flight (tensor memory and shared
    memory may then be released), without deadlock."""
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (40 * n))
        sim.run(KERNELS[kernel](sim, n))


@pytest.mark.parametrize("mutation", ["no_mma_drain", "no_load_drain"])
def test_teardown_without_a_drain_is_caught(mutation):
    """Both MMA threads skipping their drain wait (either one alone is covered by the
    other's, since the drain barrier counts both commits), or the loader skipping its own."""
    caught = 0
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % 200)
        try:
            sim.run(dkdv_roles(sim, 5, mutation))
        except Violation:
            caught += 1
    assert caught > 0, f"{mutation} was never flagged"
