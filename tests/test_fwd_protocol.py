"""A model of the synchronisation protocol of the tensor-core attention kernel
(attn_fwd_sm100 in sequence_parallelism_attn_b200/csrc/attn_sm100.cu), run under random
latencies on the CPU with the simulator of tests/_protocol_sim.py.

Tensor memory: one score buffer S shared by the two query tiles, a P region per tile (the
bf16 probabilities), an O accumulator per tile.  Roles, in the kernel's order: the K
producer (which also loads the two Q tiles) with a ring of NSK stages, the V producer with
NSV stages, the MMA thread and the two softmax warpgroups.  The MMA thread issues S_A(0),
then S_B(0) once softmax A has read S_A(0) (sfree[0]); then per key tile j: S_A(j+1) once
softmax B has read S_B(j) (sfree[1]) and K(j+1) has landed; PV_A(j) once P_A(j) is written
(pf[0]) and V(j) has landed, committed to pvd[0]; S_B(j+1) once softmax A has read
S_A(j+1); PV_B(j) once P_B(j) is written, committed to pvd[1] and to V(j)'s empty barrier;
the last PV of each tile commits of[w].  A softmax warpgroup waits sf[w], reads S, signals
sfree[w], and before it writes P(j) over P(j-1) -- and before it rescales O -- waits for
PV(j-1) (pvd[w]); then it signals pf[w]; at the end it waits of[w] and reads O.  Checked: no
deadlock, no mbarrier phase overrun, and every read of S, P, O, a K or V stage and Q sees
the data it must.  Mutated protocols (one wait removed, or a commit moved) must be
flagged."""
import pytest

from _protocol_sim import Sim, Violation


def fwd_roles(sim, n, NSK, NSV, mutation=None):
    for name, count in (("q", 1), ("sf0", 1), ("sf1", 1), ("pf0", 1), ("pf1", 1),
                        ("of0", 1), ("of1", 1), ("drain", 1), ("sfree0", 1), ("sfree1", 1),
                        ("pvd0", 1), ("pvd1", 1)):
        sim.bar(name, count)
    for s in range(NSK):
        sim.bar(f"kf{s}", 1)
        sim.bar(f"ke{s}", 1)
    for s in range(NSV):
        sim.bar(f"vf{s}", 1)
        sim.bar(f"ve{s}", 1)
    P = {0: "PA", 1: "PB"}
    O = {0: "OA", 1: "OB"}

    def producer(is_k):
        ns, full, empty, tag = (NSK, "kf", "ke", "K") if is_k else (NSV, "vf", "ve", "V")
        if is_k:
            sim.bars["q"].arrive(tx=1)
            sim.tma_load("q", "Q", "Q")
        armed = {}
        for jt in range(n):
            slot = jt % ns
            if jt >= ns and not (yield ("wait", f"{empty}{slot}", jt // ns - 1)):
                break
            sim.bars[f"{full}{slot}"].arrive(tx=1)
            sim.tma_load(f"{full}{slot}", f"{tag}{slot}", (tag, jt))
            armed[slot] = jt
            yield None
        if is_k:
            yield ("drain", "q", 0)
        for slot, jt in armed.items():  # drain: every copy this thread started has landed
            yield ("drain", f"{full}{slot}", jt // ns)

    def s_mma(w, j):
        return (("Q", "Q"), (f"K{j % NSK}", ("K", j))), (("S", ("S", w, j)),), \
            f"S_{'AB'[w]}({j})"

    def pv_mma(w, j):
        reads = [(P[w], ("P", j)), (f"V{j % NSV}", ("V", j))]
        if j > 0:
            reads.append((O[w], ("O", j - 1)))
        return reads, [(O[w], ("O", j))], f"PV_{'AB'[w]}({j})"

    def mma():
        issued = False
        if (yield ("wait", "q", 0)) and (yield ("wait", "kf0", 0)):
            sim.mma("M", *s_mma(0, 0))
            sim.commit("M", "sf0")
            issued = True
            if mutation == "no_sfree_wait" or (yield ("wait", "sfree0", 0)):
                sim.mma("M", *s_mma(1, 0))
                sim.commit("M", "sf1")
                sim.commit("M", "ke0")
                for jt in range(n):
                    slot_v, slot_k, more = jt % NSV, (jt + 1) % NSK, jt + 1 < n
                    if more:
                        if not (yield ("wait", "sfree1", jt)):
                            break
                        if not (yield ("wait", f"kf{slot_k}", (jt + 1) // NSK)):
                            break
                        sim.mma("M", *s_mma(0, jt + 1))
                        sim.commit("M", "sf0")
                    if not (yield ("wait", f"vf{slot_v}", jt // NSV)):
                        break
                    if not (yield ("wait", "pf0", jt)):
                        break
                    sim.mma("M", *pv_mma(0, jt))
                    sim.commit("M", "pvd0")
                    if mutation == "ve_commit_early":  # V(j) released before PV_B(j) reads it
                        sim.commit("M", f"ve{slot_v}")
                    if not more:
                        sim.commit("M", "of0")
                    if more:
                        if mutation != "no_sfree_wait" and not (yield ("wait", "sfree0", jt + 1)):
                            break
                        sim.mma("M", *s_mma(1, jt + 1))
                        sim.commit("M", "sf1")
                        sim.commit("M", f"ke{slot_k}")
                    if mutation != "no_pf1_wait" and not (yield ("wait", "pf1", jt)):
                        break
                    sim.mma("M", *pv_mma(1, jt))
                    sim.commit("M", "pvd1")
                    if mutation != "ve_commit_early":
                        sim.commit("M", f"ve{slot_v}")
                    if not more:
                        sim.commit("M", "of1")
        if issued:  # every MMA this thread issued completes before tensor memory is freed
            sim.commit("M", "drain")
            if mutation != "no_mma_drain":
                yield ("drain", "drain", 0)

    def softmax(w, rescale_pattern):
        ok = True
        for jt in range(n):
            if not (yield ("wait", f"sf{w}", jt)):
                ok = False
                break
            sim.read("S", ("S", w, jt), f"softmax{w} S({jt})")
            yield None
            sim.bars[f"sfree{w}"].arrive()
            yield None
            if jt > 0 and mutation != "no_pvd_wait" and not (yield ("wait", f"pvd{w}", jt - 1)):
                ok = False
                break
            sim.write(P[w], ("P", jt))
            if jt > 0 and rescale_pattern[jt]:
                # O holds the sum through tile jt-1; it is scaled in place
                sim.read(O[w], ("O", jt - 1), f"softmax{w} rescale O({jt})")
                yield None
                sim.write(O[w], ("O", jt - 1))
            yield None
            sim.bars[f"pf{w}"].arrive()
        if ok and n > 0 and (yield ("wait", f"of{w}", 0)):
            sim.read(O[w], ("O", n - 1), f"softmax{w} epilogue O")

    roles = {"prodK": producer(True), "prodV": producer(False), "mma": mma()}
    for w in (0, 1):
        pattern = [sim.rng.random() < 0.5 for _ in range(n)]
        roles[f"sm{w}"] = softmax(w, pattern)
    return roles


@pytest.mark.parametrize("NSK,NSV", [(3, 2), (4, 4)])  # D = 128 and D = 64 rings
@pytest.mark.parametrize("n", [1, 2, 3, 5, 9])
def test_forward_protocol_holds_under_random_latencies(NSK, NSV, n):
    for seed in range(300):
        sim = Sim(seed * 7919 + n * 31 + NSK)
        sim.run(fwd_roles(sim, n, NSK, NSV))


@pytest.mark.parametrize("mutation", ["no_pf1_wait", "ve_commit_early", "no_sfree_wait",
                                      "no_pvd_wait"])
def test_forward_mutated_protocols_are_caught(mutation):
    caught = 0
    for seed in range(300):
        sim = Sim(seed)
        try:
            sim.run(fwd_roles(sim, 6, 3, 2, mutation))
        except Violation:
            caught += 1
    assert caught > 0, f"{mutation} was never flagged"


@pytest.mark.parametrize("n", [1, 3, 6])
def test_forward_abort_at_any_point_tears_down_cleanly(n):
    """A bounded wait that gives up at any step: every role stops, drains only its own
    work, and the CTA ends with no MMA or TMA load in flight, without deadlock; without the
    MMA thread's drain it may not."""
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (30 * n))
        sim.run(fwd_roles(sim, n, 3, 2))
    caught = 0
    for seed in range(400):
        sim = Sim(seed, abort_after=1 + seed % (30 * n))
        try:
            sim.run(fwd_roles(sim, n, 3, 2, "no_mma_drain"))
        except Violation:
            caught += 1
    assert caught > 0
