"""The multi-GPU data plane's exchange logic on CPU ranks (gloo, world sizes 2 and 4): the
ring schedule and its double-buffered K/V exchange, ring attention across ranks equal to
attention over the whole sequence, the ring backward (dK, dV accumulators travelling with
their chunks) equal to the whole sequence's gradients, the Ulysses pack -> all-to-all -> unpack equal to the
oracle's seq->head / head->seq bit for bit, and a rank that leaves between steps reported
as an error rather than a hang.

The computations are the oracle's here (no GPU on these ranks); on the GPU the same
functions call the library's kernels (DeviceOps), whose pack / unpack and per-step
attention + merge are checked against the oracle in tests/test_dist_gpu.py.

Sources: "Как работает sequence parallelism в контексте LLM?" section 3 (rank i holds
chunk (i - s) mod P at step s; P - 1 exchanges) and section 5 (merge of the partials);
"Метод контекстного параллелизма Ulysses" (the all-to-all before and after attention)."""
import os
import queue
import socket
import time
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, fn, args, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=20))
        res = fn(rank, world, *args)
        q.put((rank, "ok", res))
        dist.destroy_process_group()
    except BaseException as e:  # reported to the parent, which fails the test
        q.put((rank, "error", f"{type(e).__name__}: {e}\n{traceback.format_exc()}"))


def run_ranks(world, fn, *args, timeout=120):
    """Run fn(rank, world, *args) on `world` gloo ranks (spawned processes); returns
    {rank: (status, result)}."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fn, args, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    deadline = time.monotonic() + timeout
    try:
        # a rank that exits without reporting (a rank that leaves) sends nothing: collect
        # until every rank has reported or exited
        while len(out) < world and time.monotonic() < deadline:
            try:
                rank, status, res = q.get(timeout=1.0)
                out[rank] = (status, res)
            except queue.Empty:
                if all(not p.is_alive() for p in procs) and q.empty():
                    break
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


class OracleOps:
    """The oracle's arithmetic behind the data plane's compute hooks (CPU ranks only)."""

    @staticmethod
    def attend(q, k, v, causal_diagonal, scale, out, lse):
        import oracle
        o, l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale, causal_diagonal)
        out.copy_(torch.from_numpy(o))
        lse.copy_(torch.from_numpy(l))

    @staticmethod
    def merge(o_a, lse_a, o_b, lse_b):
        import oracle
        o, l = oracle.lse_merge(o_a.numpy(), lse_a.numpy(), o_b.numpy(), lse_b.numpy())
        o_a.copy_(torch.from_numpy(o))
        lse_a.copy_(torch.from_numpy(l))

    @staticmethod
    def seq2head_pack(x, H_out, P):
        import oracle
        return torch.from_numpy(oracle.seq2head(x.numpy()[None], H_out, groups=P))

    @staticmethod
    def seq2head_unpack(recv):
        import oracle
        P, B, Lc, Hl, D = recv.shape
        return torch.from_numpy(oracle.seq2head(recv.numpy(), Hl, groups=1)).view(
            B, P * Lc, Hl, D)

    @staticmethod
    def head2seq_pack(y, P):
        import oracle
        return torch.from_numpy(oracle.head2seq(y.numpy()[None], P=P))

    @staticmethod
    def head2seq_unpack(recv):
        import oracle
        P, B, Lc, Hl, D = recv.shape
        return torch.from_numpy(oracle.head2seq(recv.numpy(), P=1)).view(B, Lc, P * Hl, D)


    @staticmethod
    def attend_bwd(q, k, v, out, lse, dout, causal_diagonal, scale, dq, dk, dv):
        import oracle
        a, b, c = oracle.attention_backward_pair(q.numpy(), k.numpy(), v.numpy(), out.numpy(),
                                                 lse.numpy(), dout.numpy(), scale,
                                                 causal_diagonal)
        dq += torch.from_numpy(a)
        dk += torch.from_numpy(b)
        dv += torch.from_numpy(c)


    @staticmethod
    def replica_sum(x, H_out):
        import oracle
        return torch.from_numpy(oracle.replica_sum(x.numpy(), H_out))


class RecordingOps(OracleOps):
    """Records the first element of every chunk a rank attends to (each rank's K/V is
    filled with its own rank index)."""
    seen = []

    @staticmethod
    def attend(q, k, v, causal_diagonal, scale, out, lse):
        RecordingOps.seen.append((int(k.flatten()[0].item()), int(v.flatten()[0].item()),
                                  bool(causal_diagonal)))
        out.zero_()
        lse.fill_(0.0)

    @staticmethod
    def merge(o_a, lse_a, o_b, lse_b):
        pass


# ------------------------------------------------------------------ ring
def _ring_holds(rank, world, causal):
    from sequence_parallelism_attn_b200 import dist as rd
    q = torch.zeros(1, 4, 2, 8, dtype=torch.float64)
    k = torch.full((1, 4, 1, 8), float(rank), dtype=torch.float64)
    v = torch.full((1, 4, 1, 8), float(100 + rank), dtype=torch.float64)
    RecordingOps.seen = []
    rd.ring_attn_fwd_dist(q, k, v, causal, 0.5, out=torch.empty(1, 4, 2, 8, dtype=torch.float64),
                          lse=torch.empty(1, 2, 4, dtype=torch.float64), ops=RecordingOps)
    return RecordingOps.seen


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_rank_holds_chunk_i_minus_s(world, causal):
    """Step s of rank i attends to the chunk that rank (i - s) mod P started with; causal:
    chunks after the rank's own are skipped, its own is the diagonal."""
    res = run_ranks(world, _ring_holds, causal)
    for rank in range(world):
        status, seen = res[rank]
        assert status == "ok", seen
        want = [(j, 100 + j, causal and j == rank) for j in
                [(rank - s) % world for s in range(world)] if not (causal and j > rank)]
        assert seen == want, (rank, seen, want)


def _ring_attention(rank, world, causal, B, Lc, H_q, H_kv, D):
    from sequence_parallelism_attn_b200 import dist as rd
    g = np.random.default_rng(11)
    L = world * Lc
    q = g.standard_normal((B, L, H_q, D)) * 2.0
    k = g.standard_normal((B, L, H_kv, D))
    v = g.standard_normal((B, L, H_kv, D))
    sl = slice(rank * Lc, (rank + 1) * Lc)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, sl]))
    out = torch.empty(B, Lc, H_q, D, dtype=torch.float64)
    lse = torch.empty(B, H_q, Lc, dtype=torch.float64)
    rd.ring_attn_fwd_dist(t(q), t(k), t(v), causal, 0.3, out=out, lse=lse, ops=OracleOps)
    import oracle
    want_o, want_l = oracle.attention(q, k, v, 0.3, causal)
    return (float(np.abs(out.numpy() - want_o[:, sl]).max()),
            float(np.abs(lse.numpy() - want_l[:, :, sl]).max()))


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_equals_whole_sequence(world, causal):
    """Each rank's merged result over the exchanged chunks equals attention of its queries
    over the whole sequence (GQA 4:2, B = 2)."""
    res = run_ranks(world, _ring_attention, causal, 2, 6, 4, 2, 8)
    for rank in range(world):
        status, errs = res[rank]
        assert status == "ok", errs
        assert errs[0] <= 1e-12 and errs[1] <= 1e-12, (rank, errs)


def _ring_backward(rank, world, causal, B, Lc, H_q, H_kv, D):
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    g = np.random.default_rng(23)
    L = world * Lc
    q = g.standard_normal((B, L, H_q, D)) * 2.0
    k = g.standard_normal((B, L, H_kv, D))
    v = g.standard_normal((B, L, H_kv, D))
    dout = g.standard_normal((B, L, H_q, D))
    out, lse = oracle.attention(q, k, v, 0.3, causal)  # the forward over the whole sequence
    sl = slice(rank * Lc, (rank + 1) * Lc)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, sl]))
    dq, dk, dv = rd.ring_attn_bwd_dist(t(q), t(k), t(v), t(out),
                                       torch.from_numpy(np.ascontiguousarray(lse[:, :, sl])),
                                       t(dout), causal, 0.3, ops=OracleOps)
    want = oracle.attention_backward(q, k, v, dout, 0.3, causal)
    return [float(np.abs(got.numpy() - w[:, sl]).max()) for got, w in zip((dq, dk, dv), want)]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_equals_whole_sequence_gradients(world, causal):
    """The ring backward across ranks (K/V chunks travelling with their dK, dV accumulators,
    every rank adding its queries' share, the last pass returning them home) gives each
    rank the gradients of its chunks of the whole-sequence attention (GQA 4:2, B = 2)."""
    res = run_ranks(world, _ring_backward, causal, 2, 6, 4, 2, 8)
    for rank in range(world):
        status, errs = res[rank]
        assert status == "ok", errs
        assert max(errs) <= 1e-12, (rank, errs)


def _ring_backward_accumulators(rank, world, causal):
    """Each rank's chunk of K and V filled with the rank index + 1; the attend hook adds 1
    to every accumulator it receives and records the chunk's first K value."""
    from sequence_parallelism_attn_b200 import dist as rd
    seen = []

    class Ops(OracleOps):
        @staticmethod
        def attend_bwd(q, k, v, out, lse, dout, causal_diagonal, scale, dq, dk, dv):
            seen.append((int(k.flatten()[0].item()), bool(causal_diagonal)))
            dk += 1.0
            dv += 2.0

    z = torch.zeros(1, 3, 2, 4, dtype=torch.float64)
    k = torch.full((1, 3, 1, 4), float(rank + 1), dtype=torch.float64)
    _, dk, dv = rd.ring_attn_bwd_dist(z, k, k.clone(), z, torch.zeros(1, 2, 3, dtype=torch.float64),
                                      z, causal, 0.5, ops=Ops)
    return seen, float(dk.flatten()[0]), float(dv.flatten()[0])


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_accumulators_visit_every_rank_and_return(world, causal):
    """A chunk's accumulators come back to its own rank having collected one share from
    every rank that attends to it: all P ranks when not causal, ranks j .. P-1 for chunk j
    when causal (the chunk's own rank on the diagonal)."""
    res = run_ranks(world, _ring_backward_accumulators, causal)
    for rank in range(world):
        status, val = res[rank]
        assert status == "ok", val
        seen, dk0, dv0 = val
        want_seen = [(j + 1, causal and j == rank) for j in
                     [(rank - s) % world for s in range(world)] if not (causal and j > rank)]
        assert seen == want_seen, (rank, seen, want_seen)
        visits = world - rank if causal else world
        assert (dk0, dv0) == (float(visits), 2.0 * visits), (rank, dk0, dv0)


def _zigzag_ring(rank, world, B, Lc, H_q, H_kv, D):
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    g = np.random.default_rng(17)
    L = world * Lc
    q = g.standard_normal((B, L, H_q, D)) * 2.0   # natural (sequence) order
    k = g.standard_normal((B, L, H_kv, D))
    v = g.standard_normal((B, L, H_kv, D))
    pos = oracle.zigzag_positions(world, Lc)[rank * Lc:(rank + 1) * Lc]  # this shard's tokens
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, pos]))
    out, lse = rd.ring_attn_fwd_zigzag_dist(t(q), t(k), t(v), 0.3, ops=OracleOps)
    want_o, want_l = oracle.attention(q, k, v, 0.3, True)
    return (float(np.abs(out.numpy() - want_o[:, pos]).max()),
            float(np.abs(lse.numpy() - want_l[:, :, pos]).max()))


def _zigzag_ring_backward(rank, world, B, Lc, H_q, H_kv, D):
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    g = np.random.default_rng(29)
    L = world * Lc
    q = g.standard_normal((B, L, H_q, D)) * 2.0   # natural (sequence) order
    k = g.standard_normal((B, L, H_kv, D))
    v = g.standard_normal((B, L, H_kv, D))
    do = g.standard_normal((B, L, H_q, D))
    out, lse = oracle.attention(q, k, v, 0.3, True)
    pos = oracle.zigzag_positions(world, Lc)[rank * Lc:(rank + 1) * Lc]  # this shard's tokens
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, pos]))
    dq, dk, dv = rd.ring_attn_bwd_zigzag_dist(
        t(q), t(k), t(v), t(out), torch.from_numpy(np.ascontiguousarray(lse[:, :, pos])), t(do),
        0.3, ops=OracleOps)
    want = oracle.attention_backward(q, k, v, do, 0.3, True)
    return [float(np.abs(got.numpy() - w[:, pos]).max()) for got, w in zip((dq, dk, dv), want)]


@pytest.mark.parametrize("world", [2, 4])
def test_zigzag_ring_backward_equals_causal_gradients(world):
    """The zigzag ring's backward (shard halves, dK / dV accumulators travelling with the
    shards): each rank's gradients equal those of causal attention over the sequence in
    natural order, mapped to its shard (GQA 4:2, B = 2)."""
    res = run_ranks(world, _zigzag_ring_backward, 2, 6, 4, 2, 8)
    for rank in range(world):
        status, errs = res[rank]
        assert status == "ok", errs
        assert max(errs) <= 1e-12, (rank, errs)


@pytest.mark.parametrize("world", [2, 4])
def test_zigzag_ring_equals_causal_attention(world):
    """Shards in the zigzag layout (rank i holds segments i and 2P-1-i): each rank's rows
    equal causal attention over the sequence in natural order (GQA 4:2, B = 2)."""
    res = run_ranks(world, _zigzag_ring, 2, 6, 4, 2, 8)
    for rank in range(world):
        status, errs = res[rank]
        assert status == "ok", errs
        assert errs[0] <= 1e-12 and errs[1] <= 1e-12, (rank, errs)


# ------------------------------------------------------------------ Ulysses
def _ulysses(rank, world, B, Lc, H_q, H_kv, D):
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    g = np.random.default_rng(5)
    x = g.standard_normal((world, B, Lc, H_kv, D)).astype(np.float32)  # every rank's shard
    H_out = int(np.lcm(H_kv, world))
    y = rd.ulysses_seq2head_dist(torch.from_numpy(x[rank]), H_out, ops=OracleOps)
    want = oracle.seq2head(x, H_out)[rank]                             # [B, P*Lc, Hl, D]
    ok_fwd = y.numpy().tobytes() == want.tobytes() and y.shape == want.shape
    h = g.standard_normal((world, B, world * Lc, H_q // world, D)).astype(np.float32)
    z = rd.ulysses_head2seq_dist(torch.from_numpy(h[rank]), ops=OracleOps)
    want_z = oracle.head2seq(h)[rank]                                   # [B, Lc, H_q, D]
    ok_back = z.numpy().tobytes() == want_z.tobytes() and z.shape == want_z.shape
    return ok_fwd, ok_back


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("B", [1, 2])
def test_ulysses_pack_all_to_all_unpack_bit_exact(world, B):
    """pack -> all-to-all -> unpack on every rank equals that rank's block of the oracle's
    seq->head over all shards (with the GQA copy of 2 KV heads), and head->seq likewise."""
    res = run_ranks(world, _ulysses, B, 5, 8, 2, 4)
    for rank in range(world):
        status, ok = res[rank]
        assert status == "ok", ok
        assert ok == (True, True), (rank, ok)


# ------------------------------------------------------------------ ring x Ulysses (USP)
def _usp(rank, world, P_u, causal):
    import torch.distributed as dist
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    P_r = world // P_u
    # every rank creates every group, in the same order
    ulysses = [dist.new_group([g * P_u + u for u in range(P_u)]) for g in range(P_r)]
    rings = [dist.new_group([g * P_u + u for g in range(P_r)]) for u in range(P_u)]
    B, Ls, H_q, H_kv, D = 2, 5, 4, 1, 8
    rng = np.random.default_rng(21)
    q = rng.standard_normal((world, B, Ls, H_q, D)) * 2.0
    k = rng.standard_normal((world, B, Ls, H_kv, D))
    v = rng.standard_normal((world, B, Ls, H_kv, D))
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[rank]))
    out, lse = rd.usp_attn_fwd_dist(t(q), t(k), t(v), causal, 0.3,
                                    ulysses_group=ulysses[rank // P_u],
                                    ring_group=rings[rank % P_u], ops=OracleOps)
    seq = lambda x: np.concatenate(list(x), axis=1)  # [B, world * Ls, H, D]
    want_o, want_l = oracle.attention(seq(q), seq(k), seq(v), 0.3, causal)
    sl = slice(rank * Ls, (rank + 1) * Ls)
    u = rank % P_u
    Hl = H_q // P_u
    eo = float(np.abs(out.numpy() - want_o[:, sl]).max())
    g = rank // P_u  # the Ulysses group's tokens: the ring chunk g
    gsl = slice(g * P_u * Ls, (g + 1) * P_u * Ls)
    el = float(np.abs(lse.numpy() - want_l[:, u * Hl:(u + 1) * Hl, gsl]).max())
    return eo, el


@pytest.mark.parametrize("P_u,causal", [(2, True), (2, False), (4, True), (1, True)])
def test_usp_across_ranks_equals_whole_sequence(P_u, causal):
    """4 ranks as P_r ring groups x P_u Ulysses ranks (2 x 2, 1 x 4, 4 x 1): each rank's
    output rows, and its head block's LSE over its group's tokens, equal attention over the
    whole sequence (one KV head copied up to P_u)."""
    res = run_ranks(4, _usp, P_u, causal)
    for rank in range(4):
        status, errs = res[rank]
        assert status == "ok", errs
        assert errs[0] <= 1e-12 and errs[1] <= 1e-12, (rank, errs)


def _usp_backward(rank, world, P_u, causal, H_kv):
    import torch.distributed as dist
    from sequence_parallelism_attn_b200 import dist as rd
    import oracle
    P_r = world // P_u
    ulysses = [dist.new_group([g * P_u + u for u in range(P_u)]) for g in range(P_r)]
    rings = [dist.new_group([g * P_u + u for g in range(P_r)]) for u in range(P_u)]
    B, Ls, H_q, D = 2, 5, 4, 8
    rng = np.random.default_rng(31)
    q = rng.standard_normal((world, B, Ls, H_q, D)) * 2.0
    k = rng.standard_normal((world, B, Ls, H_kv, D))
    v = rng.standard_normal((world, B, Ls, H_kv, D))
    do = rng.standard_normal((world, B, Ls, H_q, D))
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x[rank]))
    kw = dict(ulysses_group=ulysses[rank // P_u], ring_group=rings[rank % P_u], ops=OracleOps)
    out, lse = rd.usp_attn_fwd_dist(t(q), t(k), t(v), causal, 0.3, **kw)
    dq, dk, dv = rd.usp_attn_bwd_dist(t(q), t(k), t(v), out, lse, t(do), causal, 0.3, **kw)
    seq = lambda x: np.concatenate(list(x), axis=1)  # [B, world * Ls, H, D]
    want = oracle.attention_backward(seq(q), seq(k), seq(v), seq(do), 0.3, causal)
    sl = slice(rank * Ls, (rank + 1) * Ls)
    return [float(np.abs(g.numpy() - w[:, sl]).max()) for g, w in zip((dq, dk, dv), want)]


@pytest.mark.parametrize("P_u,causal,H_kv", [(2, True, 1), (2, False, 2), (4, True, 1),
                                             (4, True, 4), (1, True, 1)])
def test_usp_backward_across_ranks_equals_whole_sequence_gradients(P_u, causal, H_kv):
    """The backward of the ring x Ulysses hybrid at four ranks (2 x 2, 1 x 4 = plain
    Ulysses, 4 x 1 = plain ring): seq->head of q, k, v, out, dout, the ring backward on the
    head blocks, head->seq of the gradients and the sum of each KV head's replicas give every
    rank its shard's gradients of whole-sequence attention (one, two or four KV heads: copied
    up to P_u or not at all)."""
    res = run_ranks(4, _usp_backward, P_u, causal, H_kv)
    for rank in range(4):
        status, errs = res[rank]
        assert status == "ok", errs
        assert max(errs) <= 1e-12, (rank, errs)


# ------------------------------------------------------------------ a rank that leaves
def _leaver(rank, world, leave_rank):
    from sequence_parallelism_attn_b200 import dist as rd
    if rank == leave_rank:
        os._exit(0)  # leaves between steps: never posts its exchange
    q = torch.zeros(1, 4, 2, 8, dtype=torch.float64)
    k = torch.zeros(1, 4, 1, 8, dtype=torch.float64)
    try:
        rd.ring_attn_fwd_dist(q, k, k.clone(), True, 0.5,
                              out=torch.empty(1, 4, 2, 8, dtype=torch.float64),
                              lse=torch.empty(1, 2, 4, dtype=torch.float64), ops=RecordingOps)
    except rd.ExchangeError as e:
        return "ExchangeError: " + str(e)[:200]
    return "completed"


def _leaver_bwd(rank, world, leave_rank):
    from sequence_parallelism_attn_b200 import dist as rd
    if rank == leave_rank:
        os._exit(0)  # leaves between steps: never posts its exchange
    z = torch.zeros(1, 4, 2, 8, dtype=torch.float64)
    k = torch.zeros(1, 4, 1, 8, dtype=torch.float64)
    try:
        rd.ring_attn_bwd_dist(z, k, k.clone(), z, torch.zeros(1, 2, 4, dtype=torch.float64), z,
                              True, 0.5, ops=RecordingOps)
    except rd.ExchangeError as e:
        return "ExchangeError: " + str(e)[:200]
    return "completed"


def test_rank_leaving_the_ring_backward_is_reported_not_hung():
    """Rank 1 of 2 exits before the ring backward's first exchange: rank 0 gets an
    ExchangeError within the process group's timeout."""
    res = run_ranks(2, _leaver_bwd, 1, timeout=90)
    assert 1 not in res
    status, msg = res[0]
    assert status == "ok" and msg.startswith("ExchangeError"), msg


def test_rank_leaving_is_reported_not_hung():
    """Rank 2 of 3 exits before the ring's first exchange: its ring neighbours get an
    ExchangeError within the process group's timeout instead of waiting for good."""
    res = run_ranks(3, _leaver, 2, timeout=90)
    assert 2 not in res
    # rank 0 receives from rank 2: its exchange must fail
    status, msg = res[0]
    assert status == "ok" and msg.startswith("ExchangeError"), msg
    # rank 1 sends to rank 2 and receives from rank 0; it ends with an error too (its
    # neighbour rank 0 gave up), never by waiting for good
    status, msg = res[1]
    assert status == "ok" and msg.startswith("ExchangeError"), msg


def test_peer_exchange_rejects_mismatched_buffers():
    """The one-kernel exchange checks its buffers before any barrier or kernel: a buffer of
    another shape or dtype, heads that do not split over the ranks, or exchanges over two
    groups in one barrier pair are refused (no process group, no GPU needed)."""
    from types import SimpleNamespace
    import torch
    from sequence_parallelism_attn_b200 import dist as rd

    def peer(shape, dtype=torch.bfloat16, world=2, group=None):
        def sync(what):
            raise AssertionError("no barrier may run for refused arguments")
        return SimpleNamespace(buf=torch.empty(shape, dtype=dtype), world=world, rank=0,
                               ptrs=[0] * world, group=group, sync=sync)

    x = torch.empty(1, 16, 2, 64, dtype=torch.bfloat16)       # B, Lc, H_in, D
    with pytest.raises(ValueError):
        rd.ulysses_seq2head_p2p(x, peer((1, 32, 1, 64)), 4)   # wants (1, 32, 2, 64)
    with pytest.raises(ValueError):
        rd.ulysses_seq2head_p2p(x, peer((1, 32, 2, 64), torch.float32), 4)
    with pytest.raises(ValueError):
        rd.ulysses_seq2head_p2p(x, peer((1, 32, 1, 64)), 3)   # 3 heads over 2 ranks
    with pytest.raises(ValueError):
        rd.ulysses_seq2head_p2p_many([(x, peer((1, 32, 2, 64), group="a"), 4),
                                      (x, peer((1, 32, 2, 64), group="b"), 4)])
    y = torch.empty(1, 32, 2, 64, dtype=torch.bfloat16)       # B, P*Lc, Hl, D
    with pytest.raises(ValueError):
        rd.ulysses_head2seq_p2p(y, peer((1, 16, 2, 64)))      # wants (1, 16, 4, 64)
