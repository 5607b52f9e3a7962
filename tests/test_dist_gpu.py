"""The multi-GPU data plane's computations on one GPU: the ring's per-step attention and
merge (RingAccumulator with the library's kernels) for P virtual ranks visiting the chunks
in ring order, against the oracle's attention over the whole sequence; the ring backward's
per-step accumulating calls against the oracle's gradients; the Ulysses pack and
unpack kernels around an all-to-all emulated on the device, bit for bit against the
oracle's seq->head / head->seq; and the distributed functions themselves through a
one-rank NCCL process group.  The exchanges between ranks are tested on CPU ranks
(tests/test_dist_host.py).

Sources: "Как работает sequence parallelism в контексте LLM?" sections 3 and 5; "Метод
контекстного параллелизма Ulysses"."""
import socket

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import dist as rd
from _util import TOL, check_grad, f64, max_abs

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    return t.view(torch.int32).numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("P", [1, 4])
def test_ring_steps_equal_whole_sequence(ra_lib, oracle_mod, P, causal):
    """Every virtual rank's accumulator over its ring steps (attention launches per held
    chunk, merges by ra_lse_merge) equals attention of its queries over the whole sequence,
    every row (B = 2, ragged chunks of 200 tokens, GQA 4:2, bf16)."""
    B, Lc, H_q, H_kv, D = 2, 200, 4, 2, 128
    g = torch.Generator().manual_seed(300 + P)
    L = P * Lc
    q = (torch.randn(B, L, H_q, D, generator=g) * 2).to(torch.bfloat16)
    k = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    scale = D ** -0.5
    want_o, want_l = oracle_mod.attention(f64(q), f64(k), f64(v), scale, causal)
    shard = lambda x, i: x[:, i * Lc:(i + 1) * Lc].contiguous().cuda()
    for i in range(P):
        acc = rd.RingAccumulator(shard(q, i), i, causal, scale)
        for j in rd.ring_schedule(i, P):
            acc.visit(j, shard(k, j), shard(v, j))
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
        sl = slice(i * Lc, (i + 1) * Lc)
        eo = max_abs(f64(acc.out), want_o[:, sl])
        el = max_abs(f64(acc.lse), want_l[:, :, sl])
        print(f"[parity] ring steps P={P} causal={causal} rank {i}: max|dO|={eo:.3e} "
              f"max|dLSE|={el:.3e}")
        assert eo <= TOL[torch.bfloat16][0] and el <= TOL[torch.bfloat16][1]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("P", [1, 3])
def test_ring_backward_steps_equal_whole_sequence_gradients(ra_lib, oracle_mod, P, causal):
    """The ring backward's per-step calls (ra_ring_attn_bwd_accumulate: each virtual rank's
    queries against every K/V chunk it visits, with the forward's final out and LSE, adding
    into its dq and into the chunk's dK, dV accumulators) sum to the gradients of attention
    over the whole sequence, every element (B = 2, ragged chunks of 200 tokens, GQA 4:2,
    bf16 in, fp32 gradients)."""
    B, Lc, H_q, H_kv, D = 2, 200, 4, 2, 128
    g = torch.Generator().manual_seed(700 + P)
    L = P * Lc
    q = (torch.randn(B, L, H_q, D, generator=g) * 2).to(torch.bfloat16)
    k = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    dout = torch.randn(B, L, H_q, D, generator=g).to(torch.bfloat16)
    scale = D ** -0.5
    # the forward over the whole sequence gives each chunk's final out (bf16) and LSE
    kc = k.view(B, P, Lc, H_kv, D).transpose(0, 1).contiguous().cuda()
    vc = v.view(B, P, Lc, H_kv, D).transpose(0, 1).contiguous().cuda()
    o, l = ra_lib.ring_attn_fwd(q.cuda(), kc, vc, causal, scale, out_dtype=torch.bfloat16)
    shard = lambda x, i: x[:, i * Lc:(i + 1) * Lc].contiguous().cuda()
    dq = torch.zeros(B, L, H_q, D, device="cuda")
    dk = torch.zeros(P, B, Lc, H_kv, D, device="cuda")
    dv = torch.zeros_like(dk)
    for i in range(P):
        dqi = torch.zeros(B, Lc, H_q, D, device="cuda")
        for j in rd.ring_schedule(i, P):
            kind = rd.chunk_pair(i, j, causal)
            if kind == "skip":
                continue
            rd.DeviceOps.attend_bwd(shard(q, i), kc[j, :], vc[j, :], o[:, i * Lc:(i + 1) * Lc].contiguous(),
                                    l[:, :, i * Lc:(i + 1) * Lc].contiguous(), shard(dout, i),
                                    kind == "diagonal", scale, dqi, dk[j], dv[j])
        dq[:, i * Lc:(i + 1) * Lc] = dqi
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    rq, rk, rv = oracle_mod.attention_backward(f64(q), f64(k), f64(v), f64(dout), scale, causal)
    seq = lambda x: x.transpose(0, 1).reshape(B, L, H_kv, D)
    name = f"ring backward steps P={P} causal={causal}"
    check_grad(name, "dq", f64(dq), rq)
    check_grad(name, "dk", f64(seq(dk)), rk)
    check_grad(name, "dv", f64(seq(dv)), rv)


@pytest.mark.parametrize("B,P,Lc", [(1, 4, 256), (2, 3, 200)])
def test_zigzag_ring_steps_equal_causal_attention(ra_lib, oracle_mod, B, P, Lc):
    """Every virtual rank's zigzag accumulator over its ring steps (attention launches on
    shard halves, merges by ra_lse_merge) equals causal attention over the natural-order
    sequence, every row; and agrees with the one-launch zigzag kernel on the same shards."""
    H_q, H_kv, D = 4, 2, 128
    g = torch.Generator().manual_seed(600 + P)
    L = P * Lc
    q = (torch.randn(B, L, H_q, D, generator=g) * 2).to(torch.bfloat16)  # natural order
    k = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, H_kv, D, generator=g).to(torch.bfloat16)
    scale = D ** -0.5
    want_o, want_l = oracle_mod.attention(f64(q), f64(k), f64(v), scale, True)
    pos = oracle_mod.zigzag_positions(P, Lc)
    shard = lambda x, i: x[:, torch.from_numpy(pos[i * Lc:(i + 1) * Lc])].contiguous().cuda()
    qz = torch.cat([shard(q, i) for i in range(P)], dim=1)  # rank-major zigzag shards
    kz = torch.stack([shard(k, i) for i in range(P)])
    vz = torch.stack([shard(v, i) for i in range(P)])
    one_o, one_l = ra_lib.ring_attn_fwd(qz, kz, vz, True, scale, layout="zigzag")
    for i in range(P):
        acc = rd.ZigzagRingAccumulator(shard(q, i), i, P, scale)
        for j in rd.ring_schedule(i, P):
            acc.visit(j, shard(k, j), shard(v, j))
        out, lse = acc.result()
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
        p_i = pos[i * Lc:(i + 1) * Lc]
        eo = max_abs(f64(out), want_o[:, p_i])
        el = max_abs(f64(lse), want_l[:, :, p_i])
        print(f"[parity] zigzag ring steps P={P} B={B} rank {i}: max|dO|={eo:.3e} "
              f"max|dLSE|={el:.3e}")
        assert eo <= TOL[torch.bfloat16][0] and el <= TOL[torch.bfloat16][1]
        sl = slice(i * Lc, (i + 1) * Lc)
        assert max_abs(f64(out), f64(one_o[:, sl])) <= 2e-2
        assert max_abs(f64(lse), f64(one_l[:, :, sl])) <= 2e-3


@pytest.mark.parametrize("B,dtype", [(1, torch.bfloat16), (2, torch.bfloat16),
                                     (2, torch.float32)])
def test_ulysses_pack_unpack_bit_exact(ra_lib, oracle_mod, B, dtype):
    """pack on every virtual rank, the all-to-all emulated on the device (block r of rank s
    to rank r), unpack: each rank's result is its block of the oracle's seq->head, with the
    GQA copy of 2 KV heads to 4; and head->seq likewise."""
    P, Lc, H_kv, H_q, D = 4, 96, 2, 8, 128
    g = torch.Generator().manual_seed(400 + B)
    x = torch.randn(P, B, Lc, H_kv, D, generator=g).to(dtype)
    H_out = int(np.lcm(H_kv, P))
    sends = [rd.DeviceOps.seq2head_pack(x[s].cuda(), H_out, P) for s in range(P)]
    want = oracle_mod.seq2head(_bits(x), H_out)
    for r in range(P):
        recv = torch.stack([sends[s][r] for s in range(P)])
        y = rd.DeviceOps.seq2head_unpack(recv)
        assert y.shape == (B, P * Lc, H_out // P, D)
        assert np.array_equal(_bits(y), want[r])
    h = torch.randn(P, B, P * Lc, H_q // P, D, generator=g).to(dtype)
    sends = [rd.DeviceOps.head2seq_pack(h[r].cuda(), P) for r in range(P)]
    want = oracle_mod.head2seq(_bits(h))
    for s in range(P):
        recv = torch.stack([sends[r][s] for r in range(P)])
        z = rd.DeviceOps.head2seq_unpack(recv)
        assert z.shape == (B, Lc, H_q, D)
        assert np.array_equal(_bits(z), want[s])
    assert ra_lib.ra_sync_status() == 0


def test_distributed_functions_on_one_rank(ra_lib, oracle_mod):
    """ring_attn_fwd_dist, the Ulysses functions and their composition (USP) through a
    one-rank NCCL process group (the all-to-all moves one block to itself; the ring has one
    step)."""
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        B, Lc, H_q, H_kv, D = 1, 300, 4, 2, 128
        g = torch.Generator().manual_seed(501)
        q = torch.randn(B, Lc, H_q, D, generator=g).to(torch.bfloat16)
        k = torch.randn(B, Lc, H_kv, D, generator=g).to(torch.bfloat16)
        v = torch.randn(B, Lc, H_kv, D, generator=g).to(torch.bfloat16)
        o, l = rd.ring_attn_fwd_dist(q.cuda(), k.cuda(), v.cuda(), True, D ** -0.5)
        want_o, want_l = oracle_mod.attention(f64(q), f64(k), f64(v), D ** -0.5, True)
        assert max_abs(f64(o), want_o) <= 1e-2 and max_abs(f64(l), want_l) <= 1e-3
        y = rd.ulysses_seq2head_dist(k.cuda(), 2)
        assert np.array_equal(_bits(y), oracle_mod.seq2head(_bits(k)[None], 2)[0])
        z = rd.ulysses_head2seq_dist(y)
        assert np.array_equal(_bits(z), _bits(k))
        z2 = torch.full_like(z, float("nan"))
        rd.ulysses_head2seq_dist(y, out=z2)  # into a caller's buffer
        assert np.array_equal(_bits(z2), _bits(k))
        uo, ul = rd.usp_attn_fwd_dist(q.cuda(), k.cuda(), v.cuda(), True, D ** -0.5)
        assert max_abs(f64(uo), want_o) <= 1e-2 and max_abs(f64(ul), want_l) <= 1e-3
        # the ring backward on one rank: one diagonal step, the accumulators' one pass home
        dout = torch.randn(B, Lc, H_q, D, generator=g).to(torch.bfloat16)
        ob = o.to(torch.bfloat16)
        gq, gk, gv = rd.ring_attn_bwd_dist(q.cuda(), k.cuda(), v.cuda(), ob, l, dout.cuda(), True,
                                           D ** -0.5)
        rq, rk, rv = oracle_mod.attention_backward(f64(q), f64(k), f64(v), f64(dout), D ** -0.5,
                                                   True)
        check_grad("ring backward, one rank", "dq", f64(gq), rq)
        check_grad("ring backward, one rank", "dk", f64(gk), rk)
        check_grad("ring backward, one rank", "dv", f64(gv), rv)
        # the Ulysses / USP backward on one rank: transforms of one block, one ring step
        ub = uo.to(torch.bfloat16)
        uq, uk, uv = rd.usp_attn_bwd_dist(q.cuda(), k.cuda(), v.cuda(), ub, ul, dout.cuda(), True,
                                          D ** -0.5)
        check_grad("USP backward, one rank", "dq", f64(uq), rq)
        check_grad("USP backward, one rank", "dk", f64(uk), rk)
        check_grad("USP backward, one rank", "dv", f64(uv), rv)
        # the zigzag ring backward on one rank (its shard is the natural order): the three
        # half-pairs of the diagonal step
        zq, zk, zv = rd.ring_attn_bwd_zigzag_dist(q.cuda(), k.cuda(), v.cuda(), ob, l,
                                                  dout.cuda(), D ** -0.5)
        check_grad("zigzag ring backward, one rank", "dq", f64(zq), rq)
        check_grad("zigzag ring backward, one rank", "dk", f64(zk), rk)
        check_grad("zigzag ring backward, one rank", "dv", f64(zv), rv)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


def test_peer_exchange_on_one_rank(ra_lib, oracle_mod):
    """The one-kernel Ulysses exchange (symmetric-memory buffers, the scatter kernels, the
    barriers around them) through a one-rank NCCL process group: the buffers are set up and
    mapped, and seq->head / head->seq give the bits of the NCCL path's functions."""
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        B, Lc, H_in, H_out, D = 2, 300, 2, 4, 128
        g = torch.Generator().manual_seed(502)
        x = torch.randn(B, Lc, H_in, D, generator=g).to(torch.bfloat16).cuda()
        heads = rd.PeerBuffers((B, Lc, H_out, D), torch.bfloat16, device="cuda")
        seq = rd.PeerBuffers((B, Lc, H_out, D), torch.bfloat16, device="cuda")
        assert heads.ptrs == [heads.buf.data_ptr()]
        for _ in range(2):  # the buffers are reused across exchanges
            y = rd.ulysses_seq2head_p2p(x, heads, H_out)
            assert np.array_equal(_bits(y), _bits(rd.ulysses_seq2head_dist(x, H_out)))
            assert np.array_equal(_bits(y), oracle_mod.seq2head(_bits(x)[None], H_out)[0])
            z = rd.ulysses_head2seq_p2p(y, seq)
            assert np.array_equal(_bits(z), _bits(rd.ulysses_head2seq_dist(y)))
        with pytest.raises(ValueError):
            rd.ulysses_seq2head_p2p(x, seq, 8)  # buffers of another shape
        torch.cuda.synchronize()
        del heads, seq, y, z
    finally:
        dist.destroy_process_group()


def test_bench_dist_path_exchanges_agree_on_one_rank(ra_lib):
    """bench.py's multi-GPU Ulysses step through a one-rank NCCL group with either exchange
    (NCCL all-to-alls with pack / unpack, or the scatter kernels into symmetric memory):
    the same bits of O in the sequence layout."""
    import importlib.util
    import os
    import torch.distributed as dist
    from sequence_parallelism_attn_b200 import synth
    spec = importlib.util.spec_from_file_location(
        "bench", os.path.join(os.path.dirname(os.path.dirname(__file__)), "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = synth.UlyssesWorkload("dist_path_small", P=4, B=1, Lc=256, H_q=8, H_kv=2, D=128,
                                  dtype=torch.bfloat16, causal=True, seed=77)
        dev = torch.device("cuda", 0)
        outs = []
        for ex in ("nccl", "p2p"):
            path = bench.DistUlyssesPath(w, dev, 0, 1, exchange=ex)
            for _ in range(2):
                path.step()
            torch.cuda.synchronize()
            outs.append(path.result().clone())
            del path
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
        assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    finally:
        dist.destroy_process_group()
