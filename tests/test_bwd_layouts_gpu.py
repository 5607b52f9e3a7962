"""GPU parity of the backward pass in the zigzag shard layout (ra_ring_attn_bwd_zigzag) and
over packed samples (ra_ring_attn_bwd_packed) against the fp64 oracle's gradients, every
element.

Zigzag: the gradients of attention over the natural token order, computed by the oracle on
the tokens put in sequence order (the oracle's zigzag_positions) and mapped back to the
shards.  Packed: every gradient sums only the pairs the forward attended, so each sample's
gradients are the oracle's gradients of its own causal attention.  Tolerance as for the
contiguous backward: max|error| <= 1e-2 max|reference| per gradient tensor, plus 1e-4 for
gradients that vanish analytically.

Sources: "Метод контекстного параллелизма Ulysses" (introduction: the zigzag layout named
beside the ring); "Paralelismo de secuencias en 🤗 accelerate", section "Configuración del
backend SP de ALST/Ulysses" (position_ids, several samples in one sequence); the gradient
is the derivative of the forward of "Как работает sequence parallelism в контексте LLM?"
sections 2, 3, 5."""
import zlib

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import assert_same_grads, check_grad, chunks_to_seq, f64

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module", autouse=True)
def _short_waits(ra_lib):
    old = ra_lib.ra_set_wait_limit_ns(2_000_000_000)
    yield
    ra_lib.ra_set_wait_limit_ns(old)


def problem(name, B, H_q, H_kv, D, P, Lc, causal, q_mult=1.0):
    w = synth.AttnWorkload(name, B=B, H_q=H_q, H_kv=H_kv, D=D, P=P, Lc=Lc,
                           dtype=torch.bfloat16, causal=causal, q_mult=q_mult,
                           seed=zlib.crc32(name.encode()) % 100000)
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return w, q, k, v, dout


def compare(name, got, want):
    for nm, a, b in zip(("dq", "dk", "dv"), got, want):
        check_grad(name, nm, f64(a) if isinstance(a, torch.Tensor) else a, b)


def gpu_grads(ra_lib, w, q, k, v, dout, **layout):
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, l = ra_lib.ring_attn_fwd(qc, kc, vc, w.causal, w.scale, out_dtype=torch.bfloat16, **layout)
    dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, w.causal, w.scale, **layout)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    return dq, chunks_to_seq(dk), chunks_to_seq(dv)


# ------------------------------------------------------------------ zigzag
def check_zigzag(ra_lib, oracle_mod, name, B, H_q, H_kv, D, P, Lc, causal, q_mult=1.0):
    w, q, k, v, dout = problem(name, B, H_q, H_kv, D, P, Lc, causal, q_mult)
    got = gpu_grads(ra_lib, w, q, k, v, dout, layout="zigzag")
    pos = oracle_mod.zigzag_positions(P, Lc)  # shard-major token -> sequence position
    inv = np.argsort(pos)                     # sequence position -> shard-major token
    rq, rk, rv = oracle_mod.attention_backward(f64(q)[:, inv], f64(chunks_to_seq(k))[:, inv],
                                               f64(chunks_to_seq(v))[:, inv], f64(dout)[:, inv],
                                               w.scale, causal)
    compare(f"zigzag {name}", got, (rq[:, pos], rk[:, pos], rv[:, pos]))


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("P,Lc", [(2, 256), (4, 200), (3, 384), (5, 2), (1, 300), (8, 128)])
def test_bwd_zigzag_every_element(ra_lib, oracle_mod, D, P, Lc):
    """Tiles straddling the shard's two segments (Lc/2 not a multiple of 128), one-token
    segments (Lc = 2), one rank, GQA 4:2, B = 2."""
    check_zigzag(ra_lib, oracle_mod, f"zz_{D}_{P}_{Lc}", 2, 4, 2, D, P, Lc, True, q_mult=2.0)


def test_bwd_zigzag_8k_gqa(ra_lib, oracle_mod):
    check_zigzag(ra_lib, oracle_mod, "zz_8k", 1, 8, 2, 128, 8, 1024, True)


def test_bwd_zigzag_noncausal_equals_contiguous(ra_lib):
    """Without a causal mask positions play no role: both layouts give the same gradients
    (dK, dV bit for bit, dQ up to the order of its reduce-adds)."""
    w, q, k, v, dout = problem("zz_nc", 2, 4, 2, 128, 3, 200, False)
    a = gpu_grads(ra_lib, w, q, k, v, dout)
    b = gpu_grads(ra_lib, w, q, k, v, dout, layout="zigzag")
    assert_same_grads(a, b, "zigzag non-causal vs contiguous")


def test_bwd_zigzag_odd_chunk_rejected(ra_lib):
    w, q, k, v, dout = problem("zz_odd", 1, 2, 2, 128, 2, 129, True)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.B, w.H_q, w.L), device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ring_attn_bwd(qc, kc, vc, o, lse, dout.cuda(), True, w.scale, layout="zigzag")
    assert e.value.status == 1


# ------------------------------------------------------------------ packed samples
def check_packed(ra_lib, oracle_mod, name, B, H_q, H_kv, D, P, Lc, lengths, q_mult=1.0):
    w, q, k, v, dout = problem(name, B, H_q, H_kv, D, P, Lc, True, q_mult)
    pid = synth.position_ids_from_lengths(lengths)
    got = gpu_grads(ra_lib, w, q, k, v, dout, position_ids=pid.cuda())
    ks, vs = chunks_to_seq(k), chunks_to_seq(v)
    want = [np.zeros(t.shape) for t in (q, ks, vs)]
    for b in range(B):
        starts = np.concatenate([[0], np.cumsum(lengths[b])])
        for s0, s1 in zip(starts[:-1], starts[1:]):
            sl = slice(int(s0), int(s1))
            g = oracle_mod.attention_backward(f64(q[b:b + 1, sl]), f64(ks[b:b + 1, sl]),
                                              f64(vs[b:b + 1, sl]), f64(dout[b:b + 1, sl]),
                                              w.scale, True)
            for out, part in zip(want, g):
                out[b, sl] = part[0]
    compare(f"packed {name}", got, want)


@pytest.mark.parametrize("D", [128, 64])
def test_bwd_packed_mixed_lengths(ra_lib, oracle_mod, D):
    """600 tokens per row: one-token and chunk-crossing samples in row 0, samples ending on
    128-token tile edges in row 1."""
    check_packed(ra_lib, oracle_mod, f"pk_{D}", 2, 4, 2, D, 3, 200,
                 [[1, 1, 150, 77, 1, 300, 70], [128, 128, 256, 88]], q_mult=2.0)


def test_bwd_packed_many_short_samples(ra_lib, oracle_mod):
    lens = [synth.packed_lengths(1024, 11 + b, 1, 40) for b in range(2)]
    check_packed(ra_lib, oracle_mod, "pk_short", 2, 4, 2, 128, 4, 256, lens)


def test_bwd_packed_one_token_samples(ra_lib, oracle_mod):
    check_packed(ra_lib, oracle_mod, "pk_ones", 1, 4, 2, 128, 2, 128, [[1] * 256])


def test_bwd_packed_8k_documents(ra_lib, oracle_mod):
    lens = synth.packed_lengths(8192, 77, 64, 2048)
    check_packed(ra_lib, oracle_mod, "pk_8k", 1, 8, 2, 128, 8, 1024, [lens])


def test_bwd_packed_single_sample_equals_causal(ra_lib):
    """One sample per row (position_ids = 0 .. L-1): the contiguous causal result (dK, dV bit
    for bit, dQ up to the order of its reduce-adds)."""
    w, q, k, v, dout = problem("pk_one", 2, 4, 2, 128, 3, 200, True)
    a = gpu_grads(ra_lib, w, q, k, v, dout)
    pid = synth.position_ids_from_lengths([[w.L]] * w.B).cuda()
    b = gpu_grads(ra_lib, w, q, k, v, dout, position_ids=pid)
    assert_same_grads(a, b, "packed single sample vs causal")


def test_bwd_packed_null_ids_rejected(ra_lib):
    w, q, k, v, dout = problem("pk_null", 1, 2, 2, 128, 2, 128, True)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    g = [torch.empty(t.shape, device="cuda") for t in (q, k, v)]
    o = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.B, w.H_q, w.L), device="cuda")
    ws = torch.empty((w.B, w.H_q, w.L), device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ra_ring_attn_bwd_packed(
            qc.data_ptr(), [kc[j].data_ptr() for j in range(w.P)],
            [vc[j].data_ptr() for j in range(w.P)], None, o.data_ptr(), lse.data_ptr(),
            dout.cuda().data_ptr(), w.P, w.B, w.H_q, w.H_kv, w.Lc, w.D, w.L * w.H_q * w.D,
            w.Lc * w.H_kv * w.D, w.scale, g[0].data_ptr(), [g[1][j].data_ptr() for j in range(w.P)],
            [g[2][j].data_ptr() for j in range(w.P)], ws.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    assert e.value.status == 1
