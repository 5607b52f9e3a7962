"""GPU tests of the deterministic backward (ra_set_bwd_deterministic(1)): dQ computed by the
query-stationary kernel, each element summed over the key tiles in one fixed order and
written once, while the key-stationary kernel computes dK and dV alone.

Checked: every gradient element against the fp64 oracle in the three shard layouts
(contiguous, zigzag, packed samples), at D = 64 and 128, over ragged and degenerate sizes;
two calls agree bit for bit on all three gradients; dK and dV are the bits of the default
mode and dQ is the default mode's up to the order of its reduce-adds; the accumulating
entry point adds the same bits a plain call returns.  Tolerances as in test_bwd_gpu.py.

Source: the backward of the forward computed in "Как работает sequence parallelism в
контексте LLM?" sections 2, 3, 5 (the pages train with ring attention; the gradient is
the derivative of the definition)."""
import zlib

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import assert_same_grads, check_grad, chunks_to_seq, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _deterministic(ra_lib):
    old_wait = ra_lib.ra_set_wait_limit_ns(2_000_000_000)
    old = ra_lib.ra_set_bwd_deterministic(True)
    yield
    ra_lib.ra_set_bwd_deterministic(old)
    ra_lib.ra_set_wait_limit_ns(old_wait)


def problem(name, B, H_q, H_kv, D, P, Lc, causal, q_mult=1.0):
    w = synth.AttnWorkload(name, B=B, H_q=H_q, H_kv=H_kv, D=D, P=P, Lc=Lc,
                           dtype=torch.bfloat16, causal=causal, q_mult=q_mult,
                           seed=zlib.crc32(name.encode()) % 100000)
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return w, q, k, v, dout


def grads(ra_lib, w, q, k, v, dout, **layout):
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, l = ra_lib.ring_attn_fwd(qc, kc, vc, w.causal, w.scale, out_dtype=torch.bfloat16, **layout)
    out = []
    for _ in range(2):
        dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, w.causal, w.scale, **layout)
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
        out.append((dq, dk, dv))
    for nm, a, b in zip(("dq", "dk", "dv"), out[0], out[1]):
        assert torch.equal(a, b), f"{w.name}: {nm} differs between two deterministic calls"
    return out[0]


def compare(name, got, want):
    for nm, a, b in zip(("dq", "dk", "dv"), got, want):
        check_grad(name, nm, f64(a), b)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("P,Lc", [(1, 256), (3, 200), (2, 129), (5, 1), (8, 512)])
def test_det_contiguous_every_element(ra_lib, oracle_mod, D, causal, P, Lc):
    w, q, k, v, dout = problem(f"det_{D}_{causal}_{P}_{Lc}", 2 if Lc < 512 else 1, 4, 2, D, P,
                               Lc, causal, q_mult=2.0)
    dq, dk, dv = grads(ra_lib, w, q, k, v, dout)
    want = oracle_mod.attention_backward(f64(q), f64(chunks_to_seq(k)), f64(chunks_to_seq(v)),
                                         f64(dout), w.scale, causal)
    compare(w.name, (dq, chunks_to_seq(dk), chunks_to_seq(dv)), want)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("P,Lc", [(2, 256), (4, 200), (3, 384), (5, 2)])
def test_det_zigzag_every_element(ra_lib, oracle_mod, D, P, Lc):
    w, q, k, v, dout = problem(f"det_zz_{D}_{P}_{Lc}", 1, 4, 2, D, P, Lc, True)
    dq, dk, dv = grads(ra_lib, w, q, k, v, dout, layout="zigzag")
    pos = oracle_mod.zigzag_positions(P, Lc)
    inv = np.argsort(pos)
    rq, rk, rv = oracle_mod.attention_backward(f64(q)[:, inv], f64(chunks_to_seq(k))[:, inv],
                                               f64(chunks_to_seq(v))[:, inv], f64(dout)[:, inv],
                                               w.scale, True)
    compare(w.name, (dq, chunks_to_seq(dk), chunks_to_seq(dv)),
            (rq[:, pos], rk[:, pos], rv[:, pos]))


@pytest.mark.parametrize("D", [128, 64])
def test_det_packed_every_element(ra_lib, oracle_mod, D):
    lengths = [[100, 1, 300, 111], [512]]
    w, q, k, v, dout = problem(f"det_pk_{D}", 2, 4, 2, D, 4, 128, True)
    pid = synth.position_ids_from_lengths(lengths)
    dq, dk, dv = grads(ra_lib, w, q, k, v, dout, position_ids=pid.cuda())
    ks, vs = chunks_to_seq(k), chunks_to_seq(v)
    want = [np.zeros(t.shape) for t in (q, ks, vs)]
    for b in range(2):
        starts = np.concatenate([[0], np.cumsum(lengths[b])])
        for s0, s1 in zip(starts[:-1], starts[1:]):
            sl = slice(int(s0), int(s1))
            g = oracle_mod.attention_backward(f64(q[b:b + 1, sl]), f64(ks[b:b + 1, sl]),
                                              f64(vs[b:b + 1, sl]), f64(dout[b:b + 1, sl]),
                                              w.scale, True)
            for out, part in zip(want, g):
                out[b, sl] = part[0]
    compare(w.name, (dq, chunks_to_seq(dk), chunks_to_seq(dv)), want)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "packed"])
def test_det_matches_default_mode(ra_lib, layout):
    """dK, dV: the default mode's bits (the same kernel computes them); dQ: the default
    mode's sum up to the order of its fp32 additions."""
    w, q, k, v, dout = problem(f"det_vs_default_{layout}", 1, 8, 2, 128, 4, 1024, True)
    kw = {}
    if layout == "zigzag":
        kw["layout"] = "zigzag"
    elif layout == "packed":
        kw["position_ids"] = synth.position_ids_from_lengths([[1000, 24, 2000, 1072]]).cuda()
    det = grads(ra_lib, w, q, k, v, dout, **kw)
    ra_lib.ra_set_bwd_deterministic(False)
    try:
        qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
        o, l = ra_lib.ring_attn_fwd(qc, kc, vc, True, w.scale, out_dtype=torch.bfloat16, **kw)
        fast = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, True, w.scale, **kw)
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    finally:
        ra_lib.ra_set_bwd_deterministic(True)
    assert_same_grads(fast, det, f"deterministic vs default, {layout}")


@pytest.mark.parametrize("causal", [True, False])
def test_det_accumulate_adds_the_plain_bits(ra_lib, causal):
    """ra_ring_attn_bwd_accumulate in the deterministic mode: the result is the fp32 sum of
    the buffers' prior values and the plain call's gradients, bit for bit."""
    w, q, k, v, dout = problem(f"det_acc_{causal}", 1, 4, 2, 128, 3, 300, causal)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, l = ra_lib.ring_attn_fwd(qc, kc, vc, causal, w.scale, out_dtype=torch.bfloat16)
    dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, causal, w.scale)
    g = torch.Generator(device="cuda").manual_seed(5)
    a_q = torch.randn(dq.shape, generator=g, device="cuda")
    a_k = torch.randn(dk.shape, generator=g, device="cuda")
    a_v = torch.randn(dv.shape, generator=g, device="cuda")
    want = (a_q + dq, a_k + dk, a_v + dv)
    got = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, causal, w.scale, dq=a_q.clone(),
                               dk=a_k.clone(), dv=a_v.clone(), accumulate=True)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    for nm, a, b in zip(("dq", "dk", "dv"), want, got):
        assert torch.equal(a, b), f"{nm}: accumulate differs from prior + plain"


def test_det_setter_returns_previous(ra_lib):
    assert ra_lib.ra_set_bwd_deterministic(True) is True
    assert ra_lib.ra_set_bwd_deterministic(False) is True
    assert ra_lib.ra_set_bwd_deterministic(True) is False


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "packed"])
def test_det_full_size_matches_default_mode(ra_lib, layout):
    """The bench's backward workload at full size (B = 1, L = 131072, H = 8, D = 128, causal;
    zigzag shards; 20 packed documents): the deterministic mode's dK, dV are the default
    mode's bits and its dQ the default mode's sum up to the order of its additions (the
    default mode is checked against the oracle at this size in test_bwd_full_gpu.py); two
    deterministic calls agree bit for bit."""
    W = synth.LONG_128K
    q, k, v = synth.attention_inputs(W, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(W.seed + 2)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    kw = {}
    if layout == "zigzag":
        kw["layout"] = "zigzag"
    elif layout == "packed":
        lens = synth.packed_lengths(W.L, W.seed + 21, 512, 32768)
        kw["position_ids"] = synth.position_ids_from_lengths([lens]).cuda()
    o, l = ra_lib.ring_attn_fwd(q, k, v, True, W.scale, out_dtype=torch.bfloat16, **kw)
    det = ra_lib.ring_attn_bwd(q, k, v, o, l, dout, True, W.scale, **kw)
    det2 = ra_lib.ring_attn_bwd(q, k, v, o, l, dout, True, W.scale, **kw)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    for nm, a, b in zip(("dq", "dk", "dv"), det, det2):
        assert torch.equal(a, b), f"{nm} differs between two deterministic calls"
    del det2
    ra_lib.ra_set_bwd_deterministic(False)
    try:
        fast = ra_lib.ring_attn_bwd(q, k, v, o, l, dout, True, W.scale, **kw)
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    finally:
        ra_lib.ra_set_bwd_deterministic(True)
    assert_same_grads(fast, det, f"full size, {layout}")
