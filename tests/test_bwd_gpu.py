"""GPU parity of ra_ring_attn_bwd (dQ, dK, dV of the tensor-core path) against the fp64
oracle's gradients, every element, at sizes up to L = 8192.

Tolerance: the gradients are products of bf16-rounded operands (P and dS are rounded to
bf16 before the tensor-core products, as Q, K, V, dO are), accumulated in fp32; each
rounding is within 2^-9 relative, so the error of a gradient element is a small multiple
of 2^-9 times the magnitudes it sums.  The bar is max|error| <= 1e-2 * max|reference| for
each gradient tensor (about five bf16 roundings at the largest element); measured errors
are 1.5e-3 .. 5.4e-3 of it.  An absolute floor of 1e-4 covers gradients that vanish analytically.

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
def _short_waits(ra_lib):
    old = ra_lib.ra_set_wait_limit_ns(2_000_000_000)
    yield
    ra_lib.ra_set_wait_limit_ns(old)


def check_grads(ra_lib, oracle_mod, name, B, H_q, H_kv, D, P, Lc, causal, q_mult=1.0):
    w = synth.AttnWorkload(name, B=B, H_q=H_q, H_kv=H_kv, D=D, P=P, Lc=Lc,
                           dtype=torch.bfloat16, causal=causal, q_mult=q_mult,
                           seed=zlib.crc32(name.encode()) % 100000)
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, l = ra_lib.ring_attn_fwd(qc, kc, vc, causal, w.scale, out_dtype=torch.bfloat16)
    dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, l, doc, causal, w.scale)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    rq, rk, rv = oracle_mod.attention_backward(f64(q), f64(chunks_to_seq(k)),
                                               f64(chunks_to_seq(v)), f64(dout), w.scale, causal)
    for nm, got, ref in (("dq", f64(dq), rq), ("dk", f64(chunks_to_seq(dk)), rk),
                         ("dv", f64(chunks_to_seq(dv)), rv)):
        check_grad(name, nm, got, ref)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
def test_bwd_single_chunk(ra_lib, oracle_mod, D, causal):
    check_grads(ra_lib, oracle_mod, f"bwd1_{D}_{causal}", 1, 2, 2, D, 1, 256, causal)


@pytest.mark.parametrize("D", [128, 64])
def test_bwd_ragged_gqa_chunks(ra_lib, oracle_mod, D):
    """P = 3 chunks of 200 tokens (not a tile multiple), GQA 4:2, B = 2, causal."""
    check_grads(ra_lib, oracle_mod, f"bwd_rag_{D}", 2, 4, 2, D, 3, 200, True, q_mult=2.0)


def test_bwd_peaky_multi_chunk(ra_lib, oracle_mod):
    check_grads(ra_lib, oracle_mod, "bwd_peaky", 1, 8, 2, 128, 4, 512, True, q_mult=4.0)


@pytest.mark.parametrize("P,Lc", [(1, 1), (5, 1), (2, 129), (16, 40)])
def test_bwd_degenerate_sizes(ra_lib, oracle_mod, P, Lc):
    check_grads(ra_lib, oracle_mod, f"bwd_degen_{P}_{Lc}", 1, 4, 1, 128, P, Lc, True)


def test_bwd_8k_gqa(ra_lib, oracle_mod):
    """L = 8192 (8 ranks x 1024), H_q = 8, H_kv = 2, causal: every gradient element."""
    check_grads(ra_lib, oracle_mod, "bwd_8k", 1, 8, 2, 128, 8, 1024, True)


def padded_call(ra_lib, entry, w, q, k, v, o, lse, dout, pad_q=37, pad_kv=19, ws=True):
    """Gradients through the raw entry point with q and every K/V chunk inside larger
    NaN-filled buffers (q_bstride, kv_bstride above the dense size; the padding rows must
    never be read).  out, lse, dout and the gradients are dense."""
    L = w.L
    qp = torch.full((w.B, L + pad_q, w.H_q, w.D), float("nan"), dtype=q.dtype, device="cuda")
    qp[:, :L] = q
    kp = torch.full((w.P, w.B, w.Lc + pad_kv, w.H_kv, w.D), float("nan"), dtype=k.dtype,
                    device="cuda")
    vp = kp.clone()
    kp[:, :, :w.Lc] = k
    vp[:, :, :w.Lc] = v
    dq = torch.full((w.B, L, w.H_q, w.D), float("nan"), device="cuda")
    dk = torch.full(k.shape, float("nan"), device="cuda")
    dv = torch.full(k.shape, float("nan"), device="cuda")
    args = [qp.data_ptr(), [kp[j].data_ptr() for j in range(w.P)],
            [vp[j].data_ptr() for j in range(w.P)], o.data_ptr(), lse.data_ptr(),
            dout.data_ptr(), w.P, w.B, w.H_q, w.H_kv, w.Lc, w.D, (L + pad_q) * w.H_q * w.D,
            (w.Lc + pad_kv) * w.H_kv * w.D, w.scale, True, dq.data_ptr(),
            [dk[j].data_ptr() for j in range(w.P)], [dv[j].data_ptr() for j in range(w.P)]]
    if ws:
        wsp = torch.empty((w.B, w.H_q, L), device="cuda")
        args.append(wsp.data_ptr())
    entry(*args, torch.cuda.current_stream().cuda_stream)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    return dq, dk, dv


def test_bwd_padded_batch_strides(ra_lib):
    """B = 2 with q and the K/V chunks as slices of larger buffers: the gradients equal the
    dense call's (dK, dV bit for bit, dQ up to the order of its reduce-adds)."""
    w = synth.AttnWorkload("bwd_padded", B=2, H_q=4, H_kv=2, D=128, P=3, Lc=200,
                           dtype=torch.bfloat16, causal=True, q_mult=2.0, seed=4711)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(4712),
                       device="cuda").to(torch.bfloat16)
    o, lse = ra_lib.ring_attn_fwd(q, k, v, True, w.scale, out_dtype=torch.bfloat16)
    want = ra_lib.ring_attn_bwd(q, k, v, o, lse, dout, True, w.scale)
    got = padded_call(ra_lib, ra_lib.ra_ring_attn_bwd, w, q, k, v, o, lse, dout)
    assert_same_grads(want, got, "padded strides")


def test_bwd_rejects_unsupported_head_dim(ra_lib):
    q = torch.zeros(1, 128, 2, 32, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 128, 2, 32, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 2, 128, device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ring_attn_bwd(q, k, k, q, lse, q, True)
    assert e.value.status == 2
