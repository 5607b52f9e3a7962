"""GPU parity of ra_ring_attn_fwd against the fp64 oracle.

Small cases compare every row; the long-context workloads compare a seeded sample of
rows (plus every chunk's edge rows) against the full key range.  Tolerances: bf16 inputs
with fp32 accumulation, max-abs 1e-2 on O and 1e-3 on LSE; fp32 inputs, 1e-4 on both.

Sources: "Как работает sequence parallelism в контексте LLM?" sections 2, 3, 5 (chunked
ring with the log-sum-exp merge); "Метод контекстного параллелизма Ulysses" (the
seq->head transform feeding attention, and back)."""
import zlib

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import TOL, bf16_half_ulp, chunks_to_seq, f64, max_abs, rows_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _short_waits(ra_lib):
    old = ra_lib.ra_set_wait_limit_ns(2_000_000_000)
    yield
    ra_lib.ra_set_wait_limit_ns(old)


def run_gpu(ra_lib, w, q, k, v, out_dtype=torch.float32):
    o, l = ra_lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.causal, w.scale,
                                out_dtype=out_dtype)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    return o, l


def check_all_rows(ra_lib, oracle_mod, w):
    q, k, v = synth.attention_inputs(w)
    o, l = run_gpu(ra_lib, w, q, k, v)
    want_o, want_l = oracle_mod.ring_attention(f64(q), f64(k), f64(v), w.scale, w.causal)
    tol_o, tol_l = TOL[w.dtype]
    eo, el = max_abs(f64(o), want_o), max_abs(f64(l), want_l)
    print(f"[parity] {w.name}: max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= tol_o and el <= tol_l, (w.name, eo, el)
    return eo, el


def wl(name, **kw):
    base = dict(B=1, H_q=2, H_kv=2, D=128, P=1, Lc=128, dtype=torch.bfloat16, causal=False,
                seed=zlib.crc32(name.encode()) % 100000)
    base.update(kw)
    return synth.AttnWorkload(name, **base)


# ---------------------------------------------------------------- tensor-core path, small
@pytest.mark.parametrize("D", [128, 64])
def test_one_tile_noncausal(ra_lib, oracle_mod, D):
    check_all_rows(ra_lib, oracle_mod, wl(f"one_tile_{D}", D=D, Lc=256))


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_gqa_chunks(ra_lib, oracle_mod, D, causal):
    """Ragged chunk length (200: not a tile multiple), ragged total length (600: not a
    multiple of the 256-row CTA block), GQA 4:2, B = 2, P = 3."""
    check_all_rows(ra_lib, oracle_mod, wl(f"ragged_{D}_{causal}", B=2, H_q=4, H_kv=2, D=D, P=3,
                                          Lc=200, causal=causal))


@pytest.mark.parametrize("P,Lc,causal", [(1, 7, True), (5, 1, True), (5, 1, False),
                                         (1, 1, False), (16, 40, True), (2, 513, True)])
def test_degenerate_sizes(ra_lib, oracle_mod, P, Lc, causal):
    check_all_rows(ra_lib, oracle_mod, wl(f"degen_{P}_{Lc}_{causal}", H_q=4, H_kv=1, P=P, Lc=Lc,
                                          causal=causal))


def test_small_bf16_workload_every_row(ra_lib, oracle_mod):
    """B=1, H=8, D=64, 4 ranks x 1024 tokens, non-causal (the 4096-token workload)."""
    check_all_rows(ra_lib, oracle_mod, synth.SMALL_BF16)


def test_causal_every_row_multi_chunk(ra_lib, oracle_mod):
    check_all_rows(ra_lib, oracle_mod, wl("causal_multi", B=1, H_q=8, H_kv=2, D=128, P=4,
                                          Lc=1024, causal=True, q_mult=4.0))


def test_separate_chunk_allocations(ra_lib, oracle_mod):
    """Each virtual rank's K/V chunk in its own allocation (a host array of pointers)."""
    w = wl("separate", B=2, H_q=4, H_kv=2, D=128, P=3, Lc=300, causal=True)
    q, k, v = synth.attention_inputs(w)
    ks = [k[j].cuda().clone() for j in range(w.P)]
    vs = [v[j].cuda().clone() for j in range(w.P)]
    o, l = ra_lib.ring_attn_fwd(q.cuda(), ks, vs, True, w.scale)
    assert ra_lib.ra_sync_status() == 0
    want_o, want_l = oracle_mod.ring_attention(f64(q), f64(k), f64(v), w.scale, True)
    assert max_abs(f64(o), want_o) <= 1e-2 and max_abs(f64(l), want_l) <= 1e-3


def test_bf16_output(ra_lib, oracle_mod):
    """bf16 O: within the fp32 tolerance plus half a bf16 ulp of the oracle's value."""
    w = wl("bf16_out", B=1, H_q=4, H_kv=4, D=128, P=2, Lc=384, causal=True, q_mult=2.0)
    q, k, v = synth.attention_inputs(w)
    o, l = run_gpu(ra_lib, w, q, k, v, out_dtype=torch.bfloat16)
    assert o.dtype == torch.bfloat16
    want_o, want_l = oracle_mod.ring_attention(f64(q), f64(k), f64(v), w.scale, True)
    err = np.abs(f64(o) - want_o)
    assert np.all(err <= 1e-2 + bf16_half_ulp(want_o))
    assert max_abs(f64(l), want_l) <= 1e-3


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_padded_batch_strides(ra_lib, oracle_mod, dtype):
    """q_bstride and kv_bstride above the dense size: each batch of Q and of every K/V chunk
    is followed by padding rows filled with NaN, which must never be read."""
    w = wl(f"padded_{dtype}", B=2, H_q=4, H_kv=2, D=128, P=3, Lc=200, causal=True,
           dtype=dtype, q_mult=2.0)
    q, k, v = synth.attention_inputs(w)
    L, pad_q, pad_kv = w.L, 37, 19
    qp = torch.full((w.B, L + pad_q, w.H_q, w.D), float("nan"), dtype=dtype, device="cuda")
    qp[:, :L] = q.cuda()
    kp = torch.full((w.P, w.B, w.Lc + pad_kv, w.H_kv, w.D), float("nan"), dtype=dtype,
                    device="cuda")
    vp = kp.clone()
    kp[:, :, :w.Lc] = k.cuda()
    vp[:, :, :w.Lc] = v.cuda()
    out = torch.empty((w.B, L, w.H_q, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.H_q, L), dtype=torch.float32, device="cuda")
    in_dt = ra_lib.RA_BF16 if dtype == torch.bfloat16 else ra_lib.RA_FP32
    ra_lib.ra_ring_attn_fwd(qp.data_ptr(), [kp[j].data_ptr() for j in range(w.P)],
                            [vp[j].data_ptr() for j in range(w.P)], w.P, w.B, w.H_q, w.H_kv,
                            w.Lc, w.D, (L + pad_q) * w.H_q * w.D,
                            (w.Lc + pad_kv) * w.H_kv * w.D, w.scale, 1, in_dt, ra_lib.RA_FP32,
                            out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    want_o, want_l = oracle_mod.ring_attention(f64(q), f64(k), f64(v), w.scale, True)
    tol_o, tol_l = TOL[dtype]
    eo, el = max_abs(f64(out), want_o), max_abs(f64(lse), want_l)
    print(f"[parity] {w.name}: max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= tol_o and el <= tol_l


# ---------------------------------------------------------------- fp32 path
def test_tiny_fp32_workload_every_row(ra_lib, oracle_mod):
    """B=1, H=2, D=32, 2 ranks x 64 tokens, fp32, non-causal."""
    check_all_rows(ra_lib, oracle_mod, synth.TINY_FP32)


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fp32_ragged_gqa(ra_lib, oracle_mod, D, causal):
    check_all_rows(ra_lib, oracle_mod, wl(f"fp32_{D}_{causal}", B=2, H_q=4, H_kv=2, D=D, P=3,
                                          Lc=50, causal=causal, dtype=torch.float32, q_mult=2.0))


# ---------------------------------------------------------------- errors and the timeout path
def test_misaligned_device_pointer_rejected(ra_lib):
    q = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 256, 2, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 256, 2, 128, device="cuda")
    lse = torch.empty(1, 2, 256, device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ra_ring_attn_fwd(q.data_ptr() + 2, [k.data_ptr()], [k.data_ptr()], 1, 1, 2, 2, 256,
                                128, 256 * 2 * 128, 256 * 2 * 128, 0.1, 1, 0, 1, out.data_ptr(),
                                lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.status == 1


def test_bounded_wait_reports_timeout_and_context_survives(ra_lib, oracle_mod):
    """A withheld K tile makes the MMA thread's bounded wait expire: the kernel drains,
    frees its tensor memory and exits; ra_sync_status reports RA_ERR_TIMEOUT; the next
    launch on the same context is correct."""
    w = wl("stall", B=1, H_q=2, H_kv=2, D=128, P=2, Lc=256, causal=True)
    q, k, v = synth.attention_inputs(w)
    old = ra_lib.ra_set_wait_limit_ns(50_000_000)
    try:
        ra_lib.ra_debug_inject_stall(True)
        ra_lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, w.scale)
        assert ra_lib.ra_sync_status() == 4
        assert "bounded wait" in ra_lib.ra_last_error()
        assert ra_lib.ra_sync_status() == 0  # the error word was cleared
    finally:
        ra_lib.ra_set_wait_limit_ns(old)
    check_all_rows(ra_lib, oracle_mod, w)


# ---------------------------------------------------------------- long-context workloads
def check_sampled(ra_lib, oracle_mod, w, n_rows=2048):
    q, k, v = synth.attention_inputs(w)
    o, l = run_gpu(ra_lib, w, q, k, v)
    rows = synth.sample_rows(w.B, w.H_q, w.L, n_rows, seed=w.seed + 1, Lc=w.Lc)
    want_o, want_l = rows_oracle(oracle_mod, q, chunks_to_seq(k), chunks_to_seq(v), rows,
                                 w.scale, w.causal)
    rb, rt, rh = (torch.tensor(x) for x in rows)
    got_o = f64(o[rb, rt, rh])
    got_l = f64(l[rb, rh, rt])
    eo, el = max_abs(got_o, want_o), max_abs(got_l, want_l)
    print(f"[parity] {w.name} ({len(rows[0])} rows): max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= 1e-2 and el <= 1e-3, (w.name, eo, el)
    # every row of the full output is finite and normalised (|O| bounded by max |V|)
    assert torch.isfinite(o).all() and torch.isfinite(l).all()
    return eo, el


def test_llama8b_gqa_causal_32k_sampled(ra_lib, oracle_mod):
    """H_q=32, H_kv=8, D=128, 8 ranks x 4096 tokens, causal, Q x 4 (peaky softmax)."""
    check_sampled(ra_lib, oracle_mod, synth.LLAMA8B_GQA)


def test_long_context_128k_sampled(ra_lib, oracle_mod):
    """H=8, D=128, 16 ranks x 8192 tokens (L=131072), causal."""
    check_sampled(ra_lib, oracle_mod, synth.LONG_128K)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_ulysses_end_to_end_128k_sampled(ra_lib, oracle_mod, out_dtype):
    """seq2head(Q, K, V with the GQA copy) -> causal ring attention per head group ->
    head2seq(O), checked on sampled rows of the final sequence-sharded output against the
    oracle's own transforms and attention.  bf16 O is the benchmark's configuration (the
    attention writes bf16 O and head2seq moves those bits): each sampled element within
    the fp32 bar plus half a bf16 ulp of the oracle's value."""
    w = synth.ULYSSES_128K
    a = w.attn()
    q, k, v = synth.ulysses_inputs(w)
    qh = ra_lib.ra_ulysses_seq2head(q.cuda(), w.H_q)
    kh = ra_lib.ra_ulysses_seq2head(k.cuda(), w.H_kv_rep)
    vh = ra_lib.ra_ulysses_seq2head(v.cuda(), w.H_kv_rep)
    # head-sharded [P, B, L, Hl, D] -> attention batch = P*B ranks, K/V chunk j at token j*Lc
    qa = qh.view(a.B, a.L, a.H_q, a.D)
    kv_view = lambda x: x.view(a.B, a.P, a.Lc, a.H_kv, a.D).permute(1, 0, 2, 3, 4)
    o, l = ra_lib.ring_attn_fwd(qa, [kv_view(kh)[j] for j in range(a.P)],
                                [kv_view(vh)[j] for j in range(a.P)], True, a.scale,
                                out_dtype=out_dtype)
    o_seq = ra_lib.ra_ulysses_head2seq(o.view(w.P, w.B, a.L, a.H_q, a.D))
    assert o_seq.dtype == out_dtype
    assert ra_lib.ra_sync_status() == 0
    del qh, kh, vh, o

    # oracle side: its own transforms of the synthetic inputs
    bits = lambda t: t.contiguous().view(torch.int16).numpy()
    as_bf16 = lambda x: torch.from_numpy(x).view(torch.bfloat16)
    k_or = as_bf16(oracle_mod.seq2head(bits(k), w.H_kv_rep)).view(a.B, a.L, a.H_kv, a.D)
    v_or = as_bf16(oracle_mod.seq2head(bits(v), w.H_kv_rep)).view(a.B, a.L, a.H_kv, a.D)
    q_or = as_bf16(oracle_mod.seq2head(bits(q), w.H_q)).view(a.B, a.L, a.H_q, a.D)
    rows = synth.sample_rows(a.B, a.H_q, a.L, 2048, seed=w.seed + 1, Lc=a.Lc)
    want_o, want_l = rows_oracle(oracle_mod, q_or, k_or, v_or, rows, a.scale, True)
    # row (rank r, global token s*Lc+t, local head hh) lands at o_seq[s, b, t, r*Hl+hh]
    rb, rt, rh = (np.asarray(x) for x in rows)
    s, t = rt // w.Lc, rt % w.Lc
    r, b = rb // w.B, rb % w.B
    got = f64(o_seq[torch.tensor(s), torch.tensor(b), torch.tensor(t),
                    torch.tensor(r * a.H_q + rh)])
    got_l = f64(l[torch.tensor(rb), torch.tensor(rh), torch.tensor(rt)])
    eo, el = max_abs(got, want_o), max_abs(got_l, want_l)
    print(f"[parity] {w.name} e2e {out_dtype} ({len(rows[0])} rows): max|dO|={eo:.3e} "
          f"max|dLSE|={el:.3e}")
    slack = bf16_half_ulp(want_o) if out_dtype == torch.bfloat16 else 0.0
    assert np.all(np.abs(got - want_o) <= 1e-2 + slack), eo
    assert el <= 1e-3, el
