"""GPU parity of ra_ring_attn_fwd_packed (packed samples told apart by position_ids)
against the fp64 oracle: every row at small sizes (one-token samples, samples crossing
chunk and tile boundaries, a different packing per batch row), and sampled rows of a
131072-token sequence of seeded document lengths, each checked against the causal
attention over its own sample alone.

Source: "Paralelismo de secuencias en 🤗 accelerate", section "Configuración del backend
SP de ALST/Ulysses" (position_ids instead of an attention mask; several samples combined
into one sequence, attention staying inside each).  Tolerances as for the other paths."""
import zlib

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import TOL, chunks_to_seq, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _short_waits(ra_lib):
    old = ra_lib.ra_set_wait_limit_ns(2_000_000_000)
    yield
    ra_lib.ra_set_wait_limit_ns(old)


def wl(name, **kw):
    base = dict(B=2, H_q=4, H_kv=2, D=128, P=3, Lc=200, dtype=torch.bfloat16, causal=True,
                seed=zlib.crc32(name.encode()) % 100000, q_mult=2.0)
    base.update(kw)
    return synth.AttnWorkload(name, **base)


def run_packed(ra_lib, w, q, k, v, pid):
    o, l = ra_lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, w.scale,
                                position_ids=pid.cuda())
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    return o, l


def check_all_rows(ra_lib, oracle_mod, w, lengths):
    q, k, v = synth.attention_inputs(w)
    pid = synth.position_ids_from_lengths(lengths)
    o, l = run_packed(ra_lib, w, q, k, v, pid)
    want_o, want_l = oracle_mod.ring_attention_packed(f64(q), f64(k), f64(v), w.scale,
                                                      pid.numpy())
    tol_o, tol_l = TOL[w.dtype]
    eo, el = max_abs(f64(o), want_o), max_abs(f64(l), want_l)
    print(f"[parity] packed {w.name}: max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= tol_o and el <= tol_l, (w.name, eo, el)


@pytest.mark.parametrize("D", [128, 64])
def test_packed_bf16_mixed_lengths(ra_lib, oracle_mod, D):
    """600 tokens per row: row 0 mixes one-token and chunk-crossing samples, row 1 has
    samples ending exactly on 128-key tile edges."""
    check_all_rows(ra_lib, oracle_mod, wl(f"pk_{D}", D=D),
                   [[1, 1, 150, 77, 1, 300, 70], [128, 128, 256, 88]])


def test_packed_bf16_many_short_samples(ra_lib, oracle_mod):
    lens = [synth.packed_lengths(1024, 11 + b, 1, 40) for b in range(2)]
    check_all_rows(ra_lib, oracle_mod, wl("pk_short", P=4, Lc=256), lens)


def test_packed_bf16_one_token_samples(ra_lib, oracle_mod):
    check_all_rows(ra_lib, oracle_mod, wl("pk_ones", B=1, P=2, Lc=128), [[1] * 256])


@pytest.mark.parametrize("D", [32, 64, 128])
def test_packed_fp32(ra_lib, oracle_mod, D):
    check_all_rows(ra_lib, oracle_mod, wl(f"pk_fp32_{D}", D=D, Lc=50, dtype=torch.float32),
                   [[1, 30, 60, 9, 50], [150]])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_packed_single_sample_equals_causal(ra_lib, dtype):
    """One sample per row (position_ids = 0..L-1): bit for bit the causal contiguous result."""
    w = wl(f"pk_one_{dtype}", dtype=dtype)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    o1, l1 = ra_lib.ring_attn_fwd(q, k, v, True, w.scale)
    pid = synth.position_ids_from_lengths([[w.L]] * w.B).cuda()
    o2, l2 = ra_lib.ring_attn_fwd(q, k, v, True, w.scale, position_ids=pid)
    assert ra_lib.ra_sync_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_packed_null_ids_rejected(ra_lib):
    w = wl("pk_null")
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    out = torch.empty((w.B, w.L, w.H_q, w.D), device="cuda")
    lse = torch.empty((w.B, w.H_q, w.L), device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ra_ring_attn_fwd_packed(q.data_ptr(), [k[j].data_ptr() for j in range(w.P)],
                                       [v[j].data_ptr() for j in range(w.P)], None, w.P, w.B,
                                       w.H_q, w.H_kv, w.Lc, w.D, w.L * w.H_q * w.D,
                                       w.Lc * w.H_kv * w.D, w.scale, ra_lib.RA_BF16,
                                       ra_lib.RA_FP32, out.data_ptr(), lse.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert e.value.status == 1


def test_packed_long_context_128k_sampled(ra_lib, oracle_mod):
    """H=8, D=128, 16 ranks x 8192 tokens (L=131072), documents of 512..32768 tokens
    (log-uniform, seeded): sampled rows against causal attention over their own document."""
    w = synth.LONG_128K
    q, k, v = synth.attention_inputs(w)
    lens = synth.packed_lengths(w.L, w.seed + 21, 512, 32768)
    pid = synth.position_ids_from_lengths([lens])
    o, l = run_packed(ra_lib, w, q, k, v, pid)
    starts = np.concatenate([[0], np.cumsum(lens)])
    rb, rt, rh = synth.sample_rows(w.B, w.H_q, w.L, 2048, seed=w.seed + 9, Lc=w.Lc)
    rt = np.asarray(rt, np.int64)
    k_seq, v_seq = chunks_to_seq(k), chunks_to_seq(v)
    got_o = f64(o[torch.tensor(rb), torch.from_numpy(rt), torch.tensor(rh)])
    got_l = f64(l[torch.tensor(rb), torch.tensor(rh), torch.from_numpy(rt)])
    want_o, want_l = np.empty_like(got_o), np.empty_like(got_l)
    doc = np.searchsorted(starts, rt, side="right") - 1
    for d in np.unique(doc):
        sel = np.nonzero(doc == d)[0]
        s0, s1 = starts[d], starts[d + 1]
        rows_b = [rb[i] for i in sel]
        rows_h = [rh[i] for i in sel]
        qn = f64(q[torch.tensor(rows_b), torch.from_numpy(rt[sel]), torch.tensor(rows_h)])
        oo, ll = oracle_mod.attention_rows(qn, rows_b, rt[sel] - s0, rows_h,
                                           f64(k_seq[:, s0:s1]), f64(v_seq[:, s0:s1]), w.H_q,
                                           w.scale, True)
        want_o[sel], want_l[sel] = oo, ll
    eo, el = max_abs(got_o, want_o), max_abs(got_l, want_l)
    print(f"[parity] packed {w.name} ({len(lens)} documents, {len(rt)} rows): "
          f"max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= 1e-2 and el <= 1e-3
    assert torch.isfinite(o).all() and torch.isfinite(l).all()
