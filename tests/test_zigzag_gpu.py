"""GPU parity of ra_ring_attn_fwd_zigzag (shards in the zigzag layout) against the fp64
oracle: every row at small sizes, where zigzag tiles straddle the shard's two segments
(Lc/2 not a multiple of 128) or hold a single token (Lc = 2); a seeded row sample at
L = 131072.  Tolerances as for the contiguous layout (bf16: 1e-2 on O, 1e-3 on LSE;
fp32: 1e-4).

Source: the zigzag layout is named beside the plain ring in "Метод контекстного
параллелизма Ulysses" (introduction); the layout taken is the load-balanced one (2P
segments of Lc/2 tokens, rank i holding segments i and 2P-1-i), as the oracle states."""
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
    base = dict(B=1, H_q=2, H_kv=2, D=128, P=2, Lc=256, dtype=torch.bfloat16, causal=True,
                seed=zlib.crc32(name.encode()) % 100000)
    base.update(kw)
    return synth.AttnWorkload(name, **base)


def check_all_rows(ra_lib, oracle_mod, w):
    q, k, v = synth.attention_inputs(w)
    o, l = ra_lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.causal, w.scale,
                                layout="zigzag")
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    want_o, want_l = oracle_mod.ring_attention_zigzag(f64(q), f64(k), f64(v), w.scale, w.causal)
    tol_o, tol_l = TOL[w.dtype]
    eo, el = max_abs(f64(o), want_o), max_abs(f64(l), want_l)
    print(f"[parity] zigzag {w.name}: max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= tol_o and el <= tol_l, (w.name, eo, el)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("P,Lc", [(2, 256), (4, 200), (3, 384), (5, 2), (1, 300), (8, 128)])
def test_zigzag_bf16_every_row(ra_lib, oracle_mod, D, P, Lc):
    check_all_rows(ra_lib, oracle_mod, wl(f"zz_{D}_{P}_{Lc}", B=2, H_q=4, H_kv=2, D=D, P=P,
                                          Lc=Lc, q_mult=2.0))


def test_zigzag_peaky_multi_chunk(ra_lib, oracle_mod):
    check_all_rows(ra_lib, oracle_mod, wl("zz_peaky", B=1, H_q=8, H_kv=2, D=128, P=4, Lc=1024,
                                          q_mult=4.0))


@pytest.mark.parametrize("D", [32, 64, 128])
def test_zigzag_fp32_every_row(ra_lib, oracle_mod, D):
    check_all_rows(ra_lib, oracle_mod, wl(f"zz_fp32_{D}", B=2, H_q=4, H_kv=2, D=D, P=3, Lc=50,
                                          dtype=torch.float32, q_mult=2.0))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_zigzag_noncausal_equals_contiguous(ra_lib, dtype):
    """Without a causal mask positions play no role: both layouts give identical bits."""
    w = wl(f"zz_nc_{dtype}", B=2, H_q=4, H_kv=2, D=128, P=3, Lc=200, causal=False, dtype=dtype)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    o1, l1 = ra_lib.ring_attn_fwd(q, k, v, False, w.scale)
    o2, l2 = ra_lib.ring_attn_fwd(q, k, v, False, w.scale, layout="zigzag")
    assert ra_lib.ra_sync_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_zigzag_odd_chunk_rejected(ra_lib):
    w = wl("zz_odd", P=2, Lc=129)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ring_attn_fwd(q, k, v, True, w.scale, layout="zigzag")
    assert e.value.status == 1


def test_zigzag_long_context_128k_sampled(ra_lib, oracle_mod):
    """H=8, D=128, 16 ranks x 8192 tokens (L=131072), causal, shards in the zigzag layout:
    sampled rank-major rows against the oracle over the sequence in natural order."""
    w = synth.LONG_128K
    q, k, v = synth.attention_inputs(w)
    o, l = ra_lib.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, w.scale, layout="zigzag")
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    pos = oracle_mod.zigzag_positions(w.P, w.Lc)
    nat = np.empty(w.L, np.int64)
    nat[pos] = np.arange(w.L)
    k_nat = chunks_to_seq(k)[:, torch.from_numpy(nat)]
    v_nat = chunks_to_seq(v)[:, torch.from_numpy(nat)]
    rb, rt, rh = synth.sample_rows(w.B, w.H_q, w.L, 2048, seed=w.seed + 7, Lc=w.Lc // 2)
    rt = np.asarray(rt, np.int64)
    qn = f64(q[torch.tensor(rb), torch.from_numpy(rt), torch.tensor(rh)])
    want_o, want_l = oracle_mod.attention_rows(qn, rb, pos[rt], rh, f64(k_nat), f64(v_nat),
                                               w.H_q, w.scale, True)
    got_o = f64(o[torch.tensor(rb), torch.from_numpy(rt), torch.tensor(rh)])
    got_l = f64(l[torch.tensor(rb), torch.tensor(rh), torch.from_numpy(rt)])
    eo, el = max_abs(got_o, want_o), max_abs(got_l, want_l)
    print(f"[parity] zigzag {w.name} ({len(rt)} rows): max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= 1e-2 and el <= 1e-3
    assert torch.isfinite(o).all() and torch.isfinite(l).all()
