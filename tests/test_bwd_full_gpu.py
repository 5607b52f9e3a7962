"""GPU parity of the backward pass at the benchmarked sizes: L = 131072 (16 ranks x 8192
tokens), H = 8, D = 128, causal, bf16 O from the forward (as the benchmark feeds it), in
each shard layout -- contiguous, zigzag and 20 packed documents of 512..32768 tokens -- and
the Llama-8B-shaped GQA workload (L = 32768, H_q = 32 over H_kv = 8).

Sampled rows against the fp64 oracle's gradients over the full visible key or query range
(oracle.attention_backward_rows): dQ of >= 2048 query rows (every chunk's and, for the
zigzag layout, every segment's first and last rows and the rows on 128-row tile edges;
packed: every document's first and last rows), and dK, dV of >= 512 key rows of one kv
head (with the same edges).  Bar as for the smaller backward tests: per gradient tensor,
max|error| <= 1e-2 * max|reference| over the sampled rows (plus 1e-4 for gradients that
vanish analytically).  Beside the bar the test reports the worst elementwise relative
error over the elements above 1e-2 * max|reference|, so that errors on small gradient
elements are visible.

Sources: the derivative of the forward of "Как работает sequence parallelism в контексте
LLM?" sections 2, 3, 5 (the pages train at these lengths: "Paralelismo de secuencias en 🤗
accelerate", section "¿Por qué la paralelización de secuencias?"); the zigzag layout named
in "Метод контекстного параллелизма Ulysses" (introduction); packed samples from the
accelerate guide, section "Configuración del backend SP de ALST/Ulysses"."""
import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import check_grad, chunks_to_seq, f64

pytestmark = pytest.mark.gpu

N_Q_ROWS = 2048
N_K_ROWS = 512


@pytest.fixture(scope="module", autouse=True)
def _short_waits(ra_lib):
    old = ra_lib.ra_set_wait_limit_ns(4_000_000_000)
    yield
    ra_lib.ra_set_wait_limit_ns(old)


def _edges(L, starts, tile=128):
    """First and last row of every segment that starts at `starts`, and the rows on both
    sides of the first 128-row tile edge inside it."""
    out = set()
    bounds = sorted(set(list(starts) + [L]))
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        out.update({s0, s1 - 1, min(s0 + tile - 1, s1 - 1), min(s0 + tile, s1 - 1)})
    return sorted(out)


def _rows(B, H, L, n, seed, edge_rows, head=None):
    """n seeded (b, t, h) rows plus the edge rows (random b, h); head fixes h."""
    g = torch.Generator().manual_seed(seed)
    t = torch.randint(0, L, (n,), generator=g).tolist() + list(edge_rows)
    m = len(t)
    b = torch.randint(0, B, (m,), generator=g).tolist()
    h = [head] * m if head is not None else torch.randint(0, H, (m,), generator=g).tolist()
    return np.asarray(b), np.asarray(t, np.int64), np.asarray(h)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag", "packed"])
def test_bwd_128k_sampled(ra_lib, oracle_mod, layout):
    w = synth.LONG_128K
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    kw, pos, lo, pid = {}, None, None, None
    if layout == "zigzag":
        kw = {"layout": "zigzag"}
        pos = oracle_mod.zigzag_positions(w.P, w.Lc)
        starts = range(0, w.L, w.Lc // 2)
    elif layout == "packed":
        lens = synth.packed_lengths(w.L, w.seed + 21, 512, 32768)
        pid = synth.position_ids_from_lengths([lens] * w.B)
        kw = {"position_ids": pid.cuda()}
        lo = oracle_mod.packed_lower_bounds(pid.numpy())
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).tolist()
    else:
        starts = range(0, w.L, w.Lc)

    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = ra_lib.ring_attn_fwd(qc, kc, vc, True, w.scale, out_dtype=torch.bfloat16, **kw)
    dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, lse, doc, True, w.scale, **kw)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    dq, dk, dv = dq.cpu(), chunks_to_seq(dk.cpu()), chunks_to_seq(dv.cpu())
    del qc, kc, vc, doc, o, lse

    edges = _edges(w.L, starts)
    qr = _rows(w.B, w.H_q, w.L, N_Q_ROWS, w.seed + 31, edges)
    kv_head = int(torch.randint(0, w.H_kv, (1,), generator=torch.Generator().manual_seed(
        w.seed + 32)).item())
    kr = _rows(w.B, w.H_kv, w.L, N_K_ROWS, w.seed + 33, edges, head=kv_head)
    assert len(qr[0]) >= N_Q_ROWS and len(kr[0]) >= N_K_ROWS
    rq, rk, rv = oracle_mod.attention_backward_rows(
        f64(q), f64(chunks_to_seq(k)), f64(chunks_to_seq(v)), f64(dout), w.scale, True, qr, kr,
        positions=pos, lower_bounds=lo)
    tq = lambda x, r: f64(x[torch.from_numpy(r[0]), torch.from_numpy(r[1]),
                            torch.from_numpy(r[2])])
    check_grad(f"full {layout}", "dq", tq(dq, qr), rq)
    check_grad(f"full {layout}", "dk", tq(dk, kr), rk)
    check_grad(f"full {layout}", "dv", tq(dv, kr), rv)


def test_bwd_32k_gqa_sampled(ra_lib, oracle_mod):
    """The backward of the Llama-8B-shaped GQA workload at its benchmarked size (B = 1,
    L = 32768 as 8 ranks x 4096 tokens, H_q = 32 over H_kv = 8, D = 128, causal, Q x 4):
    sampled dQ rows of every head and dK, dV rows of one kv head, each summing the four
    query heads of its group, against the oracle over the full visible range."""
    w = synth.LLAMA8B_GQA
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = ra_lib.ring_attn_fwd(qc, kc, vc, True, w.scale, out_dtype=torch.bfloat16)
    dq, dk, dv = ra_lib.ring_attn_bwd(qc, kc, vc, o, lse, doc, True, w.scale)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    dq, dk, dv = dq.cpu(), chunks_to_seq(dk.cpu()), chunks_to_seq(dv.cpu())
    del qc, kc, vc, doc, o, lse
    edges = _edges(w.L, range(0, w.L, w.Lc))
    qr = _rows(w.B, w.H_q, w.L, N_Q_ROWS, w.seed + 41, edges)
    kr = _rows(w.B, w.H_kv, w.L, N_K_ROWS, w.seed + 43, edges, head=w.H_kv - 1)
    rq, rk, rv = oracle_mod.attention_backward_rows(
        f64(q), f64(chunks_to_seq(k)), f64(chunks_to_seq(v)), f64(dout), w.scale, True, qr, kr)
    tq = lambda x, r: f64(x[torch.from_numpy(r[0]), torch.from_numpy(r[1]),
                            torch.from_numpy(r[2])])
    check_grad("full 32k GQA", "dq", tq(dq, qr), rq)
    check_grad("full 32k GQA", "dk", tq(dk, kr), rk)
    check_grad("full 32k GQA", "dv", tq(dv, kr), rv)
