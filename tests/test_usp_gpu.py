"""GPU parity of the grouped Ulysses transforms (G head groups over P shards; bit-exact
against the oracle's index loops) and of the ring x Ulysses hybrid built from them: the
heads split over P_u groups by ra_ulysses_seq2head_grouped, each group's whole sequence
attended as P/P_u ring chunks by ra_ring_attn_fwd, and ra_ulysses_head2seq_grouped back.

Sources: "Метод контекстного параллелизма Ulysses" (the seq<->head all-to-all, the GQA
copy), "Paralelismo de secuencias en 🤗 accelerate" (USP named beside Ulysses),
"Как работает sequence parallelism в контексте LLM?" section 3 (the ring)."""
import math

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import f64, max_abs

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.int32).numpy().view(np.uint32)


@pytest.mark.parametrize("P,G,B,Lc,H_in,H_out,D,dtype", [
    (4, 2, 1, 1024, 8, 8, 128, torch.bfloat16),   # TMA path
    (6, 3, 2, 37, 6, 6, 64, torch.bfloat16),      # ragged tokens, B > 1
    (8, 2, 1, 300, 4, 4, 128, torch.bfloat16),    # GQA-sized head groups
    (4, 4, 1, 100, 2, 4, 128, torch.bfloat16),    # G = P with the KV copy
    (4, 2, 1, 64, 1, 2, 128, torch.bfloat16),     # one kv head copied to both groups
    (3, 1, 2, 50, 4, 4, 32, torch.float32),       # one group: concatenation of the shards
    (4, 2, 1, 8, 2, 2, 512, torch.float32),       # 2 KB heads: the vector path
    (2, 2, 3, 5, 2, 4, 8, torch.bfloat16),        # 16-byte heads: unvectorised path
])
def test_grouped_transforms_bit_exact(ra_lib, oracle_mod, P, G, B, Lc, H_in, H_out, D, dtype):
    g = torch.Generator().manual_seed(P * 100 + G * 10 + Lc)
    x = torch.randn(P, B, Lc, H_in, D, generator=g).to(dtype)
    y = ra_lib.ra_ulysses_seq2head(x.cuda(), H_out, groups=G)
    torch.cuda.synchronize()
    assert y.shape == (G, B, P * Lc, H_out // G, D)
    assert np.array_equal(_bits(y), oracle_mod.seq2head(_bits(x), H_out, groups=G))
    if H_in == H_out:
        z = ra_lib.ra_ulysses_head2seq(y, P=P)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(z), _bits(x))
    h = torch.randn(G, B, P * Lc, H_out // G, D, generator=g).to(dtype)
    z2 = ra_lib.ra_ulysses_head2seq(h.cuda(), P=P)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(z2), oracle_mod.head2seq(_bits(h), P=P))


def test_grouped_rejects_indivisible_heads(ra_lib):
    x = torch.zeros(4, 1, 8, 6, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ra_lib.RaError) as e:
        ra_lib.ra_ulysses_seq2head(x, 6, groups=4)  # 6 heads over 4 groups
    assert e.value.status == 1


def usp_forward(ra_lib, q, k, v, P_u, scale, causal):
    """q [P,B,Ls,H_q,D], k/v [P,B,Ls,H_kv,D] on the device -> (o [P,B,Ls,H_q,D] fp32,
    lse [B*P_u, H_q/P_u, L]) through the library's kernels only."""
    P, B, Ls, H_q, D = q.shape
    H_kv = k.shape[3]
    P_r, G = P // P_u, P_u
    H_rep = H_kv * G // math.gcd(H_kv, G)
    L = P * Ls
    qh = ra_lib.ra_ulysses_seq2head(q, H_q, groups=G)       # [G, B, L, H_q/G, D]
    kh = ra_lib.ra_ulysses_seq2head(k, H_rep, groups=G)
    vh = ra_lib.ra_ulysses_seq2head(v, H_rep, groups=G)
    Hq_l, Hkv_l, Lr = H_q // G, H_rep // G, L // P_r
    kc = [kh.view(G * B, P_r, Lr, Hkv_l, D)[:, j] for j in range(P_r)]
    vc = [vh.view(G * B, P_r, Lr, Hkv_l, D)[:, j] for j in range(P_r)]
    o, lse = ra_lib.ring_attn_fwd(qh.view(G * B, L, Hq_l, D), kc, vc, causal, scale,
                                  out_dtype=torch.float32)
    out = ra_lib.ra_ulysses_head2seq(o.view(G, B, L, Hq_l, D), P=P)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    return out, lse


@pytest.mark.parametrize("P,P_u,causal", [(4, 2, True), (4, 2, False), (6, 3, True),
                                          (8, 4, True), (4, 1, True), (4, 4, True)])
def test_usp_every_row(ra_lib, oracle_mod, P, P_u, causal):
    B, Ls, H_kv, D = 2, 96, 2, 128
    H_q = 6 if P_u == 3 else 8
    g = torch.Generator().manual_seed(P * 10 + P_u)
    q = (torch.randn(P, B, Ls, H_q, D, generator=g) * 2).to(torch.bfloat16)
    k = torch.randn(P, B, Ls, H_kv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(P, B, Ls, H_kv, D, generator=g).to(torch.bfloat16)
    scale = D ** -0.5
    out, lse = usp_forward(ra_lib, q.cuda(), k.cuda(), v.cuda(), P_u, scale, causal)
    want_o, want_l = oracle_mod.usp_attention(f64(q), f64(k), f64(v), P_u, scale, causal)
    G, L = P_u, P * Ls
    got_l = f64(lse).reshape(G, B, H_q // G, L).transpose(1, 0, 2, 3).reshape(B, H_q, L)
    eo, el = max_abs(f64(out), want_o), max_abs(got_l, want_l)
    print(f"[parity] usp P={P} P_u={P_u} causal={causal}: max|dO|={eo:.3e} max|dLSE|={el:.3e}")
    assert eo <= 1e-2 and el <= 1e-3


def test_usp_128k_sampled(ra_lib, oracle_mod):
    """The 128k-token Ulysses workload (Q [8 x 16384, 32, 128], K/V [8 x 16384, 4, 128],
    causal) as USP with 4 Ulysses groups x 2 ring chunks: sampled rows of the final
    sequence-sharded output against plain attention over the whole sequence."""
    w = synth.ULYSSES_128K
    q, k, v = synth.ulysses_inputs(w)
    G = 4
    out, lse = usp_forward(ra_lib, q.cuda(), k.cuda(), v.cuda(), G, w.attn().scale, True)
    seq = lambda x: x.permute(1, 0, 2, 3, 4).reshape(w.B, w.P * w.Lc, x.shape[3], w.D)
    rb, rt, rh = synth.sample_rows(w.B, w.H_q, w.P * w.Lc, 1024, seed=w.seed + 3, Lc=w.Lc)
    rt = np.asarray(rt, np.int64)
    qs = seq(q)
    qn = f64(qs[torch.tensor(rb), torch.from_numpy(rt), torch.tensor(rh)])
    want_o, want_l = oracle_mod.attention_rows(qn, rb, rt, rh, f64(seq(k)), f64(seq(v)),
                                               w.H_q, w.attn().scale, True)
    o_seq = seq(out.cpu())
    got_o = f64(o_seq[torch.tensor(rb), torch.from_numpy(rt), torch.tensor(rh)])
    # LSE rows of head group g = h // (H_q / G) sit at [g * B + b, h % (H_q / G), t]
    Hg = w.H_q // G
    rbn, rhn = np.asarray(rb), np.asarray(rh)
    got_l = f64(lse[torch.from_numpy((rhn // Hg) * w.B + rbn), torch.from_numpy(rhn % Hg),
                    torch.from_numpy(rt)])
    eo, el = max_abs(got_o, want_o), max_abs(got_l, want_l)
    print(f"[parity] usp 128k (4 groups x 2 ring chunks, {len(rt)} rows): max|dO|={eo:.3e} "
          f"max|dLSE|={el:.3e}")
    assert eo <= 1e-2 and el <= 1e-3, (eo, el)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
