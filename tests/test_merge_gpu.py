"""GPU parity of ra_lse_merge against the oracle's exact log-sum-exp merge
("Как работает sequence parallelism в контексте LLM?", section 5, merge step)."""
import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,L,D,frac", [
    (1, 8, 4096, 64, 0.0), (2, 4, 333, 128, 0.1), (1, 2, 128, 32, 0.3), (3, 3, 17, 4, 0.5),
    (1, 1, 5, 12, 0.0), (1, 32, 2048, 128, 0.05)])
def test_merge_matches_oracle(ra_lib, oracle_mod, B, H, L, D, frac):
    oa, la, ob, lb = synth.merge_inputs(B, H, L, D, seed=B * 100 + L, neg_inf_frac=frac)
    want_o, want_l = oracle_mod.lse_merge(f64(oa), f64(la), f64(ob), f64(lb))
    goa, gla, gob, glb = (t.cuda() for t in (oa, la, ob, lb))
    ra_lib.ra_lse_merge(goa, gla, gob, glb)
    torch.cuda.synchronize()
    got_o, got_l = f64(goa), f64(gla)
    both_empty = np.isneginf(want_l)
    assert np.array_equal(np.isneginf(got_l), both_empty)
    assert max_abs(got_l[~both_empty], want_l[~both_empty]) <= 1e-5
    assert max_abs(got_o, want_o) <= 1e-5
    # the inputs b are untouched
    assert torch.equal(gob.cpu(), ob) and torch.equal(glb.cpu(), lb)


def test_merge_of_two_chunk_partials_equals_whole(ra_lib, oracle_mod):
    """Attention over chunk 0 merged (on the GPU) with attention over chunk 1 equals
    attention over both chunks (oracle), the ring's merge step for P = 2."""
    w = synth.AttnWorkload("merge2", B=1, H_q=4, H_kv=4, D=64, P=2, Lc=256,
                           dtype=torch.bfloat16, causal=False, seed=77)
    q, k, v = synth.attention_inputs(w)
    parts = []
    for j in range(2):
        o, l = ra_lib.ring_attn_fwd(q[:, :].cuda().contiguous(), k[j:j + 1].repeat(2, 1, 1, 1, 1)
                                    .cuda(), v[j:j + 1].repeat(2, 1, 1, 1, 1).cuda(), False)
        parts.append((o, l))
    # each "partial" above attends to chunk j twice (P = 2 copies): lse is ln 2 too high,
    # the output is the single-chunk output.  Correct the lse before merging.
    oa, la = parts[0][0], parts[0][1] - float(np.log(2.0))
    ob, lb = parts[1][0], parts[1][1] - float(np.log(2.0))
    ra_lib.ra_lse_merge(oa, la, ob, lb)
    torch.cuda.synchronize()
    kk = torch.cat([k[0], k[1]], dim=1)
    vv = torch.cat([v[0], v[1]], dim=1)
    want_o, want_l = oracle_mod.attention(f64(q), f64(kk), f64(vv), w.scale, False)
    assert max_abs(f64(oa), want_o) <= 1e-2
    assert max_abs(f64(la), want_l) <= 1e-3


def test_merge_full_size_sampled(ra_lib, oracle_mod):
    """The benchmarked merge (B = 1, H = 8, L = 131072, D = 128, fp32; 10% empty partials):
    4096 seeded rows, plus the first and last row, against the oracle's merge of those
    rows; every output finite where a partial is."""
    B, H, L, D = 1, 8, 131072, 128
    oa, la, ob, lb = synth.merge_inputs(B, H, L, D, seed=1007, neg_inf_frac=0.1)
    goa, gla = oa.cuda(), la.cuda()
    ra_lib.ra_lse_merge(goa, gla, ob.cuda(), lb.cuda())
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(8)
    t = torch.cat([torch.randint(0, L, (4096,), generator=g), torch.tensor([0, L - 1])])
    h = torch.cat([torch.randint(0, H, (4096,), generator=g), torch.tensor([0, H - 1])])
    pick_o = lambda x: x[0, t, h].unsqueeze(0).unsqueeze(2)   # [1, n, 1, D]
    pick_l = lambda x: x[0, h, t].view(1, 1, -1)               # [1, 1, n]
    want_o, want_l = oracle_mod.lse_merge(f64(pick_o(oa)), f64(pick_l(la)), f64(pick_o(ob)),
                                          f64(pick_l(lb)))
    got_o, got_l = f64(pick_o(goa.cpu())), f64(pick_l(gla.cpu()))
    both_empty = np.isneginf(want_l)
    assert np.array_equal(np.isneginf(got_l), both_empty)
    assert max_abs(got_l[~both_empty], want_l[~both_empty]) <= 1e-5
    assert max_abs(got_o, want_o) <= 1e-5
    assert torch.isfinite(goa).all()
