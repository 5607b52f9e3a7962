"""Guard canaries: every output of the library is a view inside a larger buffer whose
guard regions before and after it hold a sentinel bit pattern; after the call the guards
must be unchanged (no write outside an output), and the outputs must differ from the
sentinel wherever the call defines them.  Ragged sizes (chunks and sequences that are not
tile multiples, B > 1, GQA) so that every kernel's edge handling writes near the guards."""
import math

import pytest
import torch

from sequence_parallelism_attn_b200 import synth

pytestmark = pytest.mark.gpu

PAD = 4096  # elements of guard on each side


def guarded(shape, dtype):
    n = math.prod(shape)
    buf = torch.empty(n + 2 * PAD, dtype=dtype, device="cuda")
    bits = buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32)
    bits.fill_(0x7FA5 if dtype == torch.bfloat16 else 0x7FC0DEAD)  # a NaN payload
    return buf, buf[PAD:PAD + n].view(shape)


def intact(buf, n):
    bits = buf.view(torch.int16 if buf.dtype == torch.bfloat16 else torch.int32)
    want = 0x7FA5 if buf.dtype == torch.bfloat16 else 0x7FC0DEAD
    torch.cuda.synchronize()
    return bool((bits[:PAD] == want).all()) and bool((bits[PAD + n:] == want).all())


def written(view):
    return bool(torch.isfinite(view.float()).all())


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 32)])
def test_forward_writes_only_its_outputs(ra_lib, dtype, D):
    w = synth.AttnWorkload("canary_fwd", B=2, H_q=4, H_kv=2, D=D, P=3, Lc=200, dtype=dtype,
                           causal=True, seed=5)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    ob, o = guarded((w.B, w.L, w.H_q, w.D), torch.float32)
    lb, l = guarded((w.B, w.H_q, w.L), torch.float32)
    ra_lib.ring_attn_fwd(q, k, v, True, w.scale, out=o, lse=l)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    assert intact(ob, o.numel()) and intact(lb, l.numel())
    assert written(o) and written(l)


@pytest.mark.parametrize("packed", [False, True])
def test_backward_writes_only_its_outputs(ra_lib, packed):
    w = synth.AttnWorkload("canary_bwd", B=2, H_q=4, H_kv=2, D=128, P=3, Lc=200,
                           dtype=torch.bfloat16, causal=True, seed=6)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    dout = torch.randn(q.shape, device="cuda").to(torch.bfloat16)
    pid = (synth.position_ids_from_lengths([[150, 1, 449], [600]]).cuda() if packed else None)
    o, l = ra_lib.ring_attn_fwd(q, k, v, True, w.scale, out_dtype=torch.bfloat16,
                                position_ids=pid)
    bufs = [guarded(q.shape, torch.float32), guarded(k.shape, torch.float32),
            guarded(k.shape, torch.float32), guarded((w.B, w.H_q, w.L), torch.float32)]
    (qb, dq), (kb, dk), (vb, dv), (wb, ws) = bufs
    ra_lib.ring_attn_bwd(q, k, v, o, l, dout, True, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                         position_ids=pid)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    for buf, view in bufs:
        assert intact(buf, view.numel())
    assert written(dq) and written(dk) and written(dv) and written(ws)


@pytest.mark.parametrize("P,Lc,H_in,H_out,D,dtype", [
    (4, 37, 2, 4, 128, torch.bfloat16),    # TMA path, ragged tokens, GQA copy
    (4, 8, 2, 4, 512, torch.float32),      # vector path (2 KB heads)
])
def test_permutes_write_only_their_outputs(ra_lib, P, Lc, H_in, H_out, D, dtype):
    x = torch.randn(P, 2, Lc, H_in, D, device="cuda").to(dtype)
    hb, h = guarded((P, 2, P * Lc, H_out // P, D), dtype)
    ra_lib.ra_ulysses_seq2head(x, H_out, out=h)
    torch.cuda.synchronize()
    assert intact(hb, h.numel()) and written(h)
    sb, s = guarded((P, 2, Lc, H_out, D), dtype)
    ra_lib.ra_ulysses_head2seq(h, out=s)
    torch.cuda.synchronize()
    assert intact(sb, s.numel()) and written(s)
    assert ra_lib.ra_sync_status() == 0


def test_merge_writes_only_its_outputs(ra_lib):
    oa, la, ob, lb = synth.merge_inputs(2, 3, 77, 64, seed=9, neg_inf_frac=0.0)
    obuf, o = guarded(oa.shape, torch.float32)
    lbuf, l = guarded(la.shape, torch.float32)
    o.copy_(oa.cuda())
    l.copy_(la.cuda())
    ra_lib.ra_lse_merge(o, l, ob.cuda(), lb.cuda())
    torch.cuda.synchronize()
    assert intact(obuf, o.numel()) and intact(lbuf, l.numel())
    assert written(o) and written(l)
