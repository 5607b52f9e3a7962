"""The differentiable entry points (sequence_parallelism_attn_b200.autograd): loss.backward()
through ring attention on one GPU (contiguous, zigzag and packed-sample forms) and through
the distributed ring, zigzag ring and USP on a one-rank NCCL group gives the oracle's
gradients of the same loss (the gradient bar of the backward tests).

Sources: "Как работает sequence parallelism в контексте LLM?" (training with ring
attention), "Метод контекстного параллелизма Ulysses"."""
import socket

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import autograd as rag
from sequence_parallelism_attn_b200 import synth
from _util import check_grad, chunks_to_seq, f64

pytestmark = pytest.mark.gpu


def _leaf(x):
    return x.cuda().requires_grad_(True)


@pytest.mark.parametrize("layout,causal", [("contiguous", True), ("contiguous", False),
                                           ("zigzag", True), ("packed", True)])
def test_ring_attention_backward_through_autograd(ra_lib, oracle_mod, layout, causal):
    B, P, Lc, H_q, H_kv, D = 2, 3, 200, 4, 2, 128
    w = synth.AttnWorkload(f"autograd_{layout}", B=B, H_q=H_q, H_kv=H_kv, D=D, P=P, Lc=Lc,
                           dtype=torch.bfloat16, causal=causal, q_mult=2.0, seed=811)
    q, k, v = synth.attention_inputs(w)
    g = torch.Generator().manual_seed(812)
    wt = torch.randn(q.shape, generator=g).to(torch.bfloat16)  # dLoss/dO
    kw = {}
    pid = None
    if layout == "zigzag":
        kw["layout"] = "zigzag"
    if layout == "packed":
        lens = [[120, 330, 150], [600]]
        pid = synth.position_ids_from_lengths(lens)
        kw["position_ids"] = pid.cuda()
    ql, kl, vl = _leaf(q), _leaf(k), _leaf(v)
    o = rag.ring_attention(ql, kl, vl, causal, w.scale, **kw)
    assert o.dtype == torch.bfloat16 and o.shape == q.shape
    (o.float() * wt.cuda().float()).sum().backward()
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    # the oracle's gradients of the same loss, in natural sequence order
    kseq, vseq = chunks_to_seq(k), chunks_to_seq(v)
    qn, kn, vn, dn = f64(q), f64(kseq), f64(vseq), f64(wt)
    if layout == "zigzag":
        pos = oracle_mod.zigzag_positions(P, Lc)   # shard order -> sequence positions
        inv = np.argsort(pos)
        rq, rk, rv = oracle_mod.attention_backward(qn[:, inv], kn[:, inv], vn[:, inv],
                                                   dn[:, inv], w.scale, True)
        rq, rk, rv = rq[:, pos], rk[:, pos], rv[:, pos]
    elif layout == "packed":
        rq, rk, rv = np.zeros_like(qn), np.zeros_like(kn), np.zeros_like(vn)
        for bi, ls in enumerate(lens):
            s0 = 0
            for n in ls:
                sl = slice(s0, s0 + n)
                a, b_, c = oracle_mod.attention_backward(qn[bi:bi + 1, sl], kn[bi:bi + 1, sl],
                                                         vn[bi:bi + 1, sl], dn[bi:bi + 1, sl],
                                                         w.scale, True)
                rq[bi, sl], rk[bi, sl], rv[bi, sl] = a[0], b_[0], c[0]
                s0 += n
    else:
        rq, rk, rv = oracle_mod.attention_backward(qn, kn, vn, dn, w.scale, causal)
    name = f"autograd ring_attention {layout} causal={causal}"
    check_grad(name, "dq", f64(ql.grad), rq)
    check_grad(name, "dk", f64(chunks_to_seq(kl.grad)), rk)
    check_grad(name, "dv", f64(chunks_to_seq(vl.grad)), rv)


def test_distributed_backward_through_autograd(ra_lib, oracle_mod):
    """ring_attention_dist (plain and zigzag) and usp_attention_dist on a one-rank NCCL
    group: loss.backward() gives the oracle's gradients."""
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        B, Lc, H_q, H_kv, D = 1, 300, 4, 2, 128
        g = torch.Generator().manual_seed(813)
        q = torch.randn(B, Lc, H_q, D, generator=g).to(torch.bfloat16)
        k = torch.randn(B, Lc, H_kv, D, generator=g).to(torch.bfloat16)
        v = torch.randn(B, Lc, H_kv, D, generator=g).to(torch.bfloat16)
        wt = torch.randn(B, Lc, H_q, D, generator=g).to(torch.bfloat16)
        rq, rk, rv = oracle_mod.attention_backward(f64(q), f64(k), f64(v), f64(wt), D ** -0.5,
                                                   True)
        for name, fn in (("ring", lambda a, b_, c: rag.ring_attention_dist(a, b_, c, True)),
                         ("zigzag ring", lambda a, b_, c: rag.ring_attention_dist(
                             a, b_, c, True, zigzag=True)),
                         ("USP", lambda a, b_, c: rag.usp_attention_dist(a, b_, c, True))):
            ql, kl, vl = _leaf(q), _leaf(k), _leaf(v)
            o = fn(ql, kl, vl)
            (o.float() * wt.cuda().float()).sum().backward()
            assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
            check_grad(f"autograd {name}, one rank", "dq", f64(ql.grad), rq)
            check_grad(f"autograd {name}, one rank", "dk", f64(kl.grad), rk)
            check_grad(f"autograd {name}, one rank", "dv", f64(vl.grad), rv)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


def test_ring_attention_deterministic_training_step(ra_lib):
    """With ra_set_bwd_deterministic(1), two identical loss.backward() passes through
    ring_attention give the same gradient bits (dq included)."""
    w = synth.AttnWorkload("autograd_det", B=1, H_q=8, H_kv=2, D=128, P=4, Lc=512,
                           dtype=torch.bfloat16, causal=True, seed=813)
    q, k, v = synth.attention_inputs(w)
    wt = torch.randn(q.shape, generator=torch.Generator().manual_seed(814)).to(torch.bfloat16)
    old = ra_lib.ra_set_bwd_deterministic(True)
    try:
        grads = []
        for _ in range(2):
            ql, kl, vl = _leaf(q), _leaf(k), _leaf(v)
            o = rag.ring_attention(ql, kl, vl, True, w.scale)
            (o.float() * wt.cuda().float()).sum().backward()
            assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
            grads.append((ql.grad, kl.grad, vl.grad))
    finally:
        ra_lib.ra_set_bwd_deterministic(old)
    for nm, a, b in zip(("dq", "dk", "dv"), grads[0], grads[1]):
        assert torch.equal(a, b), f"{nm} differs between two deterministic passes"
