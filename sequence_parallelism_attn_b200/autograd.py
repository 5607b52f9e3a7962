"""Differentiable entry points: torch.autograd.Function wrappers that pair each forward of
the library with its backward, so that ring attention, its zigzag and packed-sample forms,
and the distributed ring and Ulysses / USP paths can sit inside a training step
("Как работает sequence parallelism в контексте LLM?" trains with ring attention; the
accelerate guide's Ulysses / ALST backend does the same with the all-to-all form).

Every computation is a library call (ra.ring_attn_fwd / ra.ring_attn_bwd and the dist
functions); this module only saves what the backward needs and meets autograd's rules on
dtypes: the forward returns O in the inputs' dtype (bf16), keeping the fp32 LSE for the
backward, and the fp32 gradients are returned in the inputs' dtypes.
"""
from __future__ import annotations

import torch

from . import ra


class _RingAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k_chunks, v_chunks, causal, scale, layout, position_ids):
        o, lse = ra.ring_attn_fwd(q, k_chunks, v_chunks, causal, scale, out_dtype=q.dtype,
                                  layout=layout, position_ids=position_ids)
        ctx.save_for_backward(q, k_chunks, v_chunks, o, lse, position_ids)
        ctx.causal, ctx.scale, ctx.layout = causal, scale, layout
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, pid = ctx.saved_tensors
        dq, dk, dv = ra.ring_attn_bwd(q, k, v, o, lse, do.to(q.dtype).contiguous(), ctx.causal,
                                      ctx.scale, layout=ctx.layout, position_ids=pid)
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None


def ring_attention(q: torch.Tensor, k_chunks: torch.Tensor, v_chunks: torch.Tensor,
                   causal: bool = True, scale: float | None = None, layout: str = "contiguous",
                   position_ids: torch.Tensor | None = None) -> torch.Tensor:
    """Ring-chunked attention on one GPU with autograd: q [B, P*Lc, H_q, D] bf16 (dense),
    k_chunks / v_chunks [P, B, Lc, H_kv, D] bf16 (dense) -> O [B, P*Lc, H_q, D] bf16.
    layout and position_ids as for ra.ring_attn_fwd.  backward() gives dq, dk, dv (computed
    in fp32 by ra.ring_attn_bwd, returned in bf16)."""
    if q.dtype != torch.bfloat16:
        raise ValueError("the differentiable path takes bf16 inputs (the tensor-core backward)")
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return _RingAttention.apply(q.contiguous(), k_chunks.contiguous(), v_chunks.contiguous(),
                                bool(causal), float(scale), layout, position_ids)


class _RingAttentionDist(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group, zigzag):
        from . import dist as rd
        if zigzag:
            o, lse = rd.ring_attn_fwd_zigzag_dist(q, k, v, scale, group=group)
        else:
            o, lse = rd.ring_attn_fwd_dist(q, k, v, causal, scale, group=group)
        o = o.to(q.dtype)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.group, ctx.zigzag = causal, scale, group, zigzag
        return o

    @staticmethod
    def backward(ctx, do):
        from . import dist as rd
        q, k, v, o, lse = ctx.saved_tensors
        do = do.to(q.dtype).contiguous()
        if ctx.zigzag:
            dq, dk, dv = rd.ring_attn_bwd_zigzag_dist(q, k, v, o, lse, do, ctx.scale,
                                                      group=ctx.group)
        else:
            dq, dk, dv = rd.ring_attn_bwd_dist(q, k, v, o, lse, do, ctx.causal, ctx.scale,
                                               group=ctx.group)
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None


def ring_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                        scale: float | None = None, group=None,
                        zigzag: bool = False) -> torch.Tensor:
    """Ring attention across the ranks of `group` with autograd: q [B, Lc, H_q, D] and k/v
    [B, Lc, H_kv, D] (bf16, dense) are this rank's chunk (the zigzag layout's shard when
    zigzag, which is causal) -> this rank's O [B, Lc, H_q, D] bf16.  backward() runs the ring
    backward (the K/V chunks travel again with their dK, dV accumulators)."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return _RingAttentionDist.apply(q.contiguous(), k.contiguous(), v.contiguous(), bool(causal),
                                    float(scale), group, bool(zigzag))


class _USPAttentionDist(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, ulysses_group, ring_group):
        from . import dist as rd
        o, lse = rd.usp_attn_fwd_dist(q, k, v, causal, scale, ulysses_group=ulysses_group,
                                      ring_group=ring_group)
        o = o.to(q.dtype)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.groups = causal, scale, (ulysses_group, ring_group)
        return o

    @staticmethod
    def backward(ctx, do):
        from . import dist as rd
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = rd.usp_attn_bwd_dist(q, k, v, o, lse, do.to(q.dtype).contiguous(),
                                          ctx.causal, ctx.scale, ulysses_group=ctx.groups[0],
                                          ring_group=ctx.groups[1])
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None


def usp_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                       scale: float | None = None, ulysses_group=None,
                       ring_group=None) -> torch.Tensor:
    """The ring x Ulysses hybrid (plain Ulysses with a one-rank ring group) with autograd:
    q [B, Ls, H_q, D] and k/v [B, Ls, H_kv, D] (bf16, dense) are this rank's sequence shard
    with every head -> its O [B, Ls, H_q, D] bf16 (see dist.usp_attn_fwd_dist for the
    groups).  backward() runs dist.usp_attn_bwd_dist."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return _USPAttentionDist.apply(q.contiguous(), k.contiguous(), v.contiguous(), bool(causal),
                                   float(scale), ulysses_group, ring_group)
