"""ra_ring_attn_bwd_static -- the backward pass with its Delta scratch in the library's fixed
device array, so that a call allocates no device memory -- against ra_ring_attn_bwd with a
caller-provided workspace.  Both run the same kernels, so two static calls in a row must
give the existing entry point's gradients (dK and dV bit for bit, dQ up to the order of its
fp32 reduce-adds across CTAs); the second call must leave the
device's free memory and torch's allocated and reserved memory unchanged; sizes beyond
RA_BWD_STATIC_MAX_ROWS are refused before anything is enqueued.  The pages have no counterpart to this entry point."""
import gc
import zlib

import pytest
import torch

from sequence_parallelism_attn_b200 import synth
from _util import assert_same_grads

MAX_ROWS = 1 << 21  # RA_BWD_STATIC_MAX_ROWS in include/ra.h


def _problem(name, B, H_q, H_kv, P, Lc, D=128):
    w = synth.AttnWorkload(name, B=B, H_q=H_q, H_kv=H_kv, D=D, P=P, Lc=Lc,
                           dtype=torch.bfloat16, causal=True, q_mult=2.0,
                           seed=zlib.crc32(name.encode()) % 100000)
    q, k, v = (t.cuda() for t in synth.attention_inputs(w))
    g = torch.Generator(device="cuda").manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    return w, q, k, v, dout


def _static_call(ra, w, q, k, v, o, lse, dout):
    """One ra_ring_attn_bwd_static call into fresh NaN-filled gradient buffers."""
    dq = torch.full((w.B, w.L, w.H_q, w.D), float("nan"), device="cuda")
    dk = torch.full(k.shape, float("nan"), device="cuda")
    dv = torch.full(k.shape, float("nan"), device="cuda")
    call = lambda: ra.ra_ring_attn_bwd_static(
        q.data_ptr(), [k[j].data_ptr() for j in range(w.P)],
        [v[j].data_ptr() for j in range(w.P)], o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
        w.P, w.B, w.H_q, w.H_kv, w.Lc, w.D, w.L * w.H_q * w.D, w.Lc * w.H_kv * w.D, w.scale,
        True, dq.data_ptr(), [dk[j].data_ptr() for j in range(w.P)],
        [dv[j].data_ptr() for j in range(w.P)], torch.cuda.current_stream().cuda_stream)
    return (dq, dk, dv), _memory_around(ra, call)


def _memory_around(ra, call):
    """Run one static call; return (device free memory, torch allocated, torch reserved)
    before and after it.  Python's cyclic garbage collector is run first and paused during
    the call, so that no tensor left over from earlier tests is freed inside the window."""
    gc.collect()
    gc.disable()
    try:
        torch.cuda.synchronize()
        before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
                  torch.cuda.memory_reserved())
        call()
        assert ra.ra_sync_status() == 0, ra.ra_last_error()
        after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
                 torch.cuda.memory_reserved())
    finally:
        gc.enable()
    return before, after


def _assert_no_allocation(ra, w, q, k, v, o, lse, dout, mem):
    """The call changed neither torch's allocated nor its reserved memory, nor the device's
    free memory.  Free memory counts every process on the device, so on a difference the
    measurement is taken once more before it counts against the library."""
    before, after = mem
    assert before[1:] == after[1:], (before, after)
    if before[0] != after[0]:
        _, (before, after) = _static_call(ra, w, q, k, v, o, lse, dout)
    assert before == after, (before, after)


def _two_calls_match(ra, name, B, H_q, H_kv, P, Lc):
    w, q, k, v, dout = _problem(name, B, H_q, H_kv, P, Lc)
    o, lse = ra.ring_attn_fwd(q, k, v, True, w.scale, out_dtype=torch.bfloat16)
    want = ra.ring_attn_bwd(q, k, v, o, lse, dout, True, w.scale)
    assert ra.ra_sync_status() == 0, ra.ra_last_error()
    first, _ = _static_call(ra, w, q, k, v, o, lse, dout)
    second, mem = _static_call(ra, w, q, k, v, o, lse, dout)
    assert_same_grads(want, first, f"{name}: first static call")
    assert_same_grads(want, second, f"{name}: second static call")
    _assert_no_allocation(ra, w, q, k, v, o, lse, dout, mem)


@pytest.mark.gpu
def test_static_two_calls_match_workspace_entry(ra_lib):
    """Ragged GQA problem: 3 chunks of 200 tokens, H_q = 4 over H_kv = 2, B = 2, causal."""
    _two_calls_match(ra_lib, "bwd_static_small", 2, 4, 2, 3, 200)


@pytest.mark.gpu
def test_static_at_the_size_limit(ra_lib):
    """B * H_q * P * Lc exactly RA_BWD_STATIC_MAX_ROWS (2 x 16 heads x 65536 tokens)."""
    assert 2 * 16 * 8 * 8192 == MAX_ROWS
    _two_calls_match(ra_lib, "bwd_static_limit", 2, 16, 4, 8, 8192)


@pytest.mark.gpu
def test_static_padded_batch_strides(ra_lib):
    """q and the K/V chunks as slices of larger NaN-filled buffers (batch strides above the
    dense size, B = 2): the static entry gives the dense workspace call's gradients."""
    from test_bwd_gpu import padded_call
    w, q, k, v, dout = _problem("bwd_static_padded", 2, 4, 2, 3, 200)
    o, lse = ra_lib.ring_attn_fwd(q, k, v, True, w.scale, out_dtype=torch.bfloat16)
    want = ra_lib.ring_attn_bwd(q, k, v, o, lse, dout, True, w.scale)
    got = padded_call(ra_lib, ra_lib.ra_ring_attn_bwd_static, w, q, k, v, o, lse, dout,
                      ws=False)
    assert_same_grads(want, got, "static padded strides")


def test_static_rejects_sizes_beyond_the_limit():
    """Refused on the host before any CUDA call (runs without a GPU); the pointers are
    never dereferenced."""
    from sequence_parallelism_attn_b200 import build, ra
    build.build()
    lib = ra.load()
    fake = 0x10000
    for B, H_q, P, Lc in ((1, 2, 2, 1 << 20), (2, 16, 8, 8193), (1 << 30, 1 << 30, 64, 1 << 24)):
        with pytest.raises(ra.RaError) as e:
            ra.ra_ring_attn_bwd_static(fake, [fake] * P, [fake] * P, fake, fake, fake, P, B, H_q,
                                       1, Lc, 128, 1 << 40, 1 << 40, 0.1, True, fake,
                                       [fake] * P, [fake] * P, 0)
        assert e.value.status == 1  # RA_ERR_INVALID
        assert "RA_BWD_STATIC_MAX_ROWS" in lib.ra_last_error().decode()
