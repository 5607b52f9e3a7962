"""ctypes binding of libra_b200.so (the C ABI of include/ra.h), entry point for entry point.

Argument marshalling only: torch tensors are turned into device pointers, sizes and
the current CUDA stream; every step of the computation runs in the library's CUDA
kernels.  Loading fails loudly if the library has not been built -- there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libra_b200.so")

RA_OK, RA_ERR_INVALID, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_TIMEOUT = 0, 1, 2, 3, 4
RA_BF16, RA_FP32 = 0, 1
RA_MAX_P = 64
EXPORTED = ("ra_ring_attn_fwd", "ra_ring_attn_fwd_zigzag", "ra_ring_attn_fwd_packed",
            "ra_ring_attn_bwd", "ra_ring_attn_bwd_zigzag", "ra_ring_attn_bwd_packed",
            "ra_ring_attn_bwd_static", "ra_ring_attn_bwd_accumulate",
            "ra_lse_merge", "ra_ulysses_seq2head", "ra_ulysses_head2seq",
            "ra_ulysses_seq2head_grouped", "ra_ulysses_head2seq_grouped",
            "ra_ulysses_seq2head_scatter", "ra_ulysses_head2seq_scatter",
            "ra_ulysses_replica_sum", "ra_sync_status", "ra_last_error", "ra_set_wait_limit_ns",
            "ra_set_bwd_deterministic", "ra_debug_inject_stall", "ra_version")


class RaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"ra status {status}: {message}")
        self.status = status


_lib = None


def load() -> ctypes.CDLL:
    """Load libra_b200.so (built by sequence_parallelism_attn_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m sequence_parallelism_attn_b200.build` (no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    lib.ra_ring_attn_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i64, f32, i32,
                                     i32, i32, vp, vp, vp]
    lib.ra_ring_attn_fwd_zigzag.argtypes = lib.ra_ring_attn_fwd.argtypes
    lib.ra_ring_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64,
                                     i64, f32, i32, vp, vp, vp, vp, vp]
    lib.ra_ring_attn_bwd_static.argtypes = lib.ra_ring_attn_bwd.argtypes[:19] + [vp]
    lib.ra_ring_attn_bwd_zigzag.argtypes = lib.ra_ring_attn_bwd.argtypes
    lib.ra_ring_attn_bwd_accumulate.argtypes = lib.ra_ring_attn_bwd.argtypes
    lib.ra_ring_attn_bwd_packed.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                            i32, i64, i64, f32, vp, vp, vp, vp, vp]
    lib.ra_ring_attn_fwd_packed.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i64,
                                            f32, i32, i32, vp, vp, vp]
    lib.ra_lse_merge.argtypes = [vp, vp, vp, vp, i32, i32, i64, i32, vp]
    lib.ra_ulysses_seq2head.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_ulysses_head2seq.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_ulysses_seq2head_grouped.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_ulysses_head2seq_grouped.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_ulysses_replica_sum.argtypes = [vp, vp, i64, i32, i32, i32, vp]
    lib.ra_ulysses_seq2head_scatter.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_ulysses_head2seq_scatter.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.ra_sync_status.argtypes = [vp]
    for f in ("ra_ring_attn_fwd", "ra_ring_attn_fwd_zigzag", "ra_ring_attn_fwd_packed",
              "ra_ring_attn_bwd", "ra_ring_attn_bwd_zigzag", "ra_ring_attn_bwd_packed",
              "ra_ring_attn_bwd_static", "ra_ring_attn_bwd_accumulate", "ra_lse_merge",
              "ra_ulysses_seq2head", "ra_ulysses_head2seq", "ra_ulysses_seq2head_grouped",
              "ra_ulysses_head2seq_grouped", "ra_ulysses_replica_sum", "ra_sync_status",
              "ra_ulysses_seq2head_scatter", "ra_ulysses_head2seq_scatter"):
        getattr(lib, f).restype = ctypes.c_int
    lib.ra_last_error.restype = ctypes.c_char_p
    lib.ra_version.restype = ctypes.c_char_p
    lib.ra_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.ra_set_wait_limit_ns.restype = ctypes.c_ulonglong
    lib.ra_set_bwd_deterministic.argtypes = [i32]
    lib.ra_set_bwd_deterministic.restype = i32
    lib.ra_debug_inject_stall.argtypes = [i32]
    lib.ra_debug_inject_stall.restype = None
    _lib = lib
    return lib


def _check(status: int):
    if status != RA_OK:
        raise RaError(status, load().ra_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dt(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return RA_BF16
    if t == torch.float32:
        return RA_FP32
    raise ValueError(f"unsupported dtype {t}")


def version() -> str:
    return load().ra_version().decode()


# ------------------------------------------------------------------ raw entry points
def ra_ring_attn_fwd(q_ptr, k_ptrs, v_ptrs, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride, scale,
                     causal, in_dtype, out_dtype, out_ptr, lse_ptr, stream):
    """The C entry point with raw pointers (k_ptrs/v_ptrs: sequences of P device pointers)."""
    arr = ctypes.c_void_p * P
    ks, vs = arr(*k_ptrs), arr(*v_ptrs)
    _check(load().ra_ring_attn_fwd(q_ptr, ks, vs, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride,
                                   scale, int(causal), in_dtype, out_dtype, out_ptr, lse_ptr,
                                   stream))


def ra_ring_attn_fwd_zigzag(q_ptr, k_ptrs, v_ptrs, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride,
                            scale, causal, in_dtype, out_dtype, out_ptr, lse_ptr, stream):
    """The zigzag-layout C entry point with raw pointers (arguments as ra_ring_attn_fwd)."""
    arr = ctypes.c_void_p * P
    ks, vs = arr(*k_ptrs), arr(*v_ptrs)
    _check(load().ra_ring_attn_fwd_zigzag(q_ptr, ks, vs, P, B, H_q, H_kv, Lc, D, q_bstride,
                                          kv_bstride, scale, int(causal), in_dtype, out_dtype,
                                          out_ptr, lse_ptr, stream))


def ra_ring_attn_fwd_packed(q_ptr, k_ptrs, v_ptrs, pid_ptr, P, B, H_q, H_kv, Lc, D, q_bstride,
                            kv_bstride, scale, in_dtype, out_dtype, out_ptr, lse_ptr, stream):
    """The packed-samples C entry point with raw pointers (position_ids: int32 [B][P*Lc])."""
    arr = ctypes.c_void_p * P
    ks, vs = arr(*k_ptrs), arr(*v_ptrs)
    _check(load().ra_ring_attn_fwd_packed(q_ptr, ks, vs, pid_ptr, P, B, H_q, H_kv, Lc, D,
                                          q_bstride, kv_bstride, scale, in_dtype, out_dtype,
                                          out_ptr, lse_ptr, stream))


def ra_ring_attn_bwd(q_ptr, k_ptrs, v_ptrs, out_ptr, lse_ptr, dout_ptr, P, B, H_q, H_kv, Lc, D,
                     q_bstride, kv_bstride, scale, causal, dq_ptr, dk_ptrs, dv_ptrs, ws_ptr,
                     stream):
    """The backward C entry point with raw pointers (chunk pointer lists of length P)."""
    arr = ctypes.c_void_p * P
    _check(load().ra_ring_attn_bwd(q_ptr, arr(*k_ptrs), arr(*v_ptrs), out_ptr, lse_ptr, dout_ptr,
                                   P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride, scale,
                                   int(causal), dq_ptr, arr(*dk_ptrs), arr(*dv_ptrs), ws_ptr,
                                   stream))


def ra_ring_attn_bwd_zigzag(q_ptr, k_ptrs, v_ptrs, out_ptr, lse_ptr, dout_ptr, P, B, H_q, H_kv, Lc,
                            D, q_bstride, kv_bstride, scale, causal, dq_ptr, dk_ptrs, dv_ptrs,
                            ws_ptr, stream):
    """The backward C entry point for zigzag shards (raw pointers)."""
    arr = ctypes.c_void_p * P
    _check(load().ra_ring_attn_bwd_zigzag(q_ptr, arr(*k_ptrs), arr(*v_ptrs), out_ptr, lse_ptr,
                                          dout_ptr, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride,
                                          scale, int(causal), dq_ptr, arr(*dk_ptrs),
                                          arr(*dv_ptrs), ws_ptr, stream))


def ra_ring_attn_bwd_accumulate(q_ptr, k_ptrs, v_ptrs, out_ptr, lse_ptr, dout_ptr, P, B, H_q,
                                H_kv, Lc, D, q_bstride, kv_bstride, scale, causal, dq_ptr, dk_ptrs,
                                dv_ptrs, ws_ptr, stream):
    """The backward C entry point that adds into dq / dk / dv (raw pointers)."""
    arr = ctypes.c_void_p * P
    _check(load().ra_ring_attn_bwd_accumulate(q_ptr, arr(*k_ptrs), arr(*v_ptrs), out_ptr,
                                              lse_ptr, dout_ptr, P, B, H_q, H_kv, Lc, D,
                                              q_bstride, kv_bstride, scale, int(causal), dq_ptr,
                                              arr(*dk_ptrs), arr(*dv_ptrs), ws_ptr, stream))


def ra_ring_attn_bwd_packed(q_ptr, k_ptrs, v_ptrs, pid_ptr, out_ptr, lse_ptr, dout_ptr, P, B, H_q,
                            H_kv, Lc, D, q_bstride, kv_bstride, scale, dq_ptr, dk_ptrs, dv_ptrs,
                            ws_ptr, stream):
    """The backward C entry point for packed samples (raw pointers; causal)."""
    arr = ctypes.c_void_p * P
    _check(load().ra_ring_attn_bwd_packed(q_ptr, arr(*k_ptrs), arr(*v_ptrs), pid_ptr, out_ptr,
                                          lse_ptr, dout_ptr, P, B, H_q, H_kv, Lc, D, q_bstride,
                                          kv_bstride, scale, dq_ptr, arr(*dk_ptrs),
                                          arr(*dv_ptrs), ws_ptr, stream))


def ra_ring_attn_bwd_static(q_ptr, k_ptrs, v_ptrs, out_ptr, lse_ptr, dout_ptr, P, B, H_q, H_kv,
                            Lc, D, q_bstride, kv_bstride, scale, causal, dq_ptr, dk_ptrs, dv_ptrs,
                            stream):
    """The backward C entry point whose Delta scratch is the library's own fixed device
    array (no workspace pointer; B*H_q*P*Lc <= RA_BWD_STATIC_MAX_ROWS)."""
    arr = ctypes.c_void_p * P
    _check(load().ra_ring_attn_bwd_static(q_ptr, arr(*k_ptrs), arr(*v_ptrs), out_ptr, lse_ptr,
                                          dout_ptr, P, B, H_q, H_kv, Lc, D, q_bstride,
                                          kv_bstride, scale, int(causal), dq_ptr, arr(*dk_ptrs),
                                          arr(*dv_ptrs), stream))


def ring_attn_bwd(q: torch.Tensor, k_chunks: torch.Tensor, v_chunks: torch.Tensor,
                  out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor, causal: bool,
                  scale: float | None = None, dq: torch.Tensor | None = None,
                  dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, stream=None,
                  layout: str = "contiguous", position_ids: torch.Tensor | None = None,
                  accumulate: bool = False):
    """Gradients of ring_attn_fwd: q/out/dout [B, P*Lc, H_q, D] bf16 (dense), k/v chunks
    [P, B, Lc, H_kv, D] bf16, lse [B, H_q, P*Lc] fp32.  Returns (dq [B, P*Lc, H_q, D],
    dk, dv [P, B, Lc, H_kv, D]) in fp32; the fp32 workspace [B, H_q, P*Lc] is allocated
    here when not given (the library itself allocates nothing).  layout and position_ids
    as for ring_attn_fwd (the forward's).  accumulate: add into the given dq / dk / dv
    (ra_ring_attn_bwd_accumulate; contiguous layout)."""
    if layout not in ("contiguous", "zigzag"):
        raise ValueError(f"unknown layout {layout!r}")
    if position_ids is not None and (layout != "contiguous" or not causal):
        raise ValueError("packed samples need the contiguous layout and causal=True")
    if accumulate and (dq is None or dk is None or dv is None or layout != "contiguous"
                       or position_ids is not None):
        raise ValueError("accumulate needs dq, dk and dv to add into, and the contiguous layout")
    P, B, Lc, H_kv, D = k_chunks.shape
    _, L, H_q, _ = q.shape
    assert L == P * Lc and q.is_contiguous() and out.is_contiguous() and dout.is_contiguous()
    assert k_chunks.is_contiguous() and v_chunks.is_contiguous()
    if scale is None:
        scale = D ** -0.5
    dev = q.device
    if dq is None:
        dq = torch.empty((B, L, H_q, D), dtype=torch.float32, device=dev)
    if dk is None:
        dk = torch.empty((P, B, Lc, H_kv, D), dtype=torch.float32, device=dev)
    if dv is None:
        dv = torch.empty_like(dk)
    if workspace is None:
        workspace = torch.empty((B, H_q, L), dtype=torch.float32, device=dev)
    kp, vp_ = [k_chunks[j].data_ptr() for j in range(P)], [v_chunks[j].data_ptr() for j in range(P)]
    dkp, dvp = [dk[j].data_ptr() for j in range(P)], [dv[j].data_ptr() for j in range(P)]
    if position_ids is not None:
        assert position_ids.dtype == torch.int32 and position_ids.is_cuda
        assert position_ids.is_contiguous() and position_ids.shape == (B, L)
        ra_ring_attn_bwd_packed(q.data_ptr(), kp, vp_, position_ids.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), dout.data_ptr(), P, B, H_q, H_kv, Lc, D,
                                L * H_q * D, Lc * H_kv * D, float(scale), dq.data_ptr(), dkp, dvp,
                                workspace.data_ptr(), _stream(stream))
    else:
        entry = ra_ring_attn_bwd_zigzag if layout == "zigzag" else ra_ring_attn_bwd
        if accumulate:
            entry = ra_ring_attn_bwd_accumulate
        entry(q.data_ptr(), kp, vp_, out.data_ptr(), lse.data_ptr(), dout.data_ptr(), P, B, H_q,
              H_kv, Lc, D, L * H_q * D, Lc * H_kv * D, float(scale), causal, dq.data_ptr(), dkp,
              dvp, workspace.data_ptr(), _stream(stream))
    return dq, dk, dv


def ra_lse_merge(o_a: torch.Tensor, lse_a: torch.Tensor, o_b: torch.Tensor, lse_b: torch.Tensor,
                 stream=None):
    """In-place merge into (o_a, lse_a).  o [B,L,H,D] fp32, lse [B,H,L] fp32."""
    B, L, H, D = o_a.shape
    for t in (o_a, lse_a, o_b, lse_b):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    assert o_b.shape == o_a.shape and lse_a.shape == lse_b.shape == (B, H, L)
    _check(load().ra_lse_merge(o_a.data_ptr(), lse_a.data_ptr(), o_b.data_ptr(), lse_b.data_ptr(),
                               B, H, L, D, _stream(stream)))


def ra_ulysses_replica_sum(x: torch.Tensor, H_out: int, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """The gradient of the GQA copy: x [..., H_in, D] fp32 (H_in = H_out * rep) ->
    [..., H_out, D], each head the sum of its rep replicas."""
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    *lead, H_in, D = x.shape
    rows = 1
    for n in lead:
        rows *= n
    if out is None:
        out = torch.empty((*lead, H_out, D), dtype=torch.float32, device=x.device)
    assert out.is_contiguous() and out.dtype == torch.float32 and out.shape == (*lead, H_out, D)
    _check(load().ra_ulysses_replica_sum(x.data_ptr(), out.data_ptr(), rows, H_in, H_out, D,
                                         _stream(stream)))
    return out


def ra_ulysses_seq2head(x: torch.Tensor, H_out: int | None = None, out: torch.Tensor | None = None,
                        stream=None, groups: int | None = None) -> torch.Tensor:
    """[P,B,Lc,H_in,D] -> [G,B,P*Lc,H_out/G,D] (H_out defaults to H_in, G = groups to P)."""
    assert x.is_cuda and x.is_contiguous() and x.dim() == 5
    P, B, Lc, H_in, D = x.shape
    H_out = H_in if H_out is None else H_out
    G = P if groups is None else groups
    if out is None:
        out = torch.empty((G, B, P * Lc, max(H_out // G, 1), D), dtype=x.dtype, device=x.device)
    if G == P:
        _check(load().ra_ulysses_seq2head(x.data_ptr(), out.data_ptr(), P, B, Lc, H_in, H_out, D,
                                          _dt(x.dtype), _stream(stream)))
    else:
        _check(load().ra_ulysses_seq2head_grouped(x.data_ptr(), out.data_ptr(), P, G, B, Lc, H_in,
                                                  H_out, D, _dt(x.dtype), _stream(stream)))
    return out


def ra_ulysses_head2seq(x: torch.Tensor, out: torch.Tensor | None = None,
                        stream=None, P: int | None = None) -> torch.Tensor:
    """[G,B,P*Lc,H/G,D] -> [P,B,Lc,H,D] (P shards, default G)."""
    assert x.is_cuda and x.is_contiguous() and x.dim() == 5
    G, B, L, Hl, D = x.shape
    P = G if P is None else P
    Lc = L // P
    if out is None:
        out = torch.empty((P, B, Lc, Hl * G, D), dtype=x.dtype, device=x.device)
    if G == P:
        _check(load().ra_ulysses_head2seq(x.data_ptr(), out.data_ptr(), P, B, Lc, Hl * P, D,
                                          _dt(x.dtype), _stream(stream)))
    else:
        _check(load().ra_ulysses_head2seq_grouped(x.data_ptr(), out.data_ptr(), P, G, B, Lc,
                                                  Hl * G, D, _dt(x.dtype), _stream(stream)))
    return out


def ra_ulysses_seq2head_scatter(x: torch.Tensor, dst_ptrs, rank: int, H_out: int | None = None,
                                stream=None) -> None:
    """This rank's share of the Ulysses seq->head all-to-all, stored straight into the P
    destination buffers: x [B, Lc, H_in, D] (this rank's sequence shard), dst_ptrs = P device
    addresses (ints) of the ranks' [B, P*Lc, H_out/P, D] buffers (peer or local memory)."""
    assert x.is_cuda and x.is_contiguous() and x.dim() == 4
    B, Lc, H_in, D = x.shape
    P = len(dst_ptrs)
    H_out = H_in if H_out is None else H_out
    arr = (ctypes.c_void_p * P)(*dst_ptrs)
    _check(load().ra_ulysses_seq2head_scatter(x.data_ptr(), arr, P, rank, B, Lc, H_in, H_out, D,
                                              _dt(x.dtype), _stream(stream)))


def ra_ulysses_head2seq_scatter(y: torch.Tensor, dst_ptrs, rank: int, stream=None) -> None:
    """This rank's share of the Ulysses head->seq all-to-all: y [B, P*Lc, H/P, D] (this rank's
    head group over the whole sequence), dst_ptrs = P device addresses (ints) of the ranks'
    [B, Lc, H, D] buffers."""
    assert y.is_cuda and y.is_contiguous() and y.dim() == 4
    B, L, Hl, D = y.shape
    P = len(dst_ptrs)
    arr = (ctypes.c_void_p * P)(*dst_ptrs)
    _check(load().ra_ulysses_head2seq_scatter(y.data_ptr(), arr, P, rank, B, L // P, Hl * P, D,
                                              _dt(y.dtype), _stream(stream)))


def ra_sync_status(stream=None) -> int:
    """Synchronise the stream and return the kernel status (RA_OK or RA_ERR_TIMEOUT)."""
    return load().ra_sync_status(_stream(stream))


def ra_last_error() -> str:
    return load().ra_last_error().decode()


def ra_set_wait_limit_ns(ns: int) -> int:
    return load().ra_set_wait_limit_ns(ns)


def ra_set_bwd_deterministic(on: bool) -> bool:
    """Bitwise-reproducible backward (dq from the query-stationary kernel) on or off for
    every later backward call of the process; returns the previous setting."""
    return bool(load().ra_set_bwd_deterministic(1 if on else 0))


def ra_debug_inject_stall(on: bool):
    load().ra_debug_inject_stall(1 if on else 0)


# ------------------------------------------------------------------ tensor-level helper
def ring_attn_fwd(q: torch.Tensor, k_chunks, v_chunks, causal: bool, scale: float | None = None,
                  out_dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None,
                  lse: torch.Tensor | None = None, stream=None, layout: str = "contiguous",
                  position_ids: torch.Tensor | None = None):
    """Ring-chunked attention of q [B, P*Lc, H_q, D] against P K/V chunks.

    k_chunks / v_chunks: a tensor [P, B, Lc, H_kv, D] (chunk j = k_chunks[j]) or a list
    of P tensors [B, Lc, H_kv, D], each batch-contiguous with the same batch stride.
    layout: "contiguous" (rank i holds tokens i*Lc .. i*Lc+Lc-1) or "zigzag" (rank i holds
    segments i and 2P-1-i of 2P segments of Lc/2 tokens; see ra_ring_attn_fwd_zigzag).
    position_ids: int32 [B, P*Lc] on the device (packed samples, causal and contiguous
    only; see ra_ring_attn_fwd_packed).
    Returns (out [B, P*Lc, H_q, D] in out_dtype, lse [B, H_q, P*Lc] fp32).
    """
    if layout not in ("contiguous", "zigzag"):
        raise ValueError(f"unknown layout {layout!r}")
    entry = ra_ring_attn_fwd_zigzag if layout == "zigzag" else ra_ring_attn_fwd
    if position_ids is not None:
        if layout != "contiguous" or not causal:
            raise ValueError("packed samples need the contiguous layout and causal=True")
        assert position_ids.dtype == torch.int32 and position_ids.is_cuda
        assert position_ids.is_contiguous() and position_ids.shape == (q.shape[0], q.shape[1])
        pid_ptr = position_ids.data_ptr()

        def entry(q_ptr, k_ptrs, v_ptrs, P, B, H_q, H_kv, Lc, D, qs, kvs, sc, causal_, *rest):
            ra_ring_attn_fwd_packed(q_ptr, k_ptrs, v_ptrs, pid_ptr, P, B, H_q, H_kv, Lc, D, qs,
                                    kvs, sc, *rest)
    if isinstance(k_chunks, torch.Tensor):
        k_list = [k_chunks[j] for j in range(k_chunks.shape[0])]
        v_list = [v_chunks[j] for j in range(v_chunks.shape[0])]
    else:
        k_list, v_list = list(k_chunks), list(v_chunks)
    P = len(k_list)
    B, L, H_q, D = q.shape
    _, Lc, H_kv, _ = k_list[0].shape
    assert L == P * Lc, "q length must equal P * Lc"
    assert q.stride(3) == 1 and q.stride(2) == D and q.stride(1) == H_q * D
    kv_bstride = k_list[0].stride(0)
    for t in k_list + v_list:
        assert t.shape == (B, Lc, H_kv, D) and t.dtype == q.dtype and t.is_cuda
        assert t.stride(3) == 1 and t.stride(2) == D and t.stride(1) == H_kv * D
        assert B == 1 or t.stride(0) == kv_bstride
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, L, H_q, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q, L), dtype=torch.float32, device=q.device)
    entry(q.data_ptr(), [t.data_ptr() for t in k_list], [t.data_ptr() for t in v_list],
          P, B, H_q, H_kv, Lc, D, q.stride(0) if B > 1 else L * H_q * D,
          kv_bstride if B > 1 else Lc * H_kv * D, float(scale), int(bool(causal)),
          _dt(q.dtype), _dt(out.dtype), out.data_ptr(), lse.data_ptr(), _stream(stream))
    return out, lse
