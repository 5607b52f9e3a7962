"""fp64 CPU oracle for ring-chunked attention, the log-sum-exp merge and the
Ulysses layout transforms.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The oracle shares no code
with the CUDA library (``sequence_parallelism_attn_b200``) and neither imports
the other.  The arithmetic lives in ``ra_oracle.cpp`` (plain loops, fp64); this
module only builds it and marshals numpy arrays.

Sources: "Как работает sequence parallelism в контексте LLM?" sections 2, 3, 5
(chunking, the ring, the per-chunk softmax and its merge) and "Метод
контекстного параллелизма Ulysses" (the seq<->head all-to-all and the GQA copy).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ra_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libra_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ra_oracle.cpp into libra_oracle.so (plain g++, IEEE fp64, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
           "-o", tmp, _SRC]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    lib.ora_attention.argtypes = [P, P, P, i32, i64, i32, i32, i32, f64, i32, P, P, i32]
    lib.ora_attention_rows.argtypes = [P, P, P, P, i64, P, P, i32, i64, i32, i32, i32, f64, i32,
                                       P, P, i32]
    lib.ora_ring_attention.argtypes = [P, P, P, i32, i32, i64, i32, i32, i32, f64, i32, P, P, P, P, P,
                                       i32]
    lib.ora_lse_merge.argtypes = [P, P, P, P, i32, i32, i64, i32]
    lib.ora_seq2head.argtypes = [P, P, i32, i32, i32, i64, i32, i32, i32, i32]
    lib.ora_head2seq.argtypes = [P, P, i32, i32, i32, i64, i32, i32, i32]
    lib.ora_zigzag_positions.argtypes = [i32, i64, P]
    lib.ora_attention_backward.argtypes = [P, P, P, P, i32, i64, i32, i32, i32, f64, i32, P, P,
                                           P, i32]
    lib.ora_packed_lower_bounds.argtypes = [P, i32, i64, P]
    lib.ora_attention_backward_rows.argtypes = [P, P, P, P, i32, i64, i32, i32, i32, f64, i32, P,
                                                P, i64, P, P, P, i64, P, P, P, P, P, P, i32]
    lib.ora_attention_backward_pair.argtypes = [P, P, P, P, P, P, i32, i64, i64, i32, i32, i32,
                                                f64, i32, P, P, P, i32]
    lib.ora_replica_sum.argtypes = [P, P, i64, i32, i32, i32]
    for f in ("ora_attention", "ora_attention_rows", "ora_ring_attention", "ora_lse_merge",
              "ora_seq2head", "ora_head2seq", "ora_zigzag_positions", "ora_packed_lower_bounds",
              "ora_attention_backward", "ora_attention_backward_rows",
              "ora_attention_backward_pair", "ora_replica_sum"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


def attention(q, k, v, scale: float, causal: bool, nthreads: int = 0):
    """Plain attention.  q [B,L,H_q,D], k/v [B,L,H_kv,D] -> (out [B,L,H_q,D], lse [B,H_q,L])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, H_q, D = q.shape
    H_kv = k.shape[2]
    assert k.shape == (B, L, H_kv, D) and v.shape == k.shape
    out = np.empty((B, L, H_q, D), np.float64)
    lse = np.empty((B, H_q, L), np.float64)
    rc = _load().ora_attention(_ptr(q), _ptr(k), _ptr(v), B, L, H_q, H_kv, D, float(scale),
                               int(bool(causal)), _ptr(out), _ptr(lse), nthreads)
    _check(rc, "attention")
    return out, lse


def attention_backward(q, k, v, dout, scale: float, causal: bool, nthreads: int = 0):
    """Gradients of plain attention.  q/dout [B,L,H_q,D], k/v [B,L,H_kv,D] ->
    (dq [B,L,H_q,D], dk, dv [B,L,H_kv,D])."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, L, H_q, D = q.shape
    H_kv = k.shape[2]
    assert k.shape == (B, L, H_kv, D) and v.shape == k.shape and dout.shape == q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _load().ora_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, L, H_q, H_kv,
                                        D, float(scale), int(bool(causal)), _ptr(dq), _ptr(dk),
                                        _ptr(dv), nthreads)
    _check(rc, "attention_backward")
    return dq, dk, dv


def attention_backward_pair(q, k, v, out, lse, dout, scale: float, causal: bool,
                            nthreads: int = 0):
    """One ring step's share of the gradients: queries q [B,Lq,H_q,D] (with the forward's
    final out [B,Lq,H_q,D] and lse [B,H_q,Lq] over the whole sequence, and dout) against the
    keys of one chunk k/v [B,Lk,H_kv,D]; causal: the chunk's own keys (Lq == Lk), key j
    seen by query i only when j <= i.  Returns (dq [B,Lq,H_q,D], dk, dv [B,Lk,H_kv,D])."""
    q, k, v, out, lse, dout = _f64(q), _f64(k), _f64(v), _f64(out), _f64(lse), _f64(dout)
    B, Lq, H_q, D = q.shape
    _, Lk, H_kv, _ = k.shape
    assert k.shape == (B, Lk, H_kv, D) and v.shape == k.shape
    assert out.shape == q.shape and dout.shape == q.shape and lse.shape == (B, H_q, Lq)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _load().ora_attention_backward_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                             _ptr(dout), B, Lq, Lk, H_q, H_kv, D, float(scale),
                                             int(bool(causal)), _ptr(dq), _ptr(dk), _ptr(dv),
                                             nthreads)
    _check(rc, "attention_backward_pair")
    return dq, dk, dv


def attention_backward_rows(q, k, v, dout, scale: float, causal: bool, q_rows, k_rows,
                            positions=None, lower_bounds=None, nthreads: int = 0):
    """Gradients of plain attention on sampled rows: dQ of the query rows q_rows = (b, t, h)
    and dK, dV of the key rows k_rows = (b, t, kv head).  q/dout [B,L,H_q,D], k/v
    [B,L,H_kv,D] in storage order; positions [L] (sequence position of each stored token,
    default t) and lower_bounds [B,L] (smallest key position a query may see) as for
    ring_attention.  Returns (dq [nq,D], dk [nk,D], dv [nk,D])."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, L, H_q, D = q.shape
    H_kv = k.shape[2]
    assert k.shape == (B, L, H_kv, D) and v.shape == k.shape and dout.shape == q.shape
    qb, qt, qh = (np.ascontiguousarray(x, dtype=dt) for x, dt in
                  zip(q_rows, (np.int32, np.int64, np.int32)))
    kb, kt, kg = (np.ascontiguousarray(x, dtype=dt) for x, dt in
                  zip(k_rows, (np.int32, np.int64, np.int32)))
    assert qb.shape == qt.shape == qh.shape and kb.shape == kt.shape == kg.shape
    pos = None if positions is None else np.ascontiguousarray(positions, dtype=np.int64)
    lo = None if lower_bounds is None else np.ascontiguousarray(lower_bounds, dtype=np.int64)
    assert pos is None or pos.shape == (L,)
    assert lo is None or lo.shape == (B, L)
    nq, nk = qb.shape[0], kb.shape[0]
    dq = np.empty((nq, D), np.float64)
    dk = np.empty((nk, D), np.float64)
    dv = np.empty((nk, D), np.float64)
    rc = _load().ora_attention_backward_rows(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, L, H_q, H_kv, D, float(scale),
        int(bool(causal)), _ptr(pos) if pos is not None else None,
        _ptr(lo) if lo is not None else None, nq, _ptr(qb), _ptr(qt), _ptr(qh), nk, _ptr(kb),
        _ptr(kt), _ptr(kg), _ptr(dq), _ptr(dk), _ptr(dv), nthreads)
    _check(rc, "attention_backward_rows")
    return dq, dk, dv


def attention_rows(q_rows, rb, rt, rh, k, v, H_q: int, scale: float, causal: bool,
                   nthreads: int = 0):
    """Plain attention for sampled query rows.

    q_rows [n,D] are the query vectors of rows (rb[i], rt[i], rh[i]); k/v [B,L,H_kv,D].
    Returns (out [n,D], lse [n]).
    """
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    rb = np.ascontiguousarray(rb, dtype=np.int32)
    rt = np.ascontiguousarray(rt, dtype=np.int64)
    rh = np.ascontiguousarray(rh, dtype=np.int32)
    n, D = q_rows.shape
    B, L, H_kv, Dk = k.shape
    assert Dk == D and v.shape == k.shape and rb.shape == rt.shape == rh.shape == (n,)
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().ora_attention_rows(_ptr(q_rows), _ptr(rb), _ptr(rt), _ptr(rh), n, _ptr(k),
                                    _ptr(v), B, L, H_q, H_kv, D, float(scale), int(bool(causal)),
                                    _ptr(out), _ptr(lse), nthreads)
    _check(rc, "attention_rows")
    return out, lse


def ring_attention(q, k_chunks, v_chunks, scale: float, causal: bool, step_offset=None,
                   positions=None, lower_bounds=None, nthreads: int = 0):
    """Ring form.  q [B,P*Lc,H_q,D]; k_chunks/v_chunks [P,B,Lc,H_kv,D] -> (out, lse).

    Rank i visits chunk (i - step_offset[s]) mod P at step s (default: ring order s).
    positions [P*Lc]: sequence position of each rank-major token (default: contiguous,
    position = index); the causal mask compares positions.
    lower_bounds [B, P*Lc]: smallest key position each query may see (packed samples)."""
    q, kc, vc = _f64(q), _f64(k_chunks), _f64(v_chunks)
    P, B, Lc, H_kv, D = kc.shape
    H_q = q.shape[2]
    assert q.shape == (B, P * Lc, H_q, D) and vc.shape == kc.shape
    so = None
    if step_offset is not None:
        so = np.ascontiguousarray(step_offset, dtype=np.int32)
        assert so.shape == (P,)
    pos = None
    if positions is not None:
        pos = np.ascontiguousarray(positions, dtype=np.int64)
        assert pos.shape == (P * Lc,)
    lo = None
    if lower_bounds is not None:
        lo = np.ascontiguousarray(lower_bounds, dtype=np.int64)
        assert lo.shape == (B, P * Lc)
    out = np.empty((B, P * Lc, H_q, D), np.float64)
    lse = np.empty((B, H_q, P * Lc), np.float64)
    rc = _load().ora_ring_attention(_ptr(q), _ptr(kc), _ptr(vc), P, B, Lc, H_q, H_kv, D,
                                    float(scale), int(bool(causal)),
                                    _ptr(so) if so is not None else None,
                                    _ptr(pos) if pos is not None else None,
                                    _ptr(lo) if lo is not None else None, _ptr(out), _ptr(lse),
                                    nthreads)
    _check(rc, "ring_attention")
    return out, lse


def zigzag_positions(P: int, Lc: int) -> np.ndarray:
    """Sequence position of each rank-major token in the zigzag layout: rank i holds
    segment i and segment 2P-1-i of the 2P segments of Lc/2 tokens ([P*Lc] int64)."""
    pos = np.empty((P * Lc,), np.int64)
    _check(_load().ora_zigzag_positions(P, Lc, _ptr(pos)), "zigzag_positions")
    return pos


def packed_lower_bounds(position_ids) -> np.ndarray:
    """position_ids [B, L] (0, 1, 2, ... within each packed sample) -> the position where
    each token's sample starts, [B, L] int64."""
    pid = np.ascontiguousarray(position_ids, dtype=np.int32)
    B, L = pid.shape
    lo = np.empty((B, L), np.int64)
    _check(_load().ora_packed_lower_bounds(_ptr(pid), B, L, _ptr(lo)), "packed_lower_bounds")
    return lo


def ring_attention_packed(q, k_chunks, v_chunks, scale: float, position_ids, nthreads: int = 0):
    """The causal ring form over packed samples (contiguous shards): query t sees the keys
    of its own sample up to itself."""
    return ring_attention(q, k_chunks, v_chunks, scale, True,
                          lower_bounds=packed_lower_bounds(position_ids), nthreads=nthreads)


def ring_attention_zigzag(q, k_chunks, v_chunks, scale: float, causal: bool, nthreads: int = 0):
    """The ring form over shards in the zigzag layout (see zigzag_positions)."""
    P, _, Lc = np.shape(k_chunks)[:3]
    return ring_attention(q, k_chunks, v_chunks, scale, causal,
                          positions=zigzag_positions(P, Lc), nthreads=nthreads)


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Merge of two partials.  o [B,L,H,D], lse [B,H,L] -> new (o, lse) (inputs untouched)."""
    o = _f64(o_a).copy()
    l = _f64(lse_a).copy()
    ob, lb = _f64(o_b), _f64(lse_b)
    B, L, H, D = o.shape
    assert l.shape == (B, H, L) and ob.shape == o.shape and lb.shape == l.shape
    _check(_load().ora_lse_merge(_ptr(o), _ptr(l), _ptr(ob), _ptr(lb), B, H, L, D), "lse_merge")
    return o, l


def seq2head(x: np.ndarray, H_out: int, groups: int | None = None) -> np.ndarray:
    """[P,B,Lc,H_in,D] -> [G,B,P*Lc,H_out/G,D] (G = groups, default P), any dtype, bit-exact."""
    x = np.ascontiguousarray(x)
    P, B, Lc, H_in, D = x.shape
    G = P if groups is None else groups
    if H_out % G or H_out % H_in:
        raise ValueError("seq2head: H_out must divide by the group count and by H_in")
    out = np.empty((G, B, P * Lc, H_out // G, D), x.dtype)
    _check(_load().ora_seq2head(_ptr(x), _ptr(out), P, G, B, Lc, H_in, H_out, D, x.itemsize),
           "seq2head")
    return out


def head2seq(x: np.ndarray, P: int | None = None) -> np.ndarray:
    """[G,B,P*Lc,H/G,D] -> [P,B,Lc,H,D] (P shards, default G), any dtype, bit-exact."""
    x = np.ascontiguousarray(x)
    G, B, L, Hl, D = x.shape
    P = G if P is None else P
    if L % P:
        raise ValueError("head2seq: global length must divide by P")
    Lc = L // P
    out = np.empty((P, B, Lc, Hl * G, D), x.dtype)
    _check(_load().ora_head2seq(_ptr(x), _ptr(out), P, G, B, Lc, Hl * G, D, x.itemsize),
           "head2seq")
    return out


def replica_sum(x, H_out: int) -> np.ndarray:
    """The gradient of the GQA copy: x [..., H_in, D] (H_in = H_out * rep, replica j a copy
    of head j // rep) -> [..., H_out, D], each head the sum of its replicas (fp64)."""
    x = _f64(x)
    *lead, H_in, D = x.shape
    rows = int(np.prod(lead)) if lead else 1
    out = np.empty((*lead, H_out, D), np.float64)
    _check(_load().ora_replica_sum(_ptr(x), _ptr(out), rows, H_in, H_out, D), "replica_sum")
    return out


def usp_attention(q, k, v, P_u: int, scale: float, causal: bool, nthreads: int = 0):
    """The ring x Ulysses hybrid over P sequence shards: q [P,B,Ls,H_q,D], k/v
    [P,B,Ls,H_kv,D].  The heads are split over P_u Ulysses groups (KV heads copied up to
    lcm(H_kv, P_u)), each group runs the ring over P/P_u chunks of the whole sequence, and
    the result comes back sequence-sharded: (out [P,B,Ls,H_q,D], lse [B,H_q,P*Ls])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    P, B, Ls, H_q, D = q.shape
    H_kv = k.shape[3]
    P_r = P // P_u
    assert P_r * P_u == P and H_q % P_u == 0
    H_rep = H_kv * P_u // np.gcd(H_kv, P_u)
    qh = seq2head(q, H_q, groups=P_u)             # [G, B, L, H_q/G, D]
    kh = seq2head(k, H_rep, groups=P_u)
    vh = seq2head(v, H_rep, groups=P_u)
    L = P * Ls
    Lr = L // P_r
    G, Hq_l, Hkv_l = P_u, H_q // P_u, H_rep // P_u
    qa = qh.reshape(G * B, L, Hq_l, D)
    kc = np.ascontiguousarray(kh.reshape(G * B, P_r, Lr, Hkv_l, D).transpose(1, 0, 2, 3, 4))
    vc = np.ascontiguousarray(vh.reshape(G * B, P_r, Lr, Hkv_l, D).transpose(1, 0, 2, 3, 4))
    o, lse = ring_attention(qa, kc, vc, scale, causal, nthreads=nthreads)
    out = head2seq(o.reshape(G, B, L, Hq_l, D), P=P)
    lse_full = lse.reshape(G, B, Hq_l, L).transpose(1, 0, 2, 3).reshape(B, H_q, L)
    return out, lse_full
