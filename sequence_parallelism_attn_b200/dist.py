"""The data plane across GPUs: the ring's K/V exchange and the Ulysses all-to-alls over
torch.distributed (NCCL between GPUs, one process per GPU), with the library's kernels
for every computation.

Ring ("Как работает sequence parallelism в контексте LLM?", sections 3 and 5): rank i
keeps its query chunk; at step s = 0 .. P-1 it holds K/V chunk j = (i - s) mod P and
attends its queries to it while that chunk travels on to rank i + 1 and the next one
arrives from rank i - 1 into a second buffer (P - 1 exchanges, each overlapped with one
step's attention).  Each step's partial (O, LSE) is merged into the running result by
ra_lse_merge.  Under the causal mask (global positions in rank order) chunk j < i is
wholly visible, j == i is the diagonal, and j > i is skipped: no launch, although the
chunk still travels on.

Ulysses ("Метод контекстного параллелизма Ulysses"): seq->head is pack -> all-to-all ->
unpack.  The pack is the library's grouped transform of this rank's tokens into P
destination blocks of H_out / P heads (with the GQA copy), so each peer's slice is one
contiguous block; the all-to-all swaps block r of every rank into rank r; the unpack puts
the P received token blocks in source-rank order (a view when B = 1).  head->seq is the
inverse.  No kernel reads another GPU's memory: every remote block lands in this GPU's
own buffers through NCCL before a kernel touches it.  ulysses_seq2head_p2p /
ulysses_head2seq_p2p do the same exchange with one kernel per rank that stores its share
straight into the peers' symmetric-memory buffers (PeerBuffers), between two cross-rank
barriers.

The ring backward (ring_attn_bwd_dist) moves each K/V chunk the same way, with fp32 dK, dV
accumulators that every rank adds its share into before passing them on; the last pass
returns them to the chunk's own rank.  The Ulysses / USP backward (usp_attn_bwd_dist) wraps
it in the same all-to-alls, and sums the GQA replicas' dK, dV back onto their heads.

Every rank takes the same collective steps in the same order.  A peer that leaves between
steps ends the next exchange with an error (the process group's timeout bounds the wait),
raised here as ExchangeError naming the step and the peers.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class ExchangeError(RuntimeError):
    """An exchange with a peer failed (a peer left, or the process group timed out)."""


def chunk_pair(i: int, j: int, causal: bool) -> str:
    """How query chunk i sees K/V chunk j: "full", "diagonal" (causal inside the chunk) or
    "skip" (every key after every query).  Non-causal: always "full"."""
    if not causal:
        return "full"
    if j < i:
        return "full"
    return "diagonal" if j == i else "skip"


def ring_schedule(rank: int, world: int) -> list[int]:
    """The K/V chunk rank `rank` holds at each step: (rank - s) mod world, s = 0 .. world-1."""
    return [(rank - s) % world for s in range(world)]


class DeviceOps:
    """The computations of the distributed path, each one library call."""

    @staticmethod
    def attend(q, k, v, causal_diagonal, scale, out, lse):
        from . import ra
        ra.ring_attn_fwd(q, [k], [v], causal_diagonal, scale, out=out, lse=lse)

    @staticmethod
    def merge(o_a, lse_a, o_b, lse_b):
        from . import ra
        ra.ra_lse_merge(o_a, lse_a, o_b, lse_b)

    @staticmethod
    def attend_bwd(q, k, v, out, lse, dout, causal_diagonal, scale, dq, dk, dv):
        """Add the gradient share of (these queries, one K/V chunk) into dq, dk, dv, with the
        forward's final out and lse (ra_ring_attn_bwd_accumulate)."""
        from . import ra
        ra.ring_attn_bwd(q, k.unsqueeze(0), v.unsqueeze(0), out, lse, dout, causal_diagonal,
                         scale, dq=dq, dk=dk.unsqueeze(0), dv=dv.unsqueeze(0), accumulate=True)

    @staticmethod
    def replica_sum(x, H_out):
        """[B, Lc, H_in, D] fp32 -> [B, Lc, H_out, D]: the gradient of the GQA copy, each
        head the sum of its replicas."""
        from . import ra
        return ra.ra_ulysses_replica_sum(x, H_out)

    @staticmethod
    def seq2head_pack(x, H_out, P):
        """[B, Lc, H_in, D] -> [P, B, Lc, H_out / P, D]: block r = the heads of rank r."""
        from . import ra
        return ra.ra_ulysses_seq2head(x.unsqueeze(0), H_out, groups=P)

    @staticmethod
    def seq2head_unpack(recv):
        """[P, B, Lc, Hl, D] (block s from rank s) -> [B, P * Lc, Hl, D]."""
        from . import ra
        P, B, Lc, Hl, D = recv.shape
        if B == 1:
            return recv.view(1, P * Lc, Hl, D)
        return ra.ra_ulysses_seq2head(recv, Hl, groups=1).view(B, P * Lc, Hl, D)

    @staticmethod
    def head2seq_pack(y, P):
        """[B, P * Lc, Hl, D] -> [P, B, Lc, Hl, D]: block s = the tokens of rank s."""
        from . import ra
        B, L, Hl, D = y.shape
        if B == 1:
            return y.view(P, 1, L // P, Hl, D)
        return ra.ra_ulysses_head2seq(y.unsqueeze(0), P=P)

    @staticmethod
    def head2seq_unpack(recv, out=None):
        """[P, B, Lc, Hl, D] (block r = rank r's heads) -> [B, Lc, P * Hl, D] (into `out`
        when given)."""
        from . import ra
        P, B, Lc, Hl, D = recv.shape
        dst = None if out is None else out.view(1, B, Lc, P * Hl, D)
        return ra.ra_ulysses_head2seq(recv, out=dst, P=1).view(B, Lc, P * Hl, D)


def _group_info(group):
    return dist.get_rank(group), dist.get_world_size(group)


def _peer(group, r):
    """Global rank of group rank r (P2P ops address global ranks)."""
    return r if group is None else dist.get_global_rank(group, r)


def _wait(works, what):
    try:
        for w in works:
            w.wait()
    except Exception as e:  # a peer left or the process group timed out
        raise ExchangeError(f"{what}: {e}") from e


class RingAccumulator:
    """Rank i's running attention result over the K/V chunks it visits: the first visited
    chunk writes (O, LSE) directly, every later one is attended into a partial and merged
    in (ra_lse_merge); chunks wholly after the queries (causal) are skipped."""

    def __init__(self, q, rank: int, causal: bool, scale: float | None = None, out=None,
                 lse=None, ops=DeviceOps):
        B, Lc, H_q, D = q.shape
        self.q, self.rank, self.causal, self.ops = q, rank, causal, ops
        self.scale = D ** -0.5 if scale is None else scale
        dev = q.device
        # fp32 results (float64 ones for float64 inputs, which only host-side checks use)
        rdt = torch.float64 if q.dtype == torch.float64 else torch.float32
        self.out = torch.empty((B, Lc, H_q, D), dtype=rdt, device=dev) if out is None else out
        self.lse = torch.empty((B, H_q, Lc), dtype=rdt, device=dev) if lse is None else lse
        self.part = None
        self.visited = 0

    def visit(self, j: int, k, v):
        kind = chunk_pair(self.rank, j, self.causal)
        if kind == "skip":
            return
        diag = kind == "diagonal"
        if self.visited == 0:
            self.ops.attend(self.q, k, v, diag, self.scale, self.out, self.lse)
        else:
            if self.part is None:
                self.part = (torch.empty_like(self.out), torch.empty_like(self.lse))
            self.ops.attend(self.q, k, v, diag, self.scale, *self.part)
            self.ops.merge(self.out, self.lse, *self.part)
        self.visited += 1


def _ring_exchange(k, v, group, visit):
    """The ring's exchange loop: visit(j, k_j, v_j) for the chunk held at each step, while
    the held chunk travels to rank i + 1 and the next arrives from rank i - 1 into the
    second of two receive buffers.  A buffer is received into only after the step that
    read it has been enqueued (NCCL's stream waits for it) and its own send has completed."""
    rank, world = _group_info(group)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)] if world > 1 else []
    held = (k, v)
    nxt_rank, prv_rank = _peer(group, (rank + 1) % world), _peer(group, (rank - 1) % world)
    for s, j in enumerate(ring_schedule(rank, world)):
        works = []
        if s < world - 1:
            nxt = bufs[s % 2]
            p2p = [dist.P2POp(dist.isend, held[0], nxt_rank, group),
                   dist.P2POp(dist.isend, held[1], nxt_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], prv_rank, group),
                   dist.P2POp(dist.irecv, nxt[1], prv_rank, group)]
            try:
                works = dist.batch_isend_irecv(p2p)
            except Exception as e:
                raise ExchangeError(f"ring step {s}: posting the exchange with ranks "
                                    f"{(rank + 1) % world} / {(rank - 1) % world}: {e}") from e
        visit(j, held[0], held[1])
        if works:
            _wait(works, f"ring step {s}: chunk from rank {(rank - 1) % world}")
            held = nxt


def ring_attn_fwd_dist(q, k, v, causal: bool, scale: float | None = None, group=None,
                       out=None, lse=None, ops=DeviceOps):
    """Ring attention across the ranks of `group`: q [B, Lc, H_q, D] is this rank's query
    chunk, k/v [B, Lc, H_kv, D] its K/V chunk (contiguous), rank i holding tokens
    i*Lc .. i*Lc+Lc-1 of the sequence.  Returns this rank's (out [B, Lc, H_q, D] fp32,
    lse [B, H_q, Lc] fp32), equal to attention of its queries over the whole sequence."""
    rank, _ = _group_info(group)
    acc = RingAccumulator(q, rank, causal, scale, out, lse, ops)
    _ring_exchange(k, v, group, acc.visit)
    return acc.out, acc.lse


def ring_attn_bwd_dist(q, k, v, out, lse, dout, causal: bool, scale: float | None = None,
                       group=None, ops=DeviceOps):
    """The backward of ring_attn_fwd_dist across the ranks of `group`: q, dout and out
    [B, Lc, H_q, D] are this rank's query chunk, its output gradient and the forward's
    output (bf16 on the GPU), lse [B, H_q, Lc] the forward's log-sum-exps over the whole
    sequence, k/v [B, Lc, H_kv, D] this rank's K/V chunk.  Returns (dq [B, Lc, H_q, D],
    dk, dv [B, Lc, H_kv, D]) in fp32: the gradients of the loss with respect to this rank's
    chunks.

    The K/V chunks travel the ring as in the forward (rank i holds chunk (i - s) mod P at
    step s, the next one arriving while the step computes), and each carries fp32 dK, dV
    accumulators: rank i adds the share of its queries against the held chunk into dq and
    into those accumulators (one ra_ring_attn_bwd_accumulate, with the forward's final LSE),
    then passes them on with the chunk.  After P steps every chunk's accumulators have met
    every query chunk and the last pass lands them on the chunk's own rank.  Causal: chunk
    pairs j > i add nothing, though the chunk and its accumulators still travel.  The
    accumulators move after the step that adds into them (P passes, each after its step's
    computation); the K/V chunks move during it (P - 1 passes)."""
    rank, world = _group_info(group)
    B, Lc, H_q, D = q.shape
    scale = D ** -0.5 if scale is None else scale
    gdt = torch.float64 if q.dtype == torch.float64 else torch.float32
    dq = torch.zeros(q.shape, dtype=gdt, device=q.device)
    acc = (torch.zeros(k.shape, dtype=gdt, device=k.device),
           torch.zeros(v.shape, dtype=gdt, device=v.device))
    if world > 1:
        kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
        acc_bufs = [(torch.empty_like(acc[0]), torch.empty_like(acc[1])) for _ in range(2)]
    held = (k, v)
    nxt_rank, prv_rank = _peer(group, (rank + 1) % world), _peer(group, (rank - 1) % world)
    for s, j in enumerate(ring_schedule(rank, world)):
        works = []
        if s < world - 1:
            nxt = kv_bufs[s % 2]
            p2p = [dist.P2POp(dist.isend, held[0], nxt_rank, group),
                   dist.P2POp(dist.isend, held[1], nxt_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], prv_rank, group),
                   dist.P2POp(dist.irecv, nxt[1], prv_rank, group)]
            try:
                works = dist.batch_isend_irecv(p2p)
            except Exception as e:
                raise ExchangeError(f"ring backward step {s}: posting the K/V exchange with "
                                    f"ranks {(rank + 1) % world} / {(rank - 1) % world}: {e}") from e
        kind = chunk_pair(rank, j, causal)
        if kind != "skip":
            ops.attend_bwd(q, held[0], held[1], out, lse, dout, kind == "diagonal", scale, dq,
                           acc[0], acc[1])
        if world > 1:  # the held chunk's accumulators move on; the next chunk's arrive
            racc = acc_bufs[s % 2]
            p2p = [dist.P2POp(dist.isend, acc[0], nxt_rank, group),
                   dist.P2POp(dist.isend, acc[1], nxt_rank, group),
                   dist.P2POp(dist.irecv, racc[0], prv_rank, group),
                   dist.P2POp(dist.irecv, racc[1], prv_rank, group)]
            try:
                awork = dist.batch_isend_irecv(p2p)
            except Exception as e:
                raise ExchangeError(f"ring backward step {s}: posting the dK/dV exchange: "
                                    f"{e}") from e
            _wait(awork, f"ring backward step {s}: dK/dV from rank {(rank - 1) % world}")
            acc = racc
        if works:
            _wait(works, f"ring backward step {s}: chunk from rank {(rank - 1) % world}")
            held = nxt
    return dq, acc[0], acc[1]


class ZigzagRingAccumulator:
    """Rank i's causal attention over the zigzag layout's chunks (the load-balanced layout
    named beside the ring in "Метод контекстного параллелизма Ulysses"; rank i holds the
    segments i and 2P-1-i of 2P segments of h = Lc/2 tokens).  The two query halves keep
    separate running results; against rank j's shard (segments j and 2P-1-j, key halves
    K0 and K1):
      j == i: half 0 sees K0 causally; half 1 sees K0 wholly and K1 causally;
      j <  i: both halves see K0 wholly and nothing of K1;
      j >  i: half 0 sees nothing; half 1 sees K0 and K1 wholly.
    Every rank does the same work at every step but the first."""

    def __init__(self, q, rank: int, world: int, scale: float | None = None, ops=DeviceOps):
        B, Lc, H_q, D = q.shape
        if Lc % 2:
            raise ValueError("the zigzag layout needs an even chunk length")
        self.h, self.rank, self.world = Lc // 2, rank, world
        self.q = (q[:, :self.h], q[:, self.h:])
        self.acc = tuple(RingAccumulator(qq, 0, False, scale, ops=ops) for qq in self.q)

    def _add(self, half, k, v, causal_diagonal):
        a = self.acc[half]
        a.causal = causal_diagonal  # the pair decides: "diagonal" when causal, else "full"
        a.visit(0, k, v)

    def visit(self, j: int, k, v):
        K = ((k[:, :self.h], v[:, :self.h]), (k[:, self.h:], v[:, self.h:]))
        if j == self.rank:
            self._add(0, *K[0], True)
            self._add(1, *K[0], False)
            self._add(1, *K[1], True)
        elif j < self.rank:
            self._add(0, *K[0], False)
            self._add(1, *K[0], False)
        else:
            self._add(1, *K[0], False)
            self._add(1, *K[1], False)

    def result(self):
        """(out [B, Lc, H_q, D], lse [B, H_q, Lc]) in the shard's token order."""
        out = torch.cat([self.acc[0].out, self.acc[1].out], dim=1)
        lse = torch.cat([self.acc[0].lse, self.acc[1].lse], dim=2)
        return out, lse


def ring_attn_fwd_zigzag_dist(q, k, v, scale: float | None = None, group=None, ops=DeviceOps):
    """Causal ring attention across the ranks of `group` over shards in the zigzag layout:
    q [B, Lc, H_q, D] and k/v [B, Lc, H_kv, D] are this rank's shard (its segments i and
    2P-1-i, Lc even).  Returns this rank's (out [B, Lc, H_q, D], lse [B, H_q, Lc]) in shard
    order, equal to causal attention of its queries over the sequence in natural order."""
    rank, world = _group_info(group)
    acc = ZigzagRingAccumulator(q, rank, world, scale, ops)
    _ring_exchange(k, v, group, acc.visit)
    return acc.result()


def ring_attn_bwd_zigzag_dist(q, k, v, out, lse, dout, scale: float | None = None, group=None,
                              ops=DeviceOps):
    """The backward of ring_attn_fwd_zigzag_dist (causal): q, out, dout [B, Lc, H_q, D] and
    k/v [B, Lc, H_kv, D] are this rank's shard in the zigzag layout (segments i and 2P-1-i,
    Lc even), lse [B, H_q, Lc] the forward's, in shard order.  Returns (dq, dk, dv) of the
    shard in fp32, in shard order.

    The ring backward of ring_attn_bwd_dist over the shard's halves: the K/V shards travel
    with fp32 dK, dV accumulators kept as two halves (one per segment), and against rank j's
    shard rank i adds the shares of the half-pairs that the forward attended --
      j == i: (Q0, K0) causally, (Q1, K0) wholly, (Q1, K1) causally;
      j <  i: (Q0, K0) and (Q1, K0) wholly;
      j >  i: (Q1, K0) and (Q1, K1) wholly."""
    rank, world = _group_info(group)
    B, Lc, H_q, D = q.shape
    if Lc % 2:
        raise ValueError("the zigzag layout needs an even chunk length")
    h = Lc // 2
    scale = D ** -0.5 if scale is None else scale
    gdt = torch.float64 if q.dtype == torch.float64 else torch.float32
    half = lambda x, c: x[:, c * h:(c + 1) * h].contiguous()
    Q = [half(q, c) for c in (0, 1)]
    O = [half(out, c) for c in (0, 1)]
    dO = [half(dout, c) for c in (0, 1)]
    LSE = [lse[:, :, c * h:(c + 1) * h].contiguous() for c in (0, 1)]
    dq = [torch.zeros(Q[c].shape, dtype=gdt, device=q.device) for c in (0, 1)]
    zero = lambda: torch.zeros((B, h, k.shape[2], k.shape[3]), dtype=gdt, device=k.device)
    acc = [zero(), zero(), zero(), zero()]  # dK0, dK1, dV0, dV1 of the held shard
    acc_bufs = [[torch.empty_like(a) for a in acc] for _ in range(2)] if world > 1 else []
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)] if world > 1 else []
    held = (k, v)
    nxt_rank, prv_rank = _peer(group, (rank + 1) % world), _peer(group, (rank - 1) % world)
    for s, j in enumerate(ring_schedule(rank, world)):
        works = []
        if s < world - 1:
            nxt = kv_bufs[s % 2]
            p2p = [dist.P2POp(dist.isend, held[0], nxt_rank, group),
                   dist.P2POp(dist.isend, held[1], nxt_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], prv_rank, group),
                   dist.P2POp(dist.irecv, nxt[1], prv_rank, group)]
            try:
                works = dist.batch_isend_irecv(p2p)
            except Exception as e:
                raise ExchangeError(f"zigzag ring backward step {s}: posting the K/V exchange: "
                                    f"{e}") from e
        K = [half(held[0], c) for c in (0, 1)]
        V = [half(held[1], c) for c in (0, 1)]
        if j == rank:
            pairs = ((0, 0, True), (1, 0, False), (1, 1, True))
        elif j < rank:
            pairs = ((0, 0, False), (1, 0, False))
        else:
            pairs = ((1, 0, False), (1, 1, False))
        for qc, kc, diag in pairs:
            ops.attend_bwd(Q[qc], K[kc], V[kc], O[qc], LSE[qc], dO[qc], diag, scale, dq[qc],
                           acc[kc], acc[2 + kc])
        if world > 1:
            racc = acc_bufs[s % 2]
            p2p = ([dist.P2POp(dist.isend, a, nxt_rank, group) for a in acc] +
                   [dist.P2POp(dist.irecv, r, prv_rank, group) for r in racc])
            try:
                awork = dist.batch_isend_irecv(p2p)
            except Exception as e:
                raise ExchangeError(f"zigzag ring backward step {s}: posting the dK/dV "
                                    f"exchange: {e}") from e
            _wait(awork, f"zigzag ring backward step {s}: dK/dV from rank {(rank - 1) % world}")
            acc = racc
        if works:
            _wait(works, f"zigzag ring backward step {s}: shard from rank {(rank - 1) % world}")
            held = nxt
    return (torch.cat(dq, dim=1), torch.cat(acc[:2], dim=1), torch.cat(acc[2:], dim=1))


def _all_to_all(send, group, what):
    recv = torch.empty_like(send)
    try:
        dist.all_to_all_single(recv, send, group=group)
    except Exception as e:
        raise ExchangeError(f"{what}: {e}") from e
    return recv


def ulysses_seq2head_dist(x, H_out: int | None = None, group=None, ops=DeviceOps):
    """Ulysses seq->head across the ranks of `group`: x [B, Lc, H_in, D] is this rank's
    sequence shard with every head; returns [B, P*Lc, H_out/P, D], this rank's head block
    (heads [r*H_out/P, (r+1)*H_out/P) after the GQA copy to H_out heads) over the whole
    sequence, tokens in source-rank order."""
    rank, world = _group_info(group)
    H_out = x.shape[2] if H_out is None else H_out
    if H_out % world or H_out % x.shape[2]:
        raise ValueError(f"{H_out} heads do not split over {world} ranks / copy {x.shape[2]}")
    send = ops.seq2head_pack(x, H_out, world)
    recv = _all_to_all(send, group, f"seq2head all-to-all on rank {rank}")
    return ops.seq2head_unpack(recv)


def ulysses_head2seq_dist(y, group=None, ops=DeviceOps, out=None):
    """Ulysses head->seq across the ranks of `group`: y [B, P*Lc, Hl, D] is this rank's
    head block over the whole sequence; returns [B, Lc, P*Hl, D], this rank's sequence
    shard with every head (written into `out`, contiguous, when given)."""
    rank, world = _group_info(group)
    if y.shape[1] % world:
        raise ValueError(f"sequence of {y.shape[1]} tokens does not split over {world} ranks")
    send = ops.head2seq_pack(y, world)
    recv = _all_to_all(send, group, f"head2seq all-to-all on rank {rank}")
    return ops.head2seq_unpack(recv) if out is None else ops.head2seq_unpack(recv, out=out)


# ------------------------------------------------------------------ one-kernel exchange
class PeerBuffers:
    """A buffer of one shape on every rank of `group`, each mapped into every rank's address
    space (torch symmetric memory), for the one-kernel Ulysses exchange: each rank's scatter
    kernel (ra_ulysses_*_scatter) stores its share straight into the peers' buffers over
    NVLink, in place of pack -> all_to_all -> unpack.  The kernel is handed peer addresses
    for plain 16-byte stores only; nothing reads a peer's memory.

    sync() is the cross-rank barrier around a scatter: an all-reduce of one element on the
    current stream (NCCL), so it is ordered after this rank's kernels and the process
    group's timeout bounds the wait."""

    def __init__(self, shape, dtype, group=None, device=None):
        from torch.distributed import _symmetric_memory as symm
        self.group = group
        self.rank, self.world = _group_info(group)
        pg = group if group is not None else dist.group.WORLD
        self.buf = symm.empty(*shape, dtype=dtype, device=device)
        self.handle = symm.rendezvous(self.buf, pg)
        self.ptrs = [int(a) for a in self.handle.buffer_ptrs]
        if len(self.ptrs) != self.world:
            raise RuntimeError(f"symmetric memory gave {len(self.ptrs)} buffers for "
                               f"{self.world} ranks")
        self._token = torch.zeros(1, dtype=torch.float32, device=self.buf.device)

    def sync(self, what):
        try:
            dist.all_reduce(self._token, group=self.group)
        except Exception as e:  # a peer left or the process group timed out
            raise ExchangeError(f"{what}: {e}") from e


def ulysses_seq2head_p2p(x, peer: PeerBuffers, H_out: int | None = None):
    """ulysses_seq2head_dist with the exchange done by one kernel per rank: x [B, Lc, H_in, D]
    is this rank's sequence shard; every rank stores its share into every rank's buffer of
    `peer` ([B, P*Lc, H_out/P, D]), which is returned.  It stays valid until the next
    exchange through the same buffers."""
    return ulysses_seq2head_p2p_many([(x, peer, H_out)])[0]


def ulysses_seq2head_p2p_many(jobs):
    """Several seq->head exchanges (Q, K, V) between one pair of barriers: jobs is a list of
    (x, peer, H_out), every peer over the same group; returns the peers' buffers in order."""
    from . import ra
    if any(peer.group is not jobs[0][1].group for _, peer, _ in jobs):
        raise ValueError("the exchanges of one barrier pair must use one process group")
    for x, peer, H_out in jobs:
        B, Lc, H_in, D = x.shape
        H_out = H_in if H_out is None else H_out
        want = (B, peer.world * Lc, H_out // peer.world, D)
        if H_out % peer.world or H_out % H_in or tuple(peer.buf.shape) != want \
                or peer.buf.dtype != x.dtype:
            raise ValueError(f"peer buffers {tuple(peer.buf.shape)} {peer.buf.dtype} do not "
                             f"hold {want} {x.dtype}")
    first = jobs[0][1]
    first.sync(f"seq2head scatter on rank {first.rank}: buffers free")
    for x, peer, H_out in jobs:
        ra.ra_ulysses_seq2head_scatter(x.contiguous(), peer.ptrs, peer.rank,
                                       x.shape[2] if H_out is None else H_out)
    first.sync(f"seq2head scatter on rank {first.rank}: shares stored")
    return [peer.buf for _, peer, _ in jobs]


def ulysses_head2seq_p2p(y, peer: PeerBuffers):
    """ulysses_head2seq_dist with the exchange done by one kernel per rank: y [B, P*Lc, Hl, D]
    is this rank's head group; every rank stores its share into every rank's buffer of
    `peer` ([B, Lc, P*Hl, D]), which is returned (valid until the next exchange)."""
    from . import ra
    B, L, Hl, D = y.shape
    want = (B, L // peer.world, peer.world * Hl, D)
    if L % peer.world or tuple(peer.buf.shape) != want or peer.buf.dtype != y.dtype:
        raise ValueError(f"peer buffers {tuple(peer.buf.shape)} {peer.buf.dtype} do not hold "
                         f"{want} {y.dtype}")
    peer.sync(f"head2seq scatter on rank {peer.rank}: buffers free")
    ra.ra_ulysses_head2seq_scatter(y.contiguous(), peer.ptrs, peer.rank)
    peer.sync(f"head2seq scatter on rank {peer.rank}: shares stored")
    return peer.buf


def usp_attn_fwd_dist(q, k, v, causal: bool, scale: float | None = None, ulysses_group=None,
                      ring_group=None, ops=DeviceOps):
    """The ring x Ulysses hybrid (USP) across GPUs: the ranks form P_r ring groups of P_u
    Ulysses ranks.  q [B, Ls, H_q, D], k/v [B, Ls, H_kv, D] are this rank's sequence shard
    (every head); the P_u ranks of `ulysses_group` hold consecutive shards and share a head
    split, and `ring_group` holds the P_r ranks at this rank's place in every Ulysses group,
    in sequence order.  seq->head inside the Ulysses group gives this rank H/P_u heads over
    its group's P_u*Ls tokens (KV heads copied up to lcm(H_kv, P_u)); the ring runs across
    the ring group over P_r chunks of P_u*Ls tokens; head->seq brings the output back.
    Returns (out [B, Ls, H_q, D] fp32, lse [B, H_q/P_u, P_u*Ls] of this rank's head block
    over its Ulysses group's tokens)."""
    import math
    P_u = dist.get_world_size(ulysses_group)
    H_q, H_kv = q.shape[2], k.shape[2]
    H_rep = H_kv * P_u // math.gcd(H_kv, P_u)
    qh = ulysses_seq2head_dist(q, H_q, group=ulysses_group, ops=ops)
    kh = ulysses_seq2head_dist(k, H_rep, group=ulysses_group, ops=ops)
    vh = ulysses_seq2head_dist(v, H_rep, group=ulysses_group, ops=ops)
    o, lse = ring_attn_fwd_dist(qh, kh, vh, causal, scale, group=ring_group, ops=ops)
    return ulysses_head2seq_dist(o, group=ulysses_group, ops=ops), lse


def usp_attn_bwd_dist(q, k, v, out, lse, dout, causal: bool, scale: float | None = None,
                      ulysses_group=None, ring_group=None, ops=DeviceOps):
    """The backward of usp_attn_fwd_dist (and of plain Ulysses: a ring group of one rank).
    q, dout and out [B, Ls, H_q, D] (the forward's output, bf16 on the GPU) and k/v
    [B, Ls, H_kv, D] are this rank's sequence shard with every head; lse is the one
    usp_attn_fwd_dist returned (this rank's head block over its Ulysses group's tokens).
    Returns (dq [B, Ls, H_q, D], dk, dv [B, Ls, H_kv, D]) in fp32, the gradients of this
    rank's shard.

    Inside the Ulysses group: seq->head of q, k, v (the GQA copy to lcm(H_kv, P_u) heads),
    out and dout; across the ring group: the ring backward on the head blocks
    (ring_attn_bwd_dist); inside the Ulysses group again: head->seq of the three gradients,
    and the replicas' dK, dV summed back onto the H_kv heads (the copy's gradient,
    ra_ulysses_replica_sum).  The forward's head-layout tensors are exchanged again here
    rather than kept from the forward."""
    import math
    P_u = dist.get_world_size(ulysses_group)
    H_q, H_kv = q.shape[2], k.shape[2]
    H_rep = H_kv * P_u // math.gcd(H_kv, P_u)
    qh = ulysses_seq2head_dist(q, H_q, group=ulysses_group, ops=ops)
    kh = ulysses_seq2head_dist(k, H_rep, group=ulysses_group, ops=ops)
    vh = ulysses_seq2head_dist(v, H_rep, group=ulysses_group, ops=ops)
    oh = ulysses_seq2head_dist(out, H_q, group=ulysses_group, ops=ops)
    doh = ulysses_seq2head_dist(dout, H_q, group=ulysses_group, ops=ops)
    dqh, dkh, dvh = ring_attn_bwd_dist(qh, kh, vh, oh, lse, doh, causal, scale, group=ring_group,
                                       ops=ops)
    dq = ulysses_head2seq_dist(dqh, group=ulysses_group, ops=ops)
    dk = ulysses_head2seq_dist(dkh, group=ulysses_group, ops=ops)
    dv = ulysses_head2seq_dist(dvh, group=ulysses_group, ops=ops)
    if H_rep != H_kv:
        dk, dv = ops.replica_sum(dk, H_kv), ops.replica_sum(dv, H_kv)
    return dq, dk, dv

