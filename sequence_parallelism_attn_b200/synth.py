"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and lays them out; it holds none of the
attention, merge or permute arithmetic, so both the CUDA path and the CPU oracle
can consume what it makes.

Recipe (every workload): a CPU ``torch.Generator`` seeded with ``seed`` draws
Q, then K, then V as fp32 i.i.d. N(0, 1); Q is multiplied by ``q_mult`` (a power
of two, so the multiply is exact in every dtype); the tensors are then rounded
to nearest-even into the workload dtype.  The shapes follow the pages' workloads:
long contexts split into P contiguous chunks ("Как работает sequence
parallelism в контексте LLM?", section 2), Llama/Qwen-like head counts with
grouped KV heads, and the Ulysses seq-sharded activations [local_seqlen,
global_heads, head_dim] ("Метод контекстного параллелизма Ulysses").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    P: int
    Lc: int
    dtype: torch.dtype
    causal: bool
    q_mult: float = 1.0
    seed: int = 0

    @property
    def L(self) -> int:
        return self.P * self.Lc

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def flops(self) -> float:
        """Algorithmic FLOPs 4*B*H_q*L^2*D (two matmuls), halved when causal."""
        f = 4.0 * self.B * self.H_q * float(self.L) ** 2 * self.D
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class UlyssesWorkload:
    name: str
    P: int          # context-parallel ranks
    B: int
    Lc: int         # tokens per rank
    H_q: int        # global query heads
    H_kv: int       # global kv heads (replicated up to max(H_kv, P))
    D: int
    dtype: torch.dtype
    causal: bool
    seed: int = 0
    groups: int | None = None  # head groups G (Ulysses: G = P; ring x Ulysses hybrid: G < P)

    @property
    def G(self) -> int:
        return self.P if self.groups is None else self.groups

    @property
    def H_kv_rep(self) -> int:
        """KV heads after the GQA copy: the least count that both the head groups and the
        source heads divide (8 for 4 KV heads on 8 ranks)."""
        return math.lcm(self.H_kv, self.G)

    def attn(self) -> AttnWorkload:
        """The attention after seq->head: the head groups become the batch.  Ulysses itself
        (no groups given) runs the ring over the P chunks of Lc tokens; the hybrid over the
        P/G chunks each group's ring ranks hold."""
        P_r = self.P if self.groups is None else self.P // self.G
        return AttnWorkload(self.name + "/attn", B=self.G * self.B, H_q=self.H_q // self.G,
                            H_kv=self.H_kv_rep // self.G, D=self.D, P=P_r,
                            Lc=self.P * self.Lc // P_r, dtype=self.dtype, causal=self.causal,
                            seed=self.seed)

    def permute_bytes(self) -> int:
        """Bytes a permute step must move: read each input once, write every output once."""
        es = torch.tensor([], dtype=self.dtype).element_size()
        n_tok = self.P * self.B * self.Lc
        q = 2 * n_tok * self.H_q * self.D                      # Q in, Q out
        kv = 2 * n_tok * (self.H_kv + self.H_kv_rep) * self.D  # K and V: in once, replicas out
        o = 2 * n_tok * self.H_q * self.D                      # O back, same size as Q
        return (q + kv + o) * es


@dataclass(frozen=True)
class MergeWorkload:
    """Two partial attention results (O [B,L,H,D], LSE [B,H,L], fp32) merged into one."""
    name: str
    B: int
    H: int
    L: int
    D: int
    seed: int = 0

    def bytes(self) -> int:
        """Bytes a merge must move: read O_a, O_b and both LSEs, write O_a and LSE_a."""
        return self.B * self.H * self.L * (3 * self.D * 4 + 12)


# The workloads, named by what they are.
TINY_FP32 = AttnWorkload("tiny_fp32_L128", B=1, H_q=2, H_kv=2, D=32, P=2, Lc=64,
                         dtype=torch.float32, causal=False, seed=1001)
SMALL_BF16 = AttnWorkload("bf16_L4096_H8_D64", B=1, H_q=8, H_kv=8, D=64, P=4, Lc=1024,
                          dtype=torch.bfloat16, causal=False, seed=1002)
LLAMA8B_GQA = AttnWorkload("llama8b_gqa_causal_L32768", B=1, H_q=32, H_kv=8, D=128, P=8,
                           Lc=4096, dtype=torch.bfloat16, causal=True, q_mult=4.0, seed=1003)
LONG_128K = AttnWorkload("causal_L131072_H8_D128", B=1, H_q=8, H_kv=8, D=128, P=16, Lc=8192,
                         dtype=torch.bfloat16, causal=True, seed=1004)
ULYSSES_128K = UlyssesWorkload("ulysses_e2e_L131072", P=8, B=1, Lc=16384, H_q=32, H_kv=4,
                               D=128, dtype=torch.bfloat16, causal=True, seed=1005)
USP_128K = UlyssesWorkload("usp_e2e_L131072_G4", P=8, B=1, Lc=16384, H_q=32, H_kv=4,
                           D=128, dtype=torch.bfloat16, causal=True, seed=1005, groups=4)
ULYSSES_32K = UlyssesWorkload("ulysses_e2e_L32768", P=8, B=1, Lc=4096, H_q=32, H_kv=4,
                              D=128, dtype=torch.bfloat16, causal=True, seed=1006)
TINY_PERMUTE = UlyssesWorkload("tiny_permute", P=2, B=1, Lc=64, H_q=2, H_kv=2, D=32,
                               dtype=torch.float32, causal=False, seed=1001)
SMALL_PERMUTE = UlyssesWorkload("small_permute", P=4, B=1, Lc=1024, H_q=8, H_kv=8, D=64,
                                dtype=torch.bfloat16, causal=False, seed=1002)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device="cpu"):
    return torch.randn(*shape, generator=g, dtype=torch.float32, device=device)


def attention_inputs(w: AttnWorkload, device="cpu", seed: int | None = None):
    """Q [B, P*Lc, H_q, D] and K/V chunks [P, B, Lc, H_kv, D] (chunk j = rank j's K/V).

    With device="cuda" the numbers come from a CUDA generator (same recipe,
    different stream of numbers): used where no oracle comparison follows.
    """
    g = _gen(w.seed if seed is None else seed, device)
    q = _normal((w.B, w.L, w.H_q, w.D), g, device)
    if w.q_mult != 1.0:
        q.mul_(w.q_mult)
    k = _normal((w.P, w.B, w.Lc, w.H_kv, w.D), g, device)
    v = _normal((w.P, w.B, w.Lc, w.H_kv, w.D), g, device)
    return q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def ulysses_inputs(w: UlyssesWorkload, device="cpu", seed: int | None = None):
    """Sequence-sharded Q [P, B, Lc, H_q, D] and K/V [P, B, Lc, H_kv, D]."""
    g = _gen(w.seed if seed is None else seed, device)
    q = _normal((w.P, w.B, w.Lc, w.H_q, w.D), g, device)
    k = _normal((w.P, w.B, w.Lc, w.H_kv, w.D), g, device)
    v = _normal((w.P, w.B, w.Lc, w.H_kv, w.D), g, device)
    return q.to(w.dtype), k.to(w.dtype), v.to(w.dtype)


def merge_inputs(B: int, H: int, L: int, D: int, seed: int, neg_inf_frac: float = 0.0):
    """Two partials (o [B,L,H,D] fp32, lse [B,H,L] fp32) with lse ~ 4*N(0,1);
    a fraction of each side's rows is set to the empty partial (o = 0, lse = -inf)."""
    g = _gen(seed)
    out = []
    for _ in range(2):
        o = _normal((B, L, H, D), g)
        lse = 4.0 * _normal((B, H, L), g)
        if neg_inf_frac > 0:
            mask = torch.rand((B, H, L), generator=g) < neg_inf_frac
            lse[mask] = float("-inf")
            o.permute(0, 2, 1, 3)[mask] = 0.0
        out += [o, lse]
    return tuple(out)


def packed_lengths(L: int, seed: int, min_len: int, max_len: int) -> list[int]:
    """Seeded lengths of the samples packed into one L-token sequence: log-uniform in
    [min_len, max_len] (short and long documents alike), the last one cut to fit."""
    g = _gen(seed)
    out, total = [], 0
    lo, hi = math.log(min_len), math.log(max_len)
    while total < L:
        n = int(round(math.exp(lo + (hi - lo) * torch.rand((), generator=g).item())))
        n = max(1, min(n, L - total))
        out.append(n)
        total += n
    return out


def position_ids_from_lengths(lengths_per_row: list[list[int]]) -> torch.Tensor:
    """position_ids [B, L] int32: 0, 1, 2, ... within each packed sample."""
    rows = [torch.cat([torch.arange(n, dtype=torch.int32) for n in lens]) for lens in lengths_per_row]
    return torch.stack(rows)


def sample_rows(B: int, H_q: int, L: int, n: int, seed: int, Lc: int | None = None,
                tile: int = 128):
    """Seeded sample of (b, t, h) query rows: n random rows plus every chunk's first and
    last row and the first/last row of each 128-row tile at chunk edges."""
    g = _gen(seed)
    t = torch.randint(0, L, (n,), generator=g)
    b = torch.randint(0, B, (n,), generator=g)
    h = torch.randint(0, H_q, (n,), generator=g)
    extra_t = [0, L - 1]
    if Lc:
        for c in range(0, L, Lc):
            extra_t += [c, min(c + Lc - 1, L - 1), min(c + tile - 1, L - 1),
                        min(c + tile, L - 1)]
    extra_t = torch.tensor(sorted(set(extra_t)))
    eb = torch.randint(0, B, (len(extra_t),), generator=g)
    eh = torch.randint(0, H_q, (len(extra_t),), generator=g)
    return (torch.cat([b, eb]).tolist(), torch.cat([t, extra_t]).tolist(),
            torch.cat([h, eh]).tolist())
MERGE_128K = MergeWorkload("lse_merge_L131072_H8_D128", B=1, H=8, L=131072, D=128, seed=1007)
