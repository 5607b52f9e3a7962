"""The input recipe on the CPU: seeded, reproducible draws of the shapes each workload
names; Q scaled by an exact power of two; the algorithmic work and bytes each benchmark
line divides by; packed-sample lengths and position_ids valid for the oracle's reading;
row samples that include every chunk edge.  (Module shared by the oracle tests and the
GPU path; it draws and lays out numbers and holds none of the method's arithmetic.)"""
import math

import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth


def test_attention_inputs_shapes_and_reproducibility():
    w = synth.AttnWorkload("t", B=2, H_q=4, H_kv=2, D=16, P=3, Lc=5, dtype=torch.bfloat16,
                           causal=True, q_mult=4.0, seed=17)
    q, k, v = synth.attention_inputs(w)
    assert q.shape == (2, 15, 4, 16) and k.shape == v.shape == (3, 2, 5, 2, 16)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    q2, k2, v2 = synth.attention_inputs(w)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    # Q x 4 is exact: the same draw without the multiplier, times 4, in bf16
    w1 = synth.AttnWorkload("t", B=2, H_q=4, H_kv=2, D=16, P=3, Lc=5, dtype=torch.bfloat16,
                            causal=True, q_mult=1.0, seed=17)
    q1, k1, _ = synth.attention_inputs(w1)
    assert torch.equal(q, (q1.float() * 4).to(torch.bfloat16)) and torch.equal(k, k1)
    # another seed, other numbers
    q3, _, _ = synth.attention_inputs(w, seed=18)
    assert not torch.equal(q, q3)


def test_ulysses_inputs_and_derived_attention():
    w = synth.ULYSSES_128K
    assert w.H_kv_rep == 8 and w.G == w.P == 8
    a = w.attn()
    assert (a.B, a.H_q, a.H_kv, a.P, a.Lc, a.L) == (8, 4, 1, 8, 16384, 131072)
    u = synth.USP_128K
    au = u.attn()
    assert u.H_kv_rep == 4  # lcm(4 kv heads, 4 groups): one kv head per group
    assert (u.G, au.B, au.H_q, au.H_kv, au.P, au.Lc) == (4, 4, 8, 1, 2, 65536)
    small = synth.UlyssesWorkload("s", P=4, B=1, Lc=3, H_q=8, H_kv=2, D=8,
                                  dtype=torch.bfloat16, causal=True, seed=3)
    q, k, v = synth.ulysses_inputs(small)
    assert q.shape == (4, 1, 3, 8, 8) and k.shape == v.shape == (4, 1, 3, 2, 8)


def test_work_and_bytes_of_the_benchmark_lines():
    # causal attention FLOPs 4 B H L^2 D / 2 (the 128k long-context and Ulysses steps)
    assert synth.LONG_128K.flops() == 4.0 * 8 * 131072 ** 2 * 128 / 2
    assert math.isclose(synth.LONG_128K.flops(), 3.518e13, rel_tol=1e-3)
    assert math.isclose(synth.ULYSSES_128K.attn().flops(), 1.407e14, rel_tol=1e-3)
    # permute bytes of the Ulysses step: Q in/out, K/V in once + replicas out, O back
    assert synth.ULYSSES_128K.permute_bytes() == 5100273664
    nc = synth.AttnWorkload("nc", B=1, H_q=2, H_kv=2, D=8, P=2, Lc=4, dtype=torch.float32,
                            causal=False)
    assert nc.flops() == 4.0 * 2 * 8 ** 2 * 8


@pytest.mark.parametrize("L,lo,hi", [(131072, 512, 32768), (1024, 1, 40), (8192, 64, 2048)])
def test_packed_lengths_and_position_ids(oracle_mod, L, lo, hi):
    lens = synth.packed_lengths(L, 42, lo, hi)
    assert sum(lens) == L and all(1 <= n <= hi for n in lens)
    assert all(n >= lo for n in lens[:-1])  # only the last one is cut to fit
    assert lens == synth.packed_lengths(L, 42, lo, hi)
    pid = synth.position_ids_from_lengths([lens]).numpy()
    assert pid.dtype == np.int32 and pid.shape == (1, L)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    assert np.all(pid[0, starts] == 0) and np.count_nonzero(pid[0] == 0) == len(lens)
    # the oracle's reading accepts them, and each token's sample starts where it should
    lower = oracle_mod.packed_lower_bounds(pid)
    want = np.repeat(starts, lens)
    assert np.array_equal(lower[0], want)


def test_sample_rows_cover_every_chunk_edge():
    B, H, L, Lc = 2, 4, 1000, 300
    rb, rt, rh = synth.sample_rows(B, H, L, 64, seed=5, Lc=Lc)
    assert len(rb) == len(rt) == len(rh) >= 64
    assert all(0 <= b < B for b in rb) and all(0 <= h < H for h in rh)
    assert all(0 <= t < L for t in rt)
    for c in range(0, L, Lc):
        assert c in rt and min(c + Lc - 1, L - 1) in rt
    assert 0 in rt and L - 1 in rt
    assert synth.sample_rows(B, H, L, 64, seed=5, Lc=Lc) == (rb, rt, rh)
