"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Nothing here compares the oracle with itself by retyping its formulas: the pins
are a hand-derived worked example (tests/golden), closed forms, the float64
library routine torch.nn.functional.scaled_dot_product_attention, brute force
in 50-digit decimal arithmetic on tiny inputs, and invariants that a dropped
term, a wrong sign or index, or a transposed operand would break.

Sources: "Как работает sequence parallelism в контексте LLM?" sections 2, 3, 5
(chunking, ring order, the per-chunk softmax merged across steps) and "Метод
контекстного параллелизма Ulysses" (the seq<->head transform and the GQA copy).
"""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def exact_attention(q, k, v, scale, causal):
    """Attention of every query row by its definition with exactly rounded sums (math.fsum
    for the dot products, for the sum of exponentials and for each output element's
    weighted sum of V): O [B,L,H_q,D] and LSE [B,H_q,L] to within a few ulps of the
    real values."""
    B, L, H_q, _ = q.shape
    D = v.shape[3]
    rep = H_q // k.shape[2]
    out = np.empty((B, L, H_q, D))
    lse = np.empty((B, H_q, L))
    for b in range(B):
        for h in range(H_q):
            kh, vh = k[b, :, h // rep], v[b, :, h // rep]
            for t in range(L):
                n = t + 1 if causal else L
                s = [scale * math.fsum(q[b, t, h] * kh[j]) for j in range(n)]
                m = max(s)
                l = m + math.log(math.fsum(math.exp(x - m) for x in s))
                w = [math.exp(x - l) for x in s]
                lse[b, h, t] = l
                for d in range(D):
                    out[b, t, h, d] = math.fsum(w[j] * vh[j, d] for j in range(n))
    return out, lse


def exact_lse(q, k, scale, causal):
    """The log-sum-exp of every query row by its definition with exactly rounded sums."""
    return exact_attention(q, k, np.zeros(k.shape[:3] + (1,)), scale, causal)[1]


def torch_sdpa(q, k, v, scale, causal):
    """float64 library attention (torch SDPA) for the output; the LSE, which the library
    does not return, by its definition with exactly rounded sums.  (torch's own float64
    matmul + logsumexp on the CPU was seen, in about one process in twenty, to take a path
    about 1e-10 off the exact value, so it serves as no reference.)
    q [B,L,H_q,D], k/v [B,L,H_kv,D] -> out, lse."""
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, scale=scale, is_causal=causal, enable_gqa=True)
    return out.permute(0, 2, 1, 3).numpy(), exact_lse(q, k, scale, causal)


# ---------------------------------------------------------------- worked example
def test_golden_three_keys(oracle_mod):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "attention_three_keys.txt"))
            if l.strip() and not l.startswith("#")]
    q = np.tile(np.array([math.log(3.0), math.log(2.0)]), (1, 3, 1, 1))
    k = np.array([[0, 0], [1, 0], [0, 1]], np.float64).reshape(1, 3, 1, 2)
    v = np.array([[6, 0], [0, 6], [3, 3]], np.float64).reshape(1, 3, 1, 2)
    for causal in (0, 1):
        out, lse = oracle_mod.attention(q, k, v, 1.0, bool(causal))
        for r in rows:
            if int(r[0]) != causal:
                continue
            t = int(r[1])
            np.testing.assert_allclose(out[0, t, 0], [float(r[2]), float(r[3])], atol=1e-13)
            np.testing.assert_allclose(lse[0, 0, t], math.log(float(r[4])), atol=1e-13)


# ---------------------------------------------------------------- library routine
@pytest.mark.parametrize("B,L,H_q,H_kv,D,causal", [
    (1, 37, 2, 2, 8, False), (2, 64, 4, 2, 16, True), (1, 50, 6, 3, 32, True),
    (1, 129, 8, 1, 4, False), (1, 33, 4, 4, 64, True)])
def test_plain_matches_torch_sdpa_fp64(oracle_mod, B, L, H_q, H_kv, D, causal):
    """O and LSE against the definition with exactly rounded sums at 1e-12, and O against
    the float64 library routine as a second, independent implementation.  The library
    comparison is held to 1e-9: torch's float64 CPU path was once seen 6.8e-10 off the
    exact value, a fault of the library, not of the oracle, which the exact reference
    bounds at 1e-12."""
    q = rnd((B, L, H_q, D), 1, 2.0)
    k = rnd((B, L, H_kv, D), 2)
    v = rnd((B, L, H_kv, D), 3)
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle_mod.attention(q, k, v, scale, causal)
    ex_o, ex_l = exact_attention(q, k, v, scale, causal)
    np.testing.assert_allclose(out, ex_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ex_l, rtol=0, atol=1e-12)
    ref_o, _ = torch_sdpa(q, k, v, scale, causal)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-9)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_constant_scores_give_mean_of_v(oracle_mod, causal):
    B, L, H_q, H_kv, D = 2, 40, 4, 2, 8
    q = np.zeros((B, L, H_q, D))
    k = rnd((B, L, H_kv, D), 5)
    v = rnd((B, L, H_kv, D), 6)
    out, lse = oracle_mod.attention(q, k, v, 0.3, causal)
    for h in range(H_q):
        g = h // (H_q // H_kv)
        for t in range(L):
            n = t + 1 if causal else L
            np.testing.assert_allclose(out[:, t, h], v[:, :n, g].mean(axis=1), atol=1e-13)
            np.testing.assert_allclose(lse[:, h, t], math.log(n), atol=1e-13)


def test_one_dominant_key(oracle_mod):
    B, L, H, D = 1, 24, 2, 4
    q = rnd((B, L, H, D), 7)
    k = rnd((B, L, H, D), 8) * 0.1
    v = rnd((B, L, H, D), 9)
    j = 11
    k[0, j] = 200.0 * q[0, 5]  # row 5's score with key j dominates by a huge margin
    out, lse = oracle_mod.attention(q, k, v, 1.0, False)
    np.testing.assert_allclose(out[0, 5], v[0, j], atol=1e-12)
    s = 200.0 * np.sum(q[0, 5] ** 2, axis=-1)  # per head
    np.testing.assert_allclose(lse[0, :, 5], s, rtol=1e-12)


def test_first_causal_row_is_v0(oracle_mod):
    q, k, v = rnd((2, 16, 4, 8), 10), rnd((2, 16, 2, 8), 11), rnd((2, 16, 2, 8), 12)
    out, lse = oracle_mod.attention(q, k, v, 0.5, True)
    for h in range(4):
        np.testing.assert_allclose(out[:, 0, h], v[:, 0, h // 2], atol=1e-14)
        np.testing.assert_allclose(lse[:, h, 0],
                                   0.5 * np.sum(q[:, 0, h] * k[:, 0, h // 2], -1), atol=1e-14)


def test_causal_row_equals_prefix_attention(oracle_mod):
    q, k, v = rnd((1, 30, 2, 8), 13), rnd((1, 30, 2, 8), 14), rnd((1, 30, 2, 8), 15)
    out, lse = oracle_mod.attention(q, k, v, 0.4, True)
    for t in (0, 7, 29):
        o2, l2 = oracle_mod.attention(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], 0.4, False)
        np.testing.assert_allclose(out[:, t], o2[:, t], atol=1e-13)
        np.testing.assert_allclose(lse[:, :, t], l2[:, :, t], atol=1e-13)


# ---------------------------------------------------------------- brute force
def _decimal_attention(q, k, v, scale, causal):
    getcontext().prec = 50
    B, L, H_q, D = q.shape
    H_kv = k.shape[2]
    out = np.zeros(q.shape)
    lse = np.zeros((B, H_q, L))
    for b in range(B):
        for h in range(H_q):
            g = h // (H_q // H_kv)
            for t in range(L):
                keys = range(t + 1) if causal else range(L)
                s = [Decimal(scale) * sum(Decimal(q[b, t, h, d]) * Decimal(k[b, j, g, d])
                                          for d in range(D)) for j in keys]
                e = [x.exp() for x in s]
                z = sum(e)
                lse[b, h, t] = float(z.ln())
                for d in range(D):
                    out[b, t, h, d] = float(sum(ei * Decimal(v[b, j, g, d])
                                                for ei, j in zip(e, keys)) / z)
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_decimal(oracle_mod, causal):
    q, k, v = rnd((1, 9, 4, 3), 16, 3.0), rnd((1, 9, 2, 3), 17), rnd((1, 9, 2, 3), 18)
    out, lse = oracle_mod.attention(q, k, v, 0.7, causal)
    ref_o, ref_l = _decimal_attention(q, k, v, 0.7, causal)
    np.testing.assert_allclose(out, ref_o, atol=1e-13)
    np.testing.assert_allclose(lse, ref_l, atol=1e-13)


# ---------------------------------------------------------------- invariants
def test_noncausal_invariant_to_joint_kv_permutation(oracle_mod):
    q, k, v = rnd((1, 45, 4, 8), 19), rnd((1, 45, 2, 8), 20), rnd((1, 45, 2, 8), 21)
    perm = np.random.default_rng(22).permutation(45)
    o1, l1 = oracle_mod.attention(q, k, v, 0.3, False)
    o2, l2 = oracle_mod.attention(q, k[:, perm], v[:, perm], 0.3, False)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def _chunks(x, P):
    B, L, H, D = x.shape
    return np.ascontiguousarray(x.reshape(B, P, L // P, H, D).transpose(1, 0, 2, 3, 4))


@pytest.mark.parametrize("P", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_merge_equals_plain_attention(oracle_mod, P, causal):
    """Merging per-chunk partials in ring order gives exactly the unchunked result."""
    L = 16 * 6
    q, k, v = rnd((2, L, 4, 8), 23, 2.0), rnd((2, L, 2, 8), 24), rnd((2, L, 2, 8), 25)
    o_ref, l_ref = oracle_mod.attention(q, k, v, 0.35, causal)
    o, l = oracle_mod.ring_attention(q, _chunks(k, P), _chunks(v, P), 0.35, causal)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, atol=1e-12)


@pytest.mark.parametrize("order", ["reversed", "shuffled"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_order_does_not_matter(oracle_mod, order, causal):
    P, L = 8, 64
    q, k, v = rnd((1, L, 2, 8), 26), rnd((1, L, 2, 8), 27), rnd((1, L, 2, 8), 28)
    offs = list(range(P))[::-1] if order == "reversed" else \
        list(np.random.default_rng(29).permutation(P))
    o_ref, l_ref = oracle_mod.attention(q, k, v, 0.5, causal)
    o, l = oracle_mod.ring_attention(q, _chunks(k, P), _chunks(v, P), 0.5, causal, offs)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, atol=1e-12)


def test_ring_single_rank_is_plain(oracle_mod):
    q, k, v = rnd((1, 20, 2, 4), 30), rnd((1, 20, 1, 4), 31), rnd((1, 20, 1, 4), 32)
    o, l = oracle_mod.ring_attention(q, k[None], v[None], 0.5, True)
    ref_o, ref_l = torch_sdpa(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, ref_o, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, atol=1e-12)


# ---------------------------------------------------------------- zigzag layout
# The pages name ZigZag beside the plain ring ("Метод контекстного параллелизма Ulysses",
# introduction) without describing it; the reading taken: 2P segments of Lc/2 tokens,
# rank i holding segment i then segment 2P-1-i.

def test_zigzag_positions_hand_written(oracle_mod):
    # P=2, Lc=4: segments of 2 tokens {0,1} {2,3} {4,5} {6,7}; rank 0 holds segments 0 and
    # 3, rank 1 holds segments 1 and 2.
    assert list(oracle_mod.zigzag_positions(2, 4)) == [0, 1, 6, 7, 2, 3, 4, 5]
    # P=3, Lc=2: single-token segments 0..5; ranks hold (0,5), (1,4), (2,3).
    assert list(oracle_mod.zigzag_positions(3, 2)) == [0, 5, 1, 4, 2, 3]
    # one rank holds both segments in order: the identity
    assert list(oracle_mod.zigzag_positions(1, 6)) == [0, 1, 2, 3, 4, 5]


@pytest.mark.parametrize("P,Lc", [(1, 2), (2, 6), (4, 8), (5, 10), (8, 256), (16, 2)])
def test_zigzag_positions_are_a_permutation(oracle_mod, P, Lc):
    pos = oracle_mod.zigzag_positions(P, Lc)
    assert sorted(pos.tolist()) == list(range(P * Lc))


@pytest.mark.parametrize("P,Lc", [(2, 4), (4, 8), (8, 64)])
def test_zigzag_balances_causal_work(oracle_mod, P, Lc):
    """Under a causal mask a token at position p sees p+1 keys; zigzag gives every rank
    the same total, h*(2P*h+1) with h = Lc/2, while the contiguous layout does not."""
    h = Lc // 2
    pos = oracle_mod.zigzag_positions(P, Lc).reshape(P, Lc)
    work = (pos + 1).sum(axis=1)
    assert np.all(work == h * (2 * P * h + 1))
    contiguous = (np.arange(P * Lc).reshape(P, Lc) + 1).sum(axis=1)
    assert len(set(contiguous.tolist())) == P


@pytest.mark.parametrize("causal", [False, True])
def test_ring_identity_positions_equal_contiguous(oracle_mod, causal):
    P, L = 4, 48
    q, k, v = rnd((2, L, 4, 8), 60, 2.0), rnd((2, L, 2, 8), 61), rnd((2, L, 2, 8), 62)
    o0, l0 = oracle_mod.ring_attention(q, _chunks(k, P), _chunks(v, P), 0.4, causal)
    o1, l1 = oracle_mod.ring_attention(q, _chunks(k, P), _chunks(v, P), 0.4, causal,
                                       positions=np.arange(L))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


@pytest.mark.parametrize("P,Lc", [(2, 4), (3, 6), (4, 10)])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_zigzag_equals_natural_order_sdpa(oracle_mod, P, Lc, causal):
    """Shards in the zigzag layout: the result of rank-major token R equals the float64
    library attention over the sequence in natural order, at position pos[R]."""
    L = P * Lc
    q, k, v = rnd((2, L, 4, 8), 63, 2.0), rnd((2, L, 2, 8), 64), rnd((2, L, 2, 8), 65)
    pos = oracle_mod.zigzag_positions(P, Lc)
    o, l = oracle_mod.ring_attention_zigzag(q, _chunks(k, P), _chunks(v, P), 0.4, causal)
    nat = np.empty(L, np.int64)
    nat[pos] = np.arange(L)  # rank-major index of each natural position
    ref_o, ref_l = torch_sdpa(q[:, nat], k[:, nat], v[:, nat], 0.4, causal)
    np.testing.assert_allclose(o, ref_o[:, pos], atol=1e-12)
    np.testing.assert_allclose(l, ref_l[:, :, pos], atol=1e-12)


def test_ring_positions_must_be_a_permutation(oracle_mod):
    q, k, v = rnd((1, 8, 2, 4), 66), rnd((1, 8, 2, 4), 67), rnd((1, 8, 2, 4), 68)
    with pytest.raises(ValueError):
        oracle_mod.ring_attention(q, _chunks(k, 2), _chunks(v, 2), 0.5, True,
                                  positions=[0, 1, 2, 3, 4, 5, 6, 6])
    with pytest.raises(ValueError):
        oracle_mod.zigzag_positions(2, 3)  # odd chunk length


# ---------------------------------------------------------------- packed samples
# "Paralelismo de secuencias en 🤗 accelerate", section "Configuración del backend SP de
# ALST/Ulysses": sequence parallelism is driven by position_ids and several samples may be
# combined into one sequence; reading: samples are contiguous, position_ids count
# 0, 1, 2, ... within each, and attention stays inside a sample.

def _pid_from_lengths(lengths):
    return np.concatenate([np.arange(n) for n in lengths])


def test_packed_lower_bounds_hand_written(oracle_mod):
    lo = oracle_mod.packed_lower_bounds(np.array([[0, 1, 2, 0, 1, 0, 0, 1]]))
    assert lo.tolist() == [[0, 0, 0, 3, 3, 5, 6, 6]]
    with pytest.raises(ValueError):
        oracle_mod.packed_lower_bounds(np.array([[0, 2, 3]]))  # skips a position
    with pytest.raises(ValueError):
        oracle_mod.packed_lower_bounds(np.array([[1, 2, 3]]))  # does not start a sample


@pytest.mark.parametrize("P", [1, 3, 4])
def test_packed_equals_independent_samples_sdpa(oracle_mod, P):
    """Each packed sample's rows equal float64 library causal attention over that sample
    alone; two batch rows packed differently."""
    L = 60
    lengths = [[7, 1, 20, 32], [60]] if P != 3 else [[13, 13, 34], [1, 1, 58]]
    pid = np.stack([_pid_from_lengths(x) for x in lengths])
    q, k, v = rnd((2, L, 4, 8), 70, 2.0), rnd((2, L, 2, 8), 71), rnd((2, L, 2, 8), 72)
    o, l = oracle_mod.ring_attention_packed(q, _chunks(k, P), _chunks(v, P), 0.4, pid)
    for b in range(2):
        s0 = 0
        for n in lengths[b]:
            sl = slice(s0, s0 + n)
            ro, rl = torch_sdpa(q[b:b + 1, sl], k[b:b + 1, sl], v[b:b + 1, sl], 0.4, True)
            np.testing.assert_allclose(o[b, sl], ro[0], atol=1e-12)
            np.testing.assert_allclose(l[b, :, sl], rl[0], atol=1e-12)
            s0 += n


def test_packed_single_sample_is_causal_ring(oracle_mod):
    L, P = 48, 4
    q, k, v = rnd((1, L, 2, 8), 73), rnd((1, L, 1, 8), 74), rnd((1, L, 1, 8), 75)
    o0, l0 = oracle_mod.ring_attention(q, _chunks(k, P), _chunks(v, P), 0.5, True)
    o1, l1 = oracle_mod.ring_attention_packed(q, _chunks(k, P), _chunks(v, P), 0.5,
                                              np.arange(L)[None])
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_packed_one_token_samples_closed_form(oracle_mod):
    """Every token its own sample: each query sees only its own key, so O = v and
    LSE = scale * q.k (GQA: query head h reads kv head h // 2)."""
    L, P = 16, 2
    q, k, v = rnd((1, L, 4, 8), 76), rnd((1, L, 2, 8), 77), rnd((1, L, 2, 8), 78)
    o, l = oracle_mod.ring_attention_packed(q, _chunks(k, P), _chunks(v, P), 0.3,
                                            np.zeros((1, L), np.int64))
    kv_head = np.arange(4) // 2
    np.testing.assert_allclose(o[0], v[0][:, kv_head], atol=1e-14)
    want_l = 0.3 * np.einsum("thd,thd->ht", q[0], k[0][:, kv_head])
    np.testing.assert_allclose(l[0], want_l, atol=1e-13)


def test_attention_rows_sample(oracle_mod):
    q, k, v = rnd((2, 40, 4, 8), 33), rnd((2, 40, 2, 8), 34), rnd((2, 40, 2, 8), 35)
    rb, rt, rh = [0, 1, 1, 0], [0, 39, 17, 5], [3, 0, 2, 1]
    o, l = oracle_mod.attention_rows(q[rb, rt, rh], rb, rt, rh, k, v, 4, 0.3, True)
    ref_o, ref_l = torch_sdpa(q, k, v, 0.3, True)
    np.testing.assert_allclose(o, ref_o[rb, rt, rh], atol=1e-12)
    np.testing.assert_allclose(l, ref_l[rb, rh, rt], atol=1e-12)


def test_invalid_arguments_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.seq2head(np.zeros((2, 1, 4, 3, 8)), 3)  # 3 heads over 2 ranks
    with pytest.raises(ValueError):
        oracle_mod.attention_rows(np.zeros((1, 4)), [0], [99], [0], np.zeros((1, 8, 1, 4)),
                                  np.zeros((1, 8, 1, 4)), 1, 1.0, False)


# ---------------------------------------------------------------- merge
def test_merge_of_key_halves_equals_whole(oracle_mod):
    """Attention over keys [0,m) merged with attention over [m,L) is attention over [0,L)."""
    q, k, v = rnd((2, 33, 4, 8), 36, 2.0), rnd((2, 33, 4, 8), 37), rnd((2, 33, 4, 8), 38)
    m = 13
    o_full, l_full = oracle_mod.attention(q, k, v, 0.4, False)
    oa, la = _attend_subset(oracle_mod, q, k, v, 0.4, 0, m)
    ob, lb = _attend_subset(oracle_mod, q, k, v, 0.4, m, 33)
    o, l = oracle_mod.lse_merge(oa, la, ob, lb)
    np.testing.assert_allclose(o, o_full, atol=1e-12)
    np.testing.assert_allclose(l, l_full, atol=1e-12)


def _attend_subset(oracle_mod, q, k, v, scale, lo, hi):
    """Attention of every query row against keys [lo, hi) only, via attention_rows."""
    B, L, H, D = q.shape
    rb, rt, rh = np.meshgrid(np.arange(B), np.arange(L), np.arange(H), indexing="ij")
    rb, rt, rh = rb.ravel(), rt.ravel(), rh.ravel()
    o, l = oracle_mod.attention_rows(q[rb, rt, rh], rb, np.zeros_like(rt), rh,
                                     k[:, lo:hi], v[:, lo:hi], H, scale, False)
    return o.reshape(B, L, H, D), l.reshape(B, L, H).transpose(0, 2, 1).copy()


def test_merge_identities(oracle_mod):
    B, L, H, D = 1, 6, 2, 4
    oa, ob = rnd((B, L, H, D), 39), rnd((B, L, H, D), 40)
    la, lb = rnd((B, H, L), 41), rnd((B, H, L), 42)
    ninf = np.full((B, H, L), -np.inf)
    # (x) (+) empty = x, empty (+) (x) = x
    o, l = oracle_mod.lse_merge(oa, la, np.zeros_like(ob), ninf)
    np.testing.assert_array_equal(o, oa)
    np.testing.assert_array_equal(l, la)
    o, l = oracle_mod.lse_merge(np.zeros_like(oa), ninf, ob, lb)
    np.testing.assert_array_equal(o, ob)
    np.testing.assert_array_equal(l, lb)
    # empty (+) empty = (0, -inf), no NaN
    o, l = oracle_mod.lse_merge(oa, ninf, ob, ninf)
    assert np.all(o == 0) and np.all(l == -np.inf)
    # equal lse: the average, lse + ln 2
    o, l = oracle_mod.lse_merge(oa, la, ob, la)
    np.testing.assert_allclose(o, 0.5 * (oa + ob), atol=1e-15)
    np.testing.assert_allclose(l, la + math.log(2), atol=1e-15)
    # weights e^(la-l), e^(lb-l) with l = log(e^la + e^lb): closed form for lb = la + ln 3
    o, l = oracle_mod.lse_merge(oa, la, ob, la + math.log(3))
    np.testing.assert_allclose(o, 0.25 * oa + 0.75 * ob, atol=1e-14)
    np.testing.assert_allclose(l, la + math.log(4), atol=1e-14)
    # commutative
    o1, l1 = oracle_mod.lse_merge(oa, la, ob, lb)
    o2, l2 = oracle_mod.lse_merge(ob, lb, oa, la)
    np.testing.assert_allclose(o1, o2, atol=1e-15)
    np.testing.assert_allclose(l1, l2, atol=1e-15)


def test_merge_large_lse_no_overflow(oracle_mod):
    oa, ob = np.ones((1, 1, 1, 4)), 3 * np.ones((1, 1, 1, 4))
    o, l = oracle_mod.lse_merge(oa, np.array([[[1000.0]]]), ob, np.array([[[1000.0]]]))
    np.testing.assert_allclose(o, 2 * np.ones((1, 1, 1, 4)))
    np.testing.assert_allclose(l, 1000 + math.log(2))


# ---------------------------------------------------------------- Ulysses permute
def _golden_ulysses():
    cases = {}
    for line in open(os.path.join(GOLDEN, "ulysses_tiny.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        head, vals = line.split(":")
        case, h_in, h_out, r = head.split()
        cases.setdefault((case, int(h_in), int(h_out)), {})[int(r)] = [int(x) for x in vals.split()]
    return cases


def test_seq2head_golden(oracle_mod):
    P, Lc = 2, 2
    for (case, H_in, H_out), per_rank in _golden_ulysses().items():
        x = np.zeros((P, 1, Lc, H_in, 1), np.int32)
        for s in range(P):
            for t in range(Lc):
                for h in range(H_in):
                    x[s, 0, t, h, 0] = 100 * s + 10 * t + h
        y = oracle_mod.seq2head(x, H_out)
        assert y.shape == (P, 1, P * Lc, H_out // P, 1)
        for r, vals in per_rank.items():
            assert y[r].ravel().tolist() == vals, (case, r)


@pytest.mark.parametrize("dtype", [np.float32, np.uint16, np.float64])
def test_seq2head_head2seq_round_trip(oracle_mod, dtype):
    P, B, Lc, H, D = 4, 2, 6, 8, 5
    x = (np.random.default_rng(43).integers(0, 60000, (P, B, Lc, H, D))).astype(dtype)
    y = oracle_mod.seq2head(x, H)
    assert y.size == x.size  # memory unchanged by the transform
    z = oracle_mod.head2seq(y)
    assert z.dtype == x.dtype and np.array_equal(z, x)


def test_seq2head_is_a_permutation_of_elements(oracle_mod):
    P, B, Lc, H, D = 4, 1, 3, 4, 2
    x = np.arange(P * B * Lc * H * D, dtype=np.int64).reshape(P, B, Lc, H, D)
    y = oracle_mod.seq2head(x, H)
    assert sorted(y.ravel().tolist()) == list(range(x.size))


def test_seq2head_gqa_replicas_copy_their_source(oracle_mod):
    P, B, Lc, H_in, H_out, D = 8, 1, 5, 4, 8, 3
    x = np.random.default_rng(44).standard_normal((P, B, Lc, H_in, D))
    y = oracle_mod.seq2head(x, H_out)  # [P, B, P*Lc, 1, D]
    glob = x.transpose(1, 0, 2, 3, 4).reshape(B, P * Lc, H_in, D)
    for r in range(P):
        np.testing.assert_array_equal(y[r, :, :, 0], glob[:, :, (r * H_in) // H_out])
    # each replicated rank pair then sees the kv head its query-head block needs:
    # with 32 query heads on 8 ranks, rank r's heads 4r..4r+3 use kv head (4r)//(32//4)
    for r in range(P):
        assert (r * H_in) // H_out == (4 * r) // (32 // H_in)


# ---------------------------------------------------------------- head groups and the USP hybrid
# The Ulysses transform with G head groups (G = P is Ulysses itself; G < P is the head split
# of the ring x Ulysses hybrid, "Paralelismo de secuencias en 🤗 accelerate" naming USP and
# "Как работает sequence parallelism в контексте LLM?" section 3 the ring over the rest).

def test_seq2head_one_group_concatenates_shards(oracle_mod):
    """G = 1: the single head group receives every shard's tokens in rank order, all heads."""
    P, B, Lc, H, D = 3, 2, 4, 5, 2
    x = np.random.default_rng(80).standard_normal((P, B, Lc, H, D))
    y = oracle_mod.seq2head(x, H, groups=1)
    assert y.shape == (1, B, P * Lc, H, D)
    np.testing.assert_array_equal(y[0], x.transpose(1, 0, 2, 3, 4).reshape(B, P * Lc, H, D))


def test_seq2head_groups_hand_written(oracle_mod):
    # P = 2 shards of 2 tokens, 4 heads, G = 2 groups of 2 heads; value = 100 s + 10 t + h
    x = np.zeros((2, 1, 2, 4, 1), np.int32)
    for s in range(2):
        for t in range(2):
            for h in range(4):
                x[s, 0, t, h, 0] = 100 * s + 10 * t + h
    y = oracle_mod.seq2head(x, 4, groups=2)
    # group 0: heads 0,1 of tokens (s,t) = (0,0),(0,1),(1,0),(1,1)
    assert y[0].ravel().tolist() == [0, 1, 10, 11, 100, 101, 110, 111]
    assert y[1].ravel().tolist() == [2, 3, 12, 13, 102, 103, 112, 113]


@pytest.mark.parametrize("P,G", [(4, 2), (6, 3), (6, 2), (3, 1), (4, 4), (2, 4)])
def test_grouped_round_trip(oracle_mod, P, G):
    B, Lc, H, D = 2, 3, 8 if G != 3 else 6, 3
    x = np.random.default_rng(81).integers(0, 1 << 30, (P, B, Lc, H, D)).astype(np.int64)
    y = oracle_mod.seq2head(x, H, groups=G)
    assert y.shape == (G, B, P * Lc, H // G, D)
    np.testing.assert_array_equal(oracle_mod.head2seq(y, P=P), x)


@pytest.mark.parametrize("P,P_u", [(4, 2), (6, 3), (4, 4), (4, 1), (8, 2)])
@pytest.mark.parametrize("causal", [False, True])
def test_usp_equals_natural_order_sdpa(oracle_mod, P, P_u, causal):
    """Ring x Ulysses over P shards (P_u head groups, GQA 4:2 with the KV copy) equals the
    float64 library attention over the whole sequence."""
    B, Ls, H_kv, D = 2, 5, 2, 8
    H_q = 6 if P_u == 3 else 4
    rng = np.random.default_rng(82 + P * 10 + P_u)
    q = rng.standard_normal((P, B, Ls, H_q, D)) * 2.0
    k = rng.standard_normal((P, B, Ls, H_kv, D))
    v = rng.standard_normal((P, B, Ls, H_kv, D))
    o, l = oracle_mod.usp_attention(q, k, v, P_u, 0.4, causal)
    seq = lambda x: x.transpose(1, 0, 2, 3, 4).reshape(B, P * Ls, x.shape[3], D)
    ref_o, ref_l = torch_sdpa(seq(q), seq(k), seq(v), 0.4, causal)
    np.testing.assert_allclose(seq(o), ref_o, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, atol=1e-12)


# ---------------------------------------------------------------- backward
# The gradients of O = softmax(scale Q K^T) V (the pages train with ring attention but give
# no backward formula; the oracle writes out the derivative of the definition).

def _torch_grads(q, k, v, dout, scale, causal):
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True)
                  for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale,
                                                           is_causal=causal, enable_gqa=True)
    out.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    return [t.grad.permute(0, 2, 1, 3).numpy() for t in (tq, tk, tv)]


@pytest.mark.parametrize("B,L,H_q,H_kv,D,causal", [(1, 9, 2, 2, 4, True), (2, 17, 4, 2, 8, True),
                                                   (1, 12, 6, 3, 8, False), (2, 5, 4, 1, 16, True)])
def test_backward_matches_torch_autograd_fp64(oracle_mod, B, L, H_q, H_kv, D, causal):
    q, k, v = rnd((B, L, H_q, D), 90, 1.5), rnd((B, L, H_kv, D), 91), rnd((B, L, H_kv, D), 92)
    dout = rnd((B, L, H_q, D), 93)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, dout, 0.37, causal)
    rq, rk, rv = _torch_grads(q, k, v, dout, 0.37, causal)
    np.testing.assert_allclose(dq, rq, atol=1e-12)
    np.testing.assert_allclose(dk, rk, atol=1e-12)
    np.testing.assert_allclose(dv, rv, atol=1e-12)


def test_backward_matches_finite_differences(oracle_mod):
    """Central differences of sum(O * dO) through the forward oracle (no library)."""
    B, L, H_q, H_kv, D = 1, 6, 2, 1, 3
    q, k, v = rnd((B, L, H_q, D), 94), rnd((B, L, H_kv, D), 95), rnd((B, L, H_kv, D), 96)
    dout = rnd((B, L, H_q, D), 97)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, dout, 0.8, True)
    loss = lambda q_, k_, v_: float(np.sum(oracle_mod.attention(q_, k_, v_, 0.8, True)[0] * dout))
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            pa = [xp if a is x else a for a in args]
            ma = [xm if a is x else a for a in args]
            fd = (loss(*pa) - loss(*ma)) / (2 * eps)
            assert abs(fd - g[idx]) < 1e-7, (name, idx, fd, g[idx])


# ---------------------------------------------------------------- backward on sampled rows
def _torch_grads_masked(q, k, v, dout, scale, visible):
    """float64 library gradients of attention under an explicit boolean mask
    visible [B, L_query, L_key] (True = attended)."""
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True)
                  for x in (q, k, v))
    mask = torch.from_numpy(visible)[:, None]
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                           scale=scale, enable_gqa=True)
    out.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    return [t.grad.permute(0, 2, 1, 3).numpy() for t in (tq, tk, tv)]


def _visible(B, L, causal, pos, lo):
    p = np.arange(L) if pos is None else np.asarray(pos)
    low = np.zeros((B, L), np.int64) if lo is None else np.asarray(lo)
    vis = np.ones((B, L, L), bool)
    if causal:
        vis &= p[None, None, :] <= p[None, :, None]
    vis &= p[None, None, :] >= low[:, :, None]
    return vis


def _sample(B, L, H, n, seed):
    g = np.random.default_rng(seed)
    return (g.integers(0, B, n), g.integers(0, L, n), g.integers(0, H, n))


@pytest.mark.parametrize("layout", ["contiguous", "noncausal", "zigzag", "permuted", "packed"])
def test_backward_rows_match_torch_autograd_masked(oracle_mod, layout):
    """dQ, dK, dV of sampled rows against float64 library autograd under the explicit mask
    that the positions and lower bounds define: contiguous causal and non-causal, the
    zigzag layout (P = 3, Lc = 10), an arbitrary permutation of positions, and packed
    samples (GQA 4:2, B = 2)."""
    B, P, Lc, H_q, H_kv, D = 2, 3, 10, 4, 2, 8
    L = P * Lc
    q, k, v = rnd((B, L, H_q, D), 120, 1.5), rnd((B, L, H_kv, D), 121), rnd((B, L, H_kv, D), 122)
    dout = rnd((B, L, H_q, D), 123)
    causal, pos, lo = layout != "noncausal", None, None
    if layout == "zigzag":
        pos = oracle_mod.zigzag_positions(P, Lc)
    elif layout == "permuted":
        pos = np.random.default_rng(5).permutation(L)
    elif layout == "packed":
        pid = np.stack([_pid_from_lengths([1, 9, 4, 16]), _pid_from_lengths([30])])
        lo = oracle_mod.packed_lower_bounds(pid)
    rq, rk, rv = _torch_grads_masked(q, k, v, dout, 0.45, _visible(B, L, causal, pos, lo))
    qr, kr = _sample(B, L, H_q, 40, 7), _sample(B, L, H_kv, 30, 8)
    dq, dk, dv = oracle_mod.attention_backward_rows(q, k, v, dout, 0.45, causal, qr, kr,
                                                    positions=pos, lower_bounds=lo)
    np.testing.assert_allclose(dq, rq[qr[0], qr[1], qr[2]], atol=1e-12)
    np.testing.assert_allclose(dk, rk[kr[0], kr[1], kr[2]], atol=1e-12)
    np.testing.assert_allclose(dv, rv[kr[0], kr[1], kr[2]], atol=1e-12)


def test_backward_rows_equal_every_row_backward(oracle_mod):
    """Every row sampled: the same numbers as the full backward (same formulas, same order
    of summation), causal GQA."""
    B, L, H_q, H_kv, D = 1, 23, 4, 1, 8
    q, k, v = rnd((B, L, H_q, D), 124), rnd((B, L, H_kv, D), 125), rnd((B, L, H_kv, D), 126)
    dout = rnd((B, L, H_q, D), 127)
    full = oracle_mod.attention_backward(q, k, v, dout, 0.3, True)
    qr = [a.ravel() for a in np.meshgrid(np.arange(B), np.arange(L), np.arange(H_q), indexing="ij")]
    kr = [a.ravel() for a in np.meshgrid(np.arange(B), np.arange(L), np.arange(H_kv), indexing="ij")]
    dq, dk, dv = oracle_mod.attention_backward_rows(q, k, v, dout, 0.3, True, qr, kr)
    np.testing.assert_allclose(dq, full[0][qr[0], qr[1], qr[2]], atol=1e-13)
    np.testing.assert_allclose(dk, full[1][kr[0], kr[1], kr[2]], atol=1e-13)
    np.testing.assert_allclose(dv, full[2][kr[0], kr[1], kr[2]], atol=1e-13)


def test_backward_rows_closed_forms(oracle_mod):
    """One-token packed samples: each query sees only its own key, P = 1, so dQ = dK = 0 and
    dV of key t is the sum of dO over the query heads of its group."""
    B, L, H_q, H_kv, D = 1, 12, 4, 2, 8
    q, k, v = rnd((B, L, H_q, D), 128), rnd((B, L, H_kv, D), 129), rnd((B, L, H_kv, D), 130)
    dout = rnd((B, L, H_q, D), 131)
    lo = np.arange(L)[None].astype(np.int64)
    qr, kr = _sample(B, L, H_q, 10, 9), _sample(B, L, H_kv, 10, 10)
    dq, dk, dv = oracle_mod.attention_backward_rows(q, k, v, dout, 0.7, True, qr, kr,
                                                    lower_bounds=lo)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)
    want = dout[kr[0], kr[1], 2 * kr[2]] + dout[kr[0], kr[1], 2 * kr[2] + 1]
    np.testing.assert_allclose(dv, want, atol=1e-14)


def test_backward_rows_invalid_arguments(oracle_mod):
    z = np.zeros((1, 4, 2, 8))
    with pytest.raises(ValueError):
        oracle_mod.attention_backward_rows(z, z, z, z, 1.0, True, ([0], [4], [0]), ([], [], []))
    with pytest.raises(ValueError):
        oracle_mod.attention_backward_rows(z, z, z, z, 1.0, True, ([], [], []), ([0], [0], [2]))
    with pytest.raises(ValueError):
        oracle_mod.attention_backward_rows(z, z, z, z, 1.0, True, ([0], [0], [0]), ([], [], []),
                                           positions=[0, 1, 1, 3])


# ---------------------------------------------------------------- one ring step's gradients
# The ring backward reuses the forward's final LSE ("Как работает sequence parallelism в
# контексте LLM?", section 5, taken to the gradient): each step's share is pinned by summing
# the shares of every chunk pair and comparing with the whole-sequence gradients (pinned
# against torch autograd above), by the one-chunk case, and by a closed form.

def _pair_shares(oracle_mod, q, k, v, dout, P, scale, causal):
    """Sum over every (query chunk i, key chunk j) pair of the oracle's one-step shares, with
    the whole sequence's out / lse; causal pairs: j < i whole, j == i causal, j > i none."""
    B, L, H_q, D = q.shape
    Lc = L // P
    out, lse = oracle_mod.attention(q, k, v, scale, causal)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for i in range(P):
        qi = slice(i * Lc, (i + 1) * Lc)
        for j in range(P):
            if causal and j > i:
                continue
            kj = slice(j * Lc, (j + 1) * Lc)
            a, b_, c = oracle_mod.attention_backward_pair(
                q[:, qi], k[:, kj], v[:, kj], out[:, qi], lse[:, :, qi], dout[:, qi], scale,
                causal and j == i)
            dq[:, qi] += a
            dk[:, kj] += b_
            dv[:, kj] += c
    return dq, dk, dv


@pytest.mark.parametrize("P,causal", [(1, True), (3, True), (4, False), (3, False)])
def test_backward_pair_shares_sum_to_whole_sequence(oracle_mod, P, causal):
    B, Lc, H_q, H_kv, D = 2, 5, 4, 2, 8
    L = P * Lc
    q, k, v = rnd((B, L, H_q, D), 110, 1.5), rnd((B, L, H_kv, D), 111), rnd((B, L, H_kv, D), 112)
    dout = rnd((B, L, H_q, D), 113)
    got = _pair_shares(oracle_mod, q, k, v, dout, P, 0.41, causal)
    want = oracle_mod.attention_backward(q, k, v, dout, 0.41, causal)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, atol=1e-12)


def test_backward_pair_one_query_one_key_closed_form(oracle_mod):
    """One query, one key: P = 1, so dS = dO.v - dO.O = 0 (O = v): dq = dk = 0, dv = dO."""
    q, k, v = rnd((1, 1, 2, 4), 114), rnd((1, 1, 1, 4), 115), rnd((1, 1, 1, 4), 116)
    dout = rnd((1, 1, 2, 4), 117)
    out, lse = oracle_mod.attention(q, k, v, 0.7, True)
    dq, dk, dv = oracle_mod.attention_backward_pair(q, k, v, out, lse, dout, 0.7, True)
    assert np.abs(dq).max() < 1e-15 and np.abs(dk).max() < 1e-15
    np.testing.assert_allclose(dv[0, 0, 0], dout[0, 0].sum(axis=0), atol=1e-15)


def test_backward_pair_rejects_causal_between_unequal_chunks(oracle_mod):
    z, zl = np.zeros((1, 4, 2, 8)), np.zeros((1, 2, 4))
    with pytest.raises(ValueError):
        oracle_mod.attention_backward_pair(z, np.zeros((1, 3, 2, 8)), np.zeros((1, 3, 2, 8)), z,
                                           zl, z, 1.0, True)


# ---------------------------------------------------------------- the GQA copy's gradient
def test_replica_sum_is_the_adjoint_of_the_copy(oracle_mod):
    """<copy(x), y> = <x, replica_sum(y)> for the repeat-interleave copy of seq->head (numpy's
    repeat as the copy), so replica_sum is the copy's transpose: the gradient rule."""
    x = rnd((3, 5, 2, 8), 120)
    y = rnd((3, 5, 6, 8), 121)
    copy = np.repeat(x, 3, axis=2)  # replica j of head j // 3
    lhs = float(np.sum(copy * y))
    rhs = float(np.sum(x * oracle_mod.replica_sum(y, 2)))
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))


def test_replica_sum_closed_forms(oracle_mod):
    y = rnd((2, 4, 3, 4), 122)
    np.testing.assert_array_equal(oracle_mod.replica_sum(y, 3), y)      # one replica each
    c = np.full((2, 4, 8, 4), 0.25)
    np.testing.assert_array_equal(oracle_mod.replica_sum(c, 2), np.full((2, 4, 2, 4), 1.0))
    h = np.arange(2 * 4 * 1, dtype=np.float64).reshape(1, 1, 8, 1)      # heads 0..7, 2 groups
    np.testing.assert_array_equal(oracle_mod.replica_sum(h, 2).ravel(), [0 + 1 + 2 + 3, 4 + 5 + 6 + 7])
    with pytest.raises(ValueError):
        oracle_mod.replica_sum(rnd((1, 1, 6, 4), 123), 4)
