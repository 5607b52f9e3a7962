"""GPU parity of the Ulysses transforms: bit-exact against the oracle's index loops.

Source: "Метод контекстного параллелизма Ulysses" (seq-sharded [local_seqlen,
global_heads, head_dim] <-> head-sharded [global_seqlen, local_heads, head_dim], KV heads
copied up under GQA)."""
import numpy as np
import pytest
import torch

from sequence_parallelism_attn_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    """The raw bits of a tensor (uint16 for bf16, uint32 for fp32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.int32).numpy().view(np.uint32)


@pytest.mark.parametrize("P,B,Lc,H_in,H_out,D,dtype", [
    (2, 1, 64, 2, 2, 32, torch.float32),       # the tiny fp32 workload
    (4, 1, 1024, 8, 8, 64, torch.bfloat16),    # [4 x 1024, 8, 64] -> [4096, 2/rank, 64]
    (8, 1, 1000, 4, 8, 128, torch.bfloat16),   # GQA copy: 4 kv heads over 8 ranks
    (4, 2, 37, 8, 8, 64, torch.bfloat16),      # ragged token count, B > 1
    (2, 3, 5, 2, 4, 8, torch.bfloat16),        # 16-byte heads (one vector): unvectorised path
    (3, 2, 11, 3, 6, 32, torch.float32),       # odd rank count, replication 2
    (1, 1, 9, 4, 4, 64, torch.bfloat16),       # one rank: identity layout
    (8, 1, 16, 1, 8, 128, torch.bfloat16),     # one kv head copied to every rank
])
def test_seq2head_bit_exact(ra_lib, oracle_mod, P, B, Lc, H_in, H_out, D, dtype):
    g = torch.Generator().manual_seed(P * 1000 + Lc)
    x = torch.randn(P, B, Lc, H_in, D, generator=g).to(dtype)
    y = ra_lib.ra_ulysses_seq2head(x.cuda(), H_out)
    torch.cuda.synchronize()
    want = oracle_mod.seq2head(_bits(x), H_out)
    assert np.array_equal(_bits(y), want)


@pytest.mark.parametrize("P,B,Lc,H,D,dtype", [
    (2, 1, 64, 2, 32, torch.float32), (4, 1, 1024, 8, 64, torch.bfloat16),
    (4, 2, 37, 8, 64, torch.bfloat16), (2, 3, 5, 4, 8, torch.bfloat16),
    (3, 2, 11, 6, 32, torch.float32), (8, 1, 300, 32, 128, torch.bfloat16)])
def test_head2seq_bit_exact(ra_lib, oracle_mod, P, B, Lc, H, D, dtype):
    g = torch.Generator().manual_seed(P * 7 + Lc)
    x = torch.randn(P, B, P * Lc, H // P, D, generator=g).to(dtype)
    y = ra_lib.ra_ulysses_head2seq(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), oracle_mod.head2seq(_bits(x)))


def test_round_trip_is_identity(ra_lib):
    w = synth.SMALL_PERMUTE
    q, _, _ = synth.ulysses_inputs(w)
    x = q.cuda()
    z = ra_lib.ra_ulysses_head2seq(ra_lib.ra_ulysses_seq2head(x))
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.int16), x.view(torch.int16))


def test_full_size_ulysses_transforms_bit_exact(ra_lib, oracle_mod):
    """The 128k-token Ulysses workload: Q [8 x 16384, 32, 128] and the GQA copy of
    K [8 x 16384, 4 -> 8, 128], each against the oracle over every element."""
    w = synth.ULYSSES_128K
    q, k, _ = synth.ulysses_inputs(w)
    for x, h_out in ((q, w.H_q), (k, w.H_kv_rep)):
        y = ra_lib.ra_ulysses_seq2head(x.cuda(), h_out)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(y), oracle_mod.seq2head(_bits(x), h_out))
        del y
    yq = oracle_mod.seq2head(_bits(q), w.H_q)
    back = ra_lib.ra_ulysses_head2seq(
        torch.from_numpy(yq.view(np.int16)).view(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_bits(back), _bits(q))


@pytest.mark.parametrize("lead,H_in,H_out,D", [((2, 300), 8, 2, 128), ((1, 1000), 6, 3, 64),
                                               ((3, 7), 4, 4, 32), ((1, 4096), 32, 1, 128)])
def test_replica_sum_matches_oracle(ra_lib, oracle_mod, lead, H_in, H_out, D):
    """The GQA copy's gradient (each head the sum of its replicas) against the oracle's fp64
    sum: every element within the rounding of an fp32 sum of rep terms, (rep - 1) 2^-24
    times the sum of their magnitudes; two calls give the same bits."""
    g = torch.Generator().manual_seed(sum(lead) + H_in)
    x = torch.randn(*lead, H_in, D, generator=g)
    got = ra_lib.ra_ulysses_replica_sum(x.cuda(), H_out)
    again = ra_lib.ra_ulysses_replica_sum(x.cuda(), H_out)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    assert torch.equal(got, again)
    want = oracle_mod.replica_sum(x.double().numpy(), H_out)
    rep = H_in // H_out
    mag = np.abs(x.double().numpy()).reshape(*lead, H_out, rep, D).sum(axis=-2)
    err = np.abs(got.double().cpu().numpy() - want)
    assert np.all(err <= (rep - 1) * 2.0 ** -24 * mag + 1e-30), float((err - (rep - 1) * 2.0 ** -24 * mag).max())



# ------------------------------------------------------------------ one kernel per rank's share
# ra_ulysses_*_scatter: every virtual rank of P stores its share of the all-to-all straight
# into the P destination buffers (separate allocations here; the peers' buffers across
# GPUs).  Each launch only stores, so the P launches need no ordering between them.
SCATTER_CASES = [
    (2, 1, 64, 2, 2, 32, torch.float32),
    (4, 1, 1024, 8, 8, 64, torch.bfloat16),
    (8, 1, 1000, 4, 8, 128, torch.bfloat16),   # GQA copy
    (4, 2, 37, 8, 8, 64, torch.bfloat16),      # ragged, B > 1
    (2, 3, 5, 2, 4, 8, torch.bfloat16),        # one vector per head: unvectorised path
    (3, 2, 11, 3, 6, 32, torch.float32),       # odd rank count
    (1, 1, 9, 4, 4, 64, torch.bfloat16),       # one rank
    (8, 1, 16, 1, 8, 128, torch.bfloat16),     # one kv head copied to every rank
]


@pytest.mark.parametrize("P,B,Lc,H_in,H_out,D,dtype", SCATTER_CASES)
def test_seq2head_scatter_bit_exact(ra_lib, oracle_mod, P, B, Lc, H_in, H_out, D, dtype):
    g = torch.Generator().manual_seed(P * 31 + Lc)
    x = torch.randn(P, B, Lc, H_in, D, generator=g).to(dtype)
    xc = x.cuda()
    Hl = H_out // P
    dst = [torch.full((B, P * Lc, Hl, D), float("nan"), dtype=dtype, device="cuda")
           for _ in range(P)]
    for s in range(P):
        ra_lib.ra_ulysses_seq2head_scatter(xc[s], [d.data_ptr() for d in dst], s, H_out)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    want = oracle_mod.seq2head(_bits(x), H_out)      # [P][B][P*Lc][Hl][D]
    for r in range(P):
        assert np.array_equal(_bits(dst[r]), want[r]), f"rank {r}'s buffer"


@pytest.mark.parametrize("P,B,Lc,H,D,dtype", [
    (2, 1, 64, 2, 32, torch.float32), (4, 1, 1024, 8, 64, torch.bfloat16),
    (4, 2, 37, 8, 64, torch.bfloat16), (2, 3, 5, 4, 8, torch.bfloat16),
    (3, 2, 11, 6, 32, torch.float32), (8, 1, 300, 32, 128, torch.bfloat16),
    (1, 1, 9, 4, 64, torch.bfloat16)])
def test_head2seq_scatter_bit_exact(ra_lib, oracle_mod, P, B, Lc, H, D, dtype):
    g = torch.Generator().manual_seed(P * 17 + Lc)
    x = torch.randn(P, B, P * Lc, H // P, D, generator=g).to(dtype)
    xc = x.cuda()
    dst = [torch.full((B, Lc, H, D), float("nan"), dtype=dtype, device="cuda") for _ in range(P)]
    for r in range(P):
        ra_lib.ra_ulysses_head2seq_scatter(xc[r], [d.data_ptr() for d in dst], r)
    assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
    want = oracle_mod.head2seq(_bits(x))               # [P][B][Lc][H][D]
    for s in range(P):
        assert np.array_equal(_bits(dst[s]), want[s]), f"rank {s}'s shard"


def test_scatter_full_size_matches_the_permutes(ra_lib):
    """The Ulysses workload at its full size (8 ranks x 16384 tokens, Q with 32 heads, K with
    4 heads copied to 8): every virtual rank's scatter gives the bits of the whole-tensor
    seq2head, and the head2seq scatter of the result gives the input back."""
    w = synth.ULYSSES_128K
    q, k, _ = synth.ulysses_inputs(w)
    for x, H_out in ((q.cuda(), w.H_q), (k.cuda(), w.H_kv_rep)):
        P, B, Lc, H_in, D = x.shape
        ref = ra_lib.ra_ulysses_seq2head(x, H_out)
        dst = torch.empty_like(ref)
        ptrs = [dst[r].data_ptr() for r in range(P)]
        for s in range(P):
            ra_lib.ra_ulysses_seq2head_scatter(x[s], ptrs, s, H_out)
        assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
        assert torch.equal(dst.view(torch.int16), ref.view(torch.int16))
        if H_out == H_in:
            back = torch.empty_like(x)
            bptrs = [back[s].data_ptr() for s in range(P)]
            for r in range(P):
                ra_lib.ra_ulysses_head2seq_scatter(dst[r], bptrs, r)
            assert ra_lib.ra_sync_status() == 0, ra_lib.ra_last_error()
            assert torch.equal(back.view(torch.int16), x.view(torch.int16))
        del ref, dst
