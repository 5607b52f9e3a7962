"""Helpers for the GPU parity tests: tolerances, comparisons and the oracle call shapes."""
import numpy as np
import torch

# Tolerances fixed for this path: bf16 inputs with fp32 accumulation -> max-abs 1e-2 on O
# and 1e-3 on LSE; fp32 inputs -> 1e-4 on both.
TOL = {torch.bfloat16: (1e-2, 1e-3), torch.float32: (1e-4, 1e-4)}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a (bf16 or fp32) tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def chunks_to_seq(x: torch.Tensor) -> torch.Tensor:
    """[P, B, Lc, H, D] chunk-major K/V -> [B, P*Lc, H, D] in global token order."""
    P, B, Lc, H, D = x.shape
    return x.permute(1, 0, 2, 3, 4).reshape(B, P * Lc, H, D)


def max_abs(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    assert np.all(np.isfinite(a)), "non-finite values in the GPU result"
    return float(np.max(np.abs(a - b)))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (8 significand bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 8)


def rows_oracle(oracle_mod, q, k_seq, v_seq, rows, scale, causal):
    """Oracle output for sampled (b, t, h) rows; q [B,L,H_q,D], k/v [B,L,H_kv,D] tensors."""
    rb, rt, rh = rows
    qn = f64(q[torch.tensor(rb), torch.tensor(rt), torch.tensor(rh)])
    return oracle_mod.attention_rows(qn, rb, rt, rh, f64(k_seq), f64(v_seq), q.shape[2], scale,
                                     causal)


# Backward bar: per gradient tensor, max|error| <= GRAD_REL * max|reference| + GRAD_ABS (the
# gradients are sums of products of bf16-rounded operands accumulated in fp32; the floor
# covers gradients that vanish analytically).
GRAD_REL = 1e-2
GRAD_ABS = 1e-4


def check_grad(name: str, nm: str, got: np.ndarray, ref: np.ndarray) -> float:
    """Assert the backward bar for one gradient tensor (or sampled rows of it) and print,
    beside it, the worst elementwise relative error over the elements whose reference is
    above 1e-2 of the largest, so that errors on small gradient elements are visible.
    Returns that relative error."""
    assert np.all(np.isfinite(got)), (name, nm)
    err = np.abs(got - ref)
    mx = float(np.abs(ref).max()) if ref.size else 0.0
    e = float(err.max()) if err.size else 0.0
    big = np.abs(ref) > 1e-2 * mx
    rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    print(f"[parity] bwd {name} {nm}: max|err|={e:.3e} max|ref|={mx:.3e} "
          f"ratio={e / max(mx, 1e-30):.2e} worst rel (|ref| > 1e-2 max)={rel:.2e}")
    assert e <= GRAD_REL * mx + GRAD_ABS, (name, nm, e, mx)
    return rel


# dQ is summed in fp32 global memory from one contribution per key tile, added by bulk
# reduce-adds whose order across CTAs varies from call to call, while every contribution is
# the same bits in two calls on the same inputs.  Two such calls therefore agree on dK and dV
# bit for bit and on dQ up to the rounding of a reordered fp32 sum (a few units of 2^-24 of
# the partial sums per addition): the check is max|difference| <= DQ_ORDER_REL * max|dQ|.
DQ_ORDER_REL = 1e-5


def assert_same_grads(want, got, label: str = "") -> None:
    """(dq, dk, dv) of two backward calls on the same problem: dK and dV bit for bit, dQ up
    to the order of its reduce-adds (the measured difference is printed)."""
    (dq0, dk0, dv0), (dq1, dk1, dv1) = want, got
    assert torch.equal(dk0, dk1), f"{label}: dk differs"
    assert torch.equal(dv0, dv1), f"{label}: dv differs"
    assert bool(torch.isfinite(dq1).all()), f"{label}: non-finite dq"
    d = float((dq0.double() - dq1.double()).abs().max())
    m = float(dq0.double().abs().max())
    print(f"[dq order] {label}: max|diff| = {d:.3e} ({d / max(m, 1e-30):.2e} of max|dq|)")
    assert d <= DQ_ORDER_REL * m, (label, d, m)
