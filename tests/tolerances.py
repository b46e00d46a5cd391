"""Tolerances for GPU-vs-oracle comparisons (bf16 inputs, fp32 accumulation).

* Forward O: max |dO| <= 1e-2; an element above 1e-2 still passes if its error
  is within 1e-2 + half a bf16 ulp of |O_oracle| (bf16 output rounding alone
  reaches 1/64 for |O| in [4, 8), which early causal rows can hit).  The count
  of such elements is reported.
* LSE: |dLSE| <= 1e-3 (absolute, natural log).
* dQ, dK, dV: relative L2 error <= 2e-2.
"""
import numpy as np

O_ATOL = 1e-2
LSE_ATOL = 1e-3
GRAD_REL_L2 = 2e-2


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, (np.floor(np.log2(ax)) - 8).astype(np.int64))


def check_o(o_gpu, o_ref, what="O"):
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite values"
    err = np.abs(o_gpu - o_ref)
    over = err > O_ATOL
    n_over = int(over.sum())
    if n_over:
        bound = O_ATOL + bf16_half_ulp(o_ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond 1e-2 + half-ulp; "
                               f"max err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")
    return float(err.max()), n_over


def check_lse(lse_gpu, lse_ref, what="LSE"):
    a = np.asarray(lse_gpu, np.float64)
    b = np.asarray(lse_ref, np.float64)
    assert a.shape == b.shape
    both_inf = np.isneginf(a) & np.isneginf(b)
    assert np.array_equal(np.isneginf(a), np.isneginf(b)), f"{what}: -inf pattern differs"
    err = np.abs(np.where(both_inf, 0.0, a - b))
    assert np.all(np.isfinite(err)), f"{what}: non-finite"
    assert err.max(initial=0.0) <= LSE_ATOL, f"{what}: max err {err.max():.3e}"
    return float(err.max(initial=0.0))


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def check_grad(g_gpu, g_ref, what):
    g = np.asarray(g_gpu, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    e = rel_l2(g, g_ref)
    assert e <= GRAD_REL_L2, f"{what}: rel L2 {e:.3e}"
    return e
