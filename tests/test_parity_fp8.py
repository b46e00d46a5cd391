"""FP8 forward with incoherent processing: the CUDA path against the oracle.

* fa_quantize_fp8 is integer work decided by float32 arithmetic: its E4M3 codes and its
  fp32 descale factors must equal the oracle's bit for bit.
* fa_fwd_fp8 runs on codes the oracle produced.  Its reference is exact attention on the
  dequantised operands; the kernel also rounds the softmax weights P to E4M3 before the P V
  product.  The tolerance is derived from that rounding, element by element: a normal E4M3
  value is within 2^-4 of P relative, a subnormal one within 2^-10 absolute, and O is
  normalised by the sum of the rounded weights, so to first order
      |dO_ic| <= 2^-4 sum_j w_ij |v_jc - O_ic| + 2^-10 / Z_i sum_{j: t_ij < 2^-6} |v_jc - O_ic|
  with t_ij = exp(s_ij - max_j s_ij), Z_i = sum_j t_ij, w_ij = t_ij / Z_i (the kernel's weights
  are t_ij scaled by a factor >= 1, so a subnormal weight has t_ij < 2^-6 and its sum is >= Z_i).
  A 10% margin covers the second-order terms and the rounded denominator; half a bf16 ulp
  covers the output rounding.  LSE uses the exact fp32 sum: |dLSE| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
from oracle import fp8 as F
import gpu_common as gc
from tolerances import bf16_half_ulp, check_lse

pytestmark = pytest.mark.gpu


def oracle_quantize(x_bf16, signs, hadamard):
    return F.quantize(x_bf16.float().numpy(), None if signs is None else signs.numpy(), hadamard)


def gpu_quantize(x_bf16, signs, hadamard):
    xd = x_bf16.to(gc.DEV).contiguous()
    sd = signs.to(gc.DEV) if signs is not None else None
    x8, ds = fa.quantize_fp8(xd, sd, hadamard)
    torch.cuda.synchronize()
    return x8.cpu().numpy(), ds.cpu().numpy()


QUANT_CASES = [
    # B, H, N, d, hadamard, with signs
    (1, 2, 128, 64, True, True),
    (2, 3, 200, 128, True, True),
    (1, 1, 77, 128, False, False),
    (2, 2, 1, 64, True, False),
    (1, 2, 1000, 128, True, True),   # 15 full blocks of 64 rows and a ragged 40
    (1, 1, 333, 64, False, False),
]


@pytest.mark.parametrize("B,H,N,d,had,with_signs", QUANT_CASES)
def test_quantize_bit_exact(B, H, N, d, had, with_signs):
    x = W.make_attention_inputs(B, H, N, N, d, 100 + N + d, with_do=False)["q"]
    x = W.add_outlier_channels(x, [1, d // 2 + 3], 32.0)
    signs = W.make_hadamard_signs(d, 7 + d) if with_signs else None
    codes, ds = gpu_quantize(x, signs, had)
    rc, rds = oracle_quantize(x, signs, had)
    assert np.array_equal(ds, rds), (ds, rds)
    mism = codes != rc
    assert not mism.any(), f"{int(mism.sum())} codes differ, first at {np.argwhere(mism)[0]}"


def test_quantize_zero_head_and_empty():
    x = torch.zeros(1, 2, 70, 128, dtype=torch.bfloat16)
    x[0, 1] = W.make_attention_inputs(1, 1, 70, 70, 128, 3, with_do=False)["q"][0, 0]
    codes, ds = gpu_quantize(x, W.make_hadamard_signs(128, 1), True)
    rc, rds = oracle_quantize(x, W.make_hadamard_signs(128, 1), True)
    assert ds[0, 0] == 0.0 and np.array_equal(ds, rds) and np.array_equal(codes, rc)
    e = torch.zeros(2, 2, 0, 64, dtype=torch.bfloat16, device=gc.DEV)
    _, de = fa.quantize_fp8(e, None, True)
    torch.cuda.synchronize()
    assert torch.all(de == 0)


def fp8_bound(qh, kh, vh, o_ref, scale, causal):
    """Elementwise first-order bound on |O_kernel - O_ref| from the E4M3 rounding of P (one head)."""
    s = A.scaled_scores(qh, kh, scale, causal)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    t = np.exp(s - m)
    Z = t.sum(axis=1, keepdims=True)
    Zs = np.where(Z > 0, Z, 1.0)
    w = t / Zs
    bound = np.zeros_like(o_ref)
    sub = ((t < 2.0 ** -6) & np.isfinite(s)).astype(np.float64)  # masked keys carry no weight
    for c in range(vh.shape[1]):
        dev = np.abs(vh[None, :, c] - o_ref[:, c:c + 1])
        bound[:, c] = 2.0 ** -4 * (w * dev).sum(axis=1) + 2.0 ** -10 / Zs[:, 0] * (sub * dev).sum(axis=1)
    return 1.1 * bound + bf16_half_ulp(o_ref) + 1e-4


def run_fwd_fp8(q8, k8, v8, dq, dk, dv, causal, scale):
    dev = [torch.from_numpy(np.ascontiguousarray(a)).to(gc.DEV) for a in (q8, k8, v8, dq, dk, dv)]
    B, H, Nq, d = q8.shape
    o = torch.empty(B, H, Nq, d, dtype=torch.bfloat16, device=gc.DEV)
    lse = torch.empty(B, H, Nq, dtype=torch.float32, device=gc.DEV)
    fa.fa_fwd_fp8(*dev, o, lse, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return gc.f64(o), gc.f64(lse)


def quantized_inputs(B, H, Nq, Nk, d, seed, outliers=False):
    x = W.make_attention_inputs(B, H, Nq, Nk, d, seed, with_do=False)
    q, k, v = x["q"], x["k"], x["v"]
    if outliers:
        q = W.add_outlier_channels(q, [5, 70], 16.0)
        k = W.add_outlier_channels(k, [5, 70], 16.0)
    signs = W.make_hadamard_signs(d, seed + 1)
    q8, dq = oracle_quantize(q, signs, True)
    k8, dk = oracle_quantize(k, signs, True)
    v8, dv = oracle_quantize(v, None, False)
    return q8, k8, v8, dq, dk, dv


FWD_CASES = [
    # B, H, Nq, Nk, causal
    (1, 2, 128, 128, False),
    (2, 4, 1024, 1024, True),
    (2, 4, 1024, 1024, False),
    (1, 2, 300, 517, True),      # ragged, Nk > Nq
    (1, 2, 513, 1025, False),
    (2, 3, 257, 129, True),      # Nq > Nk: leading rows see no key
    (1, 1, 1, 1, False),
    (4, 16, 1024, 1024, True),   # enough query tiles for two tiles per CTA
]


@pytest.mark.parametrize("B,H,Nq,Nk,causal", FWD_CASES)
def test_fwd_fp8_matches_oracle(B, H, Nq, Nk, causal):
    d = 128
    scale = 1.0 / math.sqrt(d)
    q8, k8, v8, dq, dk, dv = quantized_inputs(B, H, Nq, Nk, d, 40 + Nq + Nk)
    o, lse = run_fwd_fp8(q8, k8, v8, dq, dk, dv, causal, scale)
    o_ref, lse_ref = F.attention_forward_fp8(q8, k8, v8, dq, dk, dv, scale, causal)
    check_lse(lse, lse_ref)
    assert np.all(np.isfinite(o))
    worst = 0.0
    heads = sorted({(0, 0), (B - 1, H - 1), (B // 2, H // 2), (0, H - 1)})  # the bound costs ~1 s per 1024^2 head
    for b, h in heads:
        qh, kh, vh = (F.e4m3_decode(c[b, h]) * float(s[b, h]) for c, s in ((q8, dq), (k8, dk), (v8, dv)))
        bound = fp8_bound(qh, kh, vh, o_ref[b, h], scale, causal)
        err = np.abs(o[b, h] - o_ref[b, h])
        assert np.all(err <= bound), f"head ({b},{h}): {int((err > bound).sum())} elements beyond the bound"
        worst = max(worst, float((err / bound).max()))
    rel = np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30)
    assert rel < 0.05, rel
    print(f"max err / bound = {worst:.3f}, rel L2 = {rel:.4f}")


def test_fwd_fp8_full_size_sampled_rows():
    """The 16 x 16384 causal d = 128 workload the bench times: sampled rows of two heads."""
    c = next(s for s in W.SWEEP if s.Nq == 16384 and s.d == 128)
    q8, k8, v8, dq, dk, dv = quantized_inputs(c.B, c.H, c.Nq, c.Nk, c.d, c.seed)
    o, lse = run_fwd_fp8(q8, k8, v8, dq, dk, dv, True, c.scale)
    for h in (0, c.H - 1):
        rows = gc.sample_rows(c.Nq, 24, 90 + h, must=(127, 128, 255, 256, c.Nq - 129))
        o_ref, lse_ref = F.attention_forward_fp8_rows(q8, k8, v8, dq, dk, dv, 0, h, rows, c.scale, True)
        check_lse(lse[0, h, rows], lse_ref)
        qh, kh, vh = (F.e4m3_decode(x[0, h]) * float(s[0, h]) for x, s in ((q8, dq), (k8, dk), (v8, dv)))
        bound = np.stack([fp8_bound(qh[r:r + 1], kh[: r + 1], vh[: r + 1], o_ref[i:i + 1], c.scale, False)[0]
                          for i, r in enumerate(rows)])
        assert np.all(np.abs(o[0, h, rows] - o_ref) <= bound)


def test_fwd_fp8_constant_values():
    """Every V row equal: O is that row whatever the weights (the rounded-sum normalisation)."""
    B, H, N, d = 1, 2, 700, 128
    q8, k8, _, dq, dk, _ = quantized_inputs(B, H, N, N, d, 3)
    row = W.make_attention_inputs(1, 1, 1, 1, d, 9, with_do=False)["v"][0, 0, 0]
    v = row.expand(B, H, N, d).contiguous()
    v8, dv = oracle_quantize(v, None, False)
    o, _ = run_fwd_fp8(q8, k8, v8, dq, dk, dv, True, 1 / math.sqrt(d))
    want = F.dequantize(v8, dv)
    assert np.allclose(o, want, rtol=2 ** -8, atol=1e-6)


@pytest.mark.parametrize("outliers", [False, True])
def test_end_to_end_accuracy_against_exact_bf16_attention(outliers):
    """attention_forward_fp8 (rotation, quantisation and the FP8 forward, all on the GPU) against exact
    attention of the original bf16 inputs; with outlier channels the rotation must lower the error,
    as the FlashAttention-3 section states."""
    B, H, N, d = 1, 4, 1024, 128
    x = W.make_attention_inputs(B, H, N, N, d, 21, with_do=False)
    q, k, v = x["q"], x["k"], x["v"]
    if outliers:
        q = W.add_outlier_channels(q, [3, 40, 77, 101], 8.0)
        k = W.add_outlier_channels(k, [3, 40, 77, 101], 8.0)
    scale = 1 / math.sqrt(d)
    o_ref, _ = A.attention_forward(gc.f64(q), gc.f64(k), gc.f64(v), scale, True)
    signs = W.make_hadamard_signs(d, 5).to(gc.DEV)
    qd, kd, vd = gc.to_dev(q, k, v)
    errs = {}
    for had in (True, False):
        o, _ = fa.attention_forward_fp8(qd, kd, vd, causal=True, scale=scale, signs=signs, hadamard=had)
        torch.cuda.synchronize()
        errs[had] = np.linalg.norm(gc.f64(o) - o_ref) / np.linalg.norm(o_ref)
    print("rel L2 vs exact bf16 attention:", errs)
    assert errs[True] < 0.1
    if outliers:
        assert errs[True] < 0.5 * errs[False]
