"""Pins for the FP8 / incoherent-processing oracle (CPU only).

What pins it, other than itself:
* E4M3 decode and encode: torch's float8_e4m3fn casts (a library routine) on all 256 codes,
  every tie between neighbouring values, and random values; hand-derived codes for
  the special cases (saturation, -0, subnormal ties).
* The Hadamard transform: scipy.linalg.hadamard (a library routine) in float64, and the
  Sylvester recursion H_2n = [[H_n, H_n], [H_n, -H_n]] evaluated recursively in float32
  (the stage order the kernel must reproduce bit for bit).
* The rotation: orthonormality, the involution (H / sqrt(d))^2 = I, and Q M (K M)^T = Q K^T.
* Quantisation: the per-head amax element lands on +-448, and every dequantised value
  is within half an E4M3 step of the rotated input.
* The pages' claim ("FlashAttention 系列技术详解", section 具体技术): incoherent
  processing lowers the quantisation error when Q and K have outlier channels.
* The FP8 reference attention equals torch's float64 attention on the dequantised operands.
The mutation tests at the end plant plausible mistakes and check that a pin rejects each.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import attention as A
from oracle import fp8 as F


def torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy().astype(np.float64)


def torch_encode(x):
    t = torch.from_numpy(np.asarray(x, np.float32).copy()).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def tie_and_grid_values():
    pos = torch_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(5)
    rnd = np.exp2(rng.uniform(-12, math.log2(448), 4000)) * rng.choice([-1, 1], 4000)
    v = np.concatenate([pos, -pos, mids, -mids, rnd]).astype(np.float32)
    return v[np.abs(v) <= 448]


# ----------------------------------------------------------------------------------------
# pin functions (take an implementation so that the mutation tests can reuse them)
# ----------------------------------------------------------------------------------------
def pin_decode(decode):
    codes = np.arange(256, dtype=np.uint8)
    ours, ref = decode(codes), torch_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def pin_encode(encode):
    v = tie_and_grid_values()
    assert np.array_equal(encode(v), torch_encode(v))
    # Hand-derived codes: 1 = 0.0111.000; 448 = 0.1111.110; saturation; -0 keeps its sign;
    # 2^-10 is the tie between 0 and 2^-9 (even code 0); 1.5 * 2^-9 the tie between codes 1 and 2.
    cases = [(1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),
             (1.5 * 2.0 ** -9, 0x02), (1000.0, 0x7E), (-1e9, 0xFE), (float("inf"), 0x7E), (-0.0, 0x80),
             (0.0, 0x00), (464.0, 0x7E), (1.0625, 0x38), (1.1875, 0x3A), (-3.0, 0xC4)]
    got = encode(np.array([v for v, _ in cases], np.float32))
    assert [int(c) for c in got] == [c for _, c in cases]


def sylvester_recursive_f32(x):
    x = np.asarray(x, np.float32)
    n = x.shape[-1]
    if n == 1:
        return x.copy()
    a = sylvester_recursive_f32(x[..., : n // 2])
    b = sylvester_recursive_f32(x[..., n // 2:])
    return np.concatenate([a + b, a - b], axis=-1)


def pin_fwht(fwht):
    rng = np.random.default_rng(1)
    for n in (1, 2, 4, 8, 16, 32, 64, 128, 256):
        x = rng.standard_normal((3, n))
        assert np.allclose(fwht(x, np.float64), x @ scipy.linalg.hadamard(n).T, rtol=0, atol=1e-12)
    for n in (64, 128):
        x = rng.standard_normal((50, n)).astype(np.float32)
        assert np.array_equal(fwht(x, np.float32), sylvester_recursive_f32(x))


def half_step(z):
    """Half the spacing of E4M3 values at |z| (subnormal spacing 2^-9 below 2^-6)."""
    az = np.abs(np.asarray(z, np.float64))
    e = np.floor(np.log2(np.maximum(az, 2.0 ** -6)))
    return np.ldexp(1.0, (e - 4).astype(np.int64))


def pin_quantize(quantize):
    rng = np.random.default_rng(2)
    for hadamard in (True, False):
        for d in (64, 128):
            x = rng.standard_normal((2, 3, 37, d)).astype(np.float32)
            x[1, 2] *= 20.0  # heads with very different ranges
            signs = rng.choice([-1.0, 1.0], d)
            codes, descale = quantize(x, signs, hadamard)
            assert codes.dtype == np.uint8 and descale.dtype == np.float32 and descale.shape == (2, 3)
            y = F.rotate(x, signs) if hadamard else x.astype(np.float64)
            r = 1.0 / math.sqrt(d) if hadamard else 1.0
            amax = np.abs(y).max(axis=(-2, -1)) / r
            for b in range(2):
                for h in range(3):
                    c = codes[b, h]
                    assert (np.abs(F.e4m3_decode(c)) == 448.0).any(), "the amax element must map to +-448"
                    assert not (np.abs(F.e4m3_decode(c)) > 448.0).any()
                    qs = 448.0 / amax[b, h]
                    deq = F.e4m3_decode(c) * float(descale[b, h])
                    bound = half_step(y[b, h] / r * qs) / qs * r * (1 + 1e-5) + 1e-6 * np.abs(y[b, h]) + 1e-30
                    assert np.all(np.abs(deq - y[b, h]) <= bound)
                    assert math.isclose(float(descale[b, h]), amax[b, h] / 448.0 * r, rel_tol=1e-6)
    z = np.zeros((1, 1, 5, 64), np.float32)
    codes, descale = quantize(z, -np.ones(64), True)
    assert descale[0, 0] == 0.0 and np.all(F.e4m3_decode(codes) == 0.0)


# ----------------------------------------------------------------------------------------
# the pins
# ----------------------------------------------------------------------------------------
def test_decode_matches_library_cast():
    pin_decode(F.e4m3_decode)


def test_encode_matches_library_cast_and_hand_codes():
    pin_encode(F.e4m3_encode)


def test_fwht_matches_sylvester_matrix_and_recursion():
    pin_fwht(F.fwht)


def test_rotation_is_orthonormal_and_preserves_scores():
    rng = np.random.default_rng(3)
    d = 128
    s = rng.choice([-1.0, 1.0], d)
    q, k = rng.standard_normal((40, d)), rng.standard_normal((50, d))
    qm, km = F.rotate(q, s), F.rotate(k, s)
    assert np.allclose(np.linalg.norm(qm, axis=1), np.linalg.norm(q, axis=1), rtol=1e-12)
    assert np.allclose(qm @ km.T, q @ k.T, rtol=0, atol=1e-10)
    assert np.allclose(F.rotate(F.rotate(q)), q, atol=1e-12)
    m = F.rotate(np.eye(d), s)  # the matrix M itself
    assert np.allclose(m @ m.T, np.eye(d), atol=1e-12)


def test_quantize_bounds():
    pin_quantize(F.quantize)


def test_incoherent_processing_lowers_error_with_outliers():
    """The section's claim: spreading outliers with the random Hadamard rotation before FP8 quantisation
    reduces the error of Q K^T."""
    rng = np.random.default_rng(4)
    d = 128
    q = rng.standard_normal((1, 1, 512, d))
    k = rng.standard_normal((1, 1, 512, d))
    for ch in (3, 40, 77, 101):
        q[..., ch] *= 40.0
        k[..., ch] *= 40.0
    s = rng.choice([-1.0, 1.0], d)
    exact = q[0, 0] @ k[0, 0].T
    errs = {}
    for had in (False, True):
        q8, dq = F.quantize(q, s, had)
        k8, dk = F.quantize(k, s, had)
        approx = F.dequantize(q8, dq)[0, 0] @ F.dequantize(k8, dk)[0, 0].T
        errs[had] = np.linalg.norm(approx - exact) / np.linalg.norm(exact)
    assert errs[True] < 0.5 * errs[False], errs


def test_fp8_reference_is_attention_on_dequantised_operands():
    rng = np.random.default_rng(6)
    x = {n: rng.standard_normal((1, 2, 70, 128)) for n in "qkv"}
    s = rng.choice([-1.0, 1.0], 128)
    q8, dq = F.quantize(x["q"], s)
    k8, dk = F.quantize(x["k"], s)
    v8, dv = F.quantize(x["v"], None, hadamard=False)
    scale = 1 / math.sqrt(128)
    for causal in (False, True):
        o, lse = F.attention_forward_fp8(q8, k8, v8, dq, dk, dv, scale, causal)
        tq, tk, tv = (torch.from_numpy(F.dequantize(c, ds)) for c, ds in ((q8, dq), (k8, dk), (v8, dv)))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        assert np.allclose(o, ref.numpy(), atol=1e-12)
        rows = np.array([0, 33, 69])
        orow, lrow = F.attention_forward_fp8_rows(q8, k8, v8, dq, dk, dv, 0, 1, rows, scale, causal)
        assert np.allclose(orow, o[0, 1, rows], atol=1e-12) and np.allclose(lrow, lse[0, 1, rows], atol=1e-12)
    # Constant V rows: the output is that constant whatever the weights.
    v_const = np.tile(rng.standard_normal(128), (1, 2, 70, 1))
    v8c, dvc = F.quantize(v_const, None, hadamard=False)
    o, _ = F.attention_forward_fp8(q8, k8, v8c, dq, dk, dvc, scale, True)
    assert np.allclose(o, F.dequantize(v8c, dvc), atol=1e-12)


# ----------------------------------------------------------------------------------------
# mutation tests: each planted mistake must fail a pin
# ----------------------------------------------------------------------------------------
def _decode_bias8(codes):
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 7
    v = np.where(e == 0, np.ldexp(m / 8.0, -7), np.ldexp(1 + m / 8.0, e - 8))
    v = np.where(c & 0x80, -v, v)
    return np.where((e == 15) & (m == 7), np.nan, v)


def _encode_ties_away(x):
    x = np.asarray(x, np.float64)
    mag = np.minimum(np.abs(x), 448.0)
    vals = F._POS_VALUES
    hi = np.minimum(np.searchsorted(vals, mag), 0x7E)
    lo = np.maximum(hi - 1, 0)
    code = np.where(vals[hi] - mag <= mag - vals[lo], hi, lo)
    return (code | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)


def _encode_drops_negative_zero(x):
    c = F.e4m3_encode(x)
    return np.where(np.asarray(x) == 0, 0, c).astype(np.uint8)


def _fwht_swapped(x, dtype=np.float64):
    y = np.array(x, dtype=dtype, copy=True)
    n = y.shape[-1]
    h = 1
    while h < n:
        z = y.reshape(*y.shape[:-1], n // (2 * h), 2, h)
        a, b = z[..., 0, :], z[..., 1, :]
        y = np.stack((a + b, b - a), axis=-2).reshape(y.shape)
        h *= 2
    return y


def _fwht_reversed_stages(x, dtype=np.float64):
    y = np.array(x, dtype=dtype, copy=True)
    n = y.shape[-1]
    h = n // 2
    while h >= 1:
        z = y.reshape(*y.shape[:-1], n // (2 * h), 2, h)
        a, b = z[..., 0, :], z[..., 1, :]
        y = np.stack((a + b, a - b), axis=-2).reshape(y.shape)
        h //= 2
    return y


def _quantize_no_rsqrt(x, signs=None, hadamard=True):
    codes, descale = F.quantize(x, signs, hadamard)
    d = np.asarray(x).shape[-1]
    return codes, (descale * np.float32(math.sqrt(d)) if hadamard else descale).astype(np.float32)


def _quantize_global_amax(x, signs=None, hadamard=True):
    y = np.asarray(x, np.float32)
    if hadamard:
        y = F.fwht(y * np.asarray(signs, np.float32), np.float32)
    amax = np.float32(np.abs(y).max())
    codes = F.e4m3_encode(y * (np.float32(448) / amax))
    r = np.float32(1 / math.sqrt(y.shape[-1])) if hadamard else np.float32(1)
    return codes, np.full(y.shape[:2], amax / np.float32(448) * r, np.float32)


def _quantize_no_signs(x, signs=None, hadamard=True):
    return F.quantize(x, None, hadamard)


@pytest.mark.parametrize("pin,impl", [
    (pin_decode, _decode_bias8),
    (pin_encode, _encode_ties_away),
    (pin_encode, _encode_drops_negative_zero),
    (pin_fwht, _fwht_swapped),
    (pin_fwht, _fwht_reversed_stages),
    (pin_quantize, _quantize_no_rsqrt),
    (pin_quantize, _quantize_global_amax),
    (pin_quantize, _quantize_no_signs),
])
def test_pins_reject_planted_mistakes(pin, impl):
    with pytest.raises(AssertionError):
        pin(impl)
