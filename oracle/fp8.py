"""CPU oracle for the FP8 forward with incoherent processing.

TEST INFRASTRUCTURE ONLY, like ``oracle.attention``: imported by ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``, never by the
product path, and sharing no code with the CUDA kernels.

Sources (page title, then section):

* "FlashAttention 系列技术详解", section 具体技术 (FlashAttention-3): the GEMMs run
  on FP8 tensor cores, which double the throughput; before quantisation, Q and K
  are multiplied by a random orthogonal matrix (a Hadamard transform, O(d log d)
  per head) so that outlier channels are spread out and the quantisation error
  drops ("incoherent processing").  Since Q M (K M)^T = Q K^T for orthogonal M,
  the attention result is unchanged in exact arithmetic.

Readings where the pages are silent (the pages name neither the FP8 format,
the scaling granularity nor the random matrix):

* The FP8 format is E4M3 in its "FN" variant: 1 sign, 4 exponent bits (bias 7),
  3 mantissa bits, no infinities, largest finite value 448, NaN = S.1111.111.
  Conversion rounds to nearest, ties to even, and saturates to +-448.
* The random orthogonal matrix is M = diag(s) H_d / sqrt(d): s a vector of
  random signs (an input, drawn by the caller) and H_d the Sylvester Hadamard
  matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]).  The same M is applied
  to Q and K; V is quantised without rotation.
* Scaling is per (batch, head): x8 = rn_e4m3(y * (448 / amax)) with amax the
  largest |y| of that head; the dequantisation factor is
  descale = (amax / 448) / sqrt(d) with the rotation (1 without), so that
  x M ~= dec(x8) * descale.
* The quantised code is an integer decided by floating point, so the oracle
  takes that decision in the kernel's precision: the transform and the scaling
  run in float32, the transform stage by stage in the order h = 1, 2, 4, ...,
  each butterfly (a, b) -> (a + b, a - b) with a the lower index.
* The reference attention is exact attention (float64) on the dequantised
  operands.  The kernel additionally rounds the softmax weights P to E4M3
  before the P V product; that error is covered by a tolerance, not modelled.
"""
from __future__ import annotations

import numpy as np

from . import attention as A

E4M3_MAX = 448.0
E4M3_MAX_CODE = 0x7E  # +448


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 (FN) byte, float64; NaN for S.1111.111."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, e - 7)
    sub = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, out)


# The 127 non-negative finite values, indexed by their code (0x00 .. 0x7E); increasing in the code.
_POS_VALUES = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(x) -> np.ndarray:
    """Round float values to E4M3 (FN) codes: nearest, ties to the even code, saturating at +-448.

    The sign bit is kept for -0.0.  NaN maps to 0x7F (with its sign).
    """
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    finite = np.isfinite(mag)
    clipped = np.where(finite, np.minimum(mag, E4M3_MAX), E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, clipped, side="left")  # first value >= |x|
    hi = np.minimum(hi, E4M3_MAX_CODE)
    lo = np.maximum(hi - 1, 0)
    v_hi, v_lo = _POS_VALUES[hi], _POS_VALUES[lo]
    exact = v_hi == clipped
    d_hi, d_lo = v_hi - clipped, clipped - v_lo
    pick_hi = exact | (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(np.isnan(x), 0x7F, code)
    sign = np.signbit(x).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def fwht(x, dtype=np.float64) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis: y = H_n x (Sylvester order).

    Stages h = 1, 2, 4, ..., n/2; in each, indices i and i + h of every block of 2h become
    (x_i + x_{i+h}, x_i - x_{i+h}).  Arithmetic in ``dtype``.
    """
    y = np.array(x, dtype=dtype, copy=True)
    n = y.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        z = y.reshape(*lead, n // (2 * h), 2, h)
        a, b = z[..., 0, :], z[..., 1, :]
        y = np.stack((a + b, a - b), axis=-2).reshape(*lead, n)
        h *= 2
    return y


def rotate(x, signs=None) -> np.ndarray:
    """x M with M = diag(signs) H_d / sqrt(d), float64 (rows of x are vectors of length d)."""
    x = np.asarray(x, dtype=np.float64)
    if signs is not None:
        x = x * np.asarray(signs, dtype=np.float64)
    return fwht(x, np.float64) / np.sqrt(x.shape[-1])


def quantize(x, signs=None, hadamard: bool = True):
    """Per-(batch, head) E4M3 quantisation of x [B, H, N, d], with incoherent processing when
    ``hadamard``.  Returns (codes uint8 [B, H, N, d], descale float32 [B, H]).

    float32 steps: y = x * signs (exact), y = H_d y (stage order of ``fwht``), amax = max |y| per
    head, qs = 448 / amax (1 when amax == 0), code = rn_e4m3(y * qs),
    descale = (amax / 448) * r with r = float32(1 / sqrt(d)) under rotation, else 1.
    """
    y = np.asarray(x, dtype=np.float32)
    d = y.shape[-1]
    if hadamard:
        if signs is not None:
            y = y * np.asarray(signs, dtype=np.float32)
        y = fwht(y, np.float32)
    amax = np.abs(y).max(axis=(-2, -1)) if y.shape[-2] > 0 else np.zeros(y.shape[:-2], np.float32)
    amax = amax.astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    qs = np.where(amax > 0, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    scaled = (y * qs[..., None, None]).astype(np.float32)
    codes = e4m3_encode(scaled)
    r = np.float32(1.0 / np.sqrt(d)) if hadamard else np.float32(1.0)
    descale = ((amax / np.float32(E4M3_MAX)).astype(np.float32) * r).astype(np.float32)
    return codes, descale


def dequantize(codes, descale) -> np.ndarray:
    """dec(codes) * descale per (batch, head), float64."""
    return e4m3_decode(codes) * np.asarray(descale, dtype=np.float64)[..., None, None]


def attention_forward_fp8(q8, k8, v8, dq, dk, dv, scale: float, causal: bool):
    """Exact attention (float64) on the dequantised operands: (O [B,H,Nq,d], LSE [B,H,Nq])."""
    return A.attention_forward(dequantize(q8, dq), dequantize(k8, dk), dequantize(v8, dv), scale, causal)


def attention_forward_fp8_rows(q8, k8, v8, dq, dk, dv, b: int, h: int, rows, scale: float, causal: bool):
    """Selected query rows of one (batch, head) of ``attention_forward_fp8``."""
    qh = e4m3_decode(q8[b, h]) * float(dq[b, h])
    kh = e4m3_decode(k8[b, h]) * float(dk[b, h])
    vh = e4m3_decode(v8[b, h]) * float(dv[b, h])
    return A.attention_forward_rows(qh, kh, vh, rows, scale, causal)
