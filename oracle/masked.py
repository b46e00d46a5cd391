"""CPU oracle for attention with an additive bias and dropout.

TEST INFRASTRUCTURE ONLY, like ``oracle.attention``: imported by ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``, never by the
product path, and sharing no code with the CUDA kernels.

Sources (page title, then section):

* "优化的注意力实现 (FlashAttention)", section 优势与集成: the manual path of the
  PyTorch example adds a bias matrix to the scaled scores (``attn_weight +=
  attn_bias``, -inf where masked), takes the row softmax, applies dropout to the
  weights and multiplies by V; the fused call takes ``attn_mask`` and
  ``dropout_p``.
* "FlashAttention 的基本原理", section 2.4 反向传播: the backward of the paper's
  algorithm also covers masking and dropout (the page leaves them out).

Readings where the pages are silent:

* The bias is an additive float tensor (bf16 values) of shape [Bb, Hb, Nq, Nk]
  with Bb in {1, B} and Hb in {1, H} (broadcast over a dimension of size 1). It
  is a constant input: no gradient flows to it. -inf masks an entry; +inf and
  NaN are not allowed. It combines with the causal mask.
* Dropout zeroes each softmax weight with probability p and scales the kept ones
  by 1 / (1 - p) (torch.dropout); LSE is that of the weights before dropout.
* The random decisions come from the counter-based generator Philox4x32-10
  (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
  SC 2011), so the backward regenerates them instead of storing an N x N mask.
  One call covers a block of 4 queries x 4 keys of one (batch, head):
  counter = (key // 4, query // 4, b * H + h, offset), key = (seed mod 2^32,
  seed // 2^32); output word (query mod 4), byte (key mod 4) (least significant
  first) is that entry's random byte u.  p is used as the byte threshold
  p8 = floor(256 p + 1/2) in [0, 255], with p the float32 value the C ABI
  receives (a tie, 256 p exactly half-way between two integers, goes up): the
  entry is kept iff u >= p8, and the kept weights are scaled by
  256 / (256 - p8).
"""
from __future__ import annotations

import math

import numpy as np

from . import attention as A

# Philox constants of the paper: round multipliers and the Weyl key increments.
PHILOX4x32 = dict(bits=32, m=(0xD2511F53, 0xCD9E8D57), w=(0x9E3779B9, 0xBB67AE85))
PHILOX4x64 = dict(bits=64, m=(0xD2E7470EE14C6C93, 0xCA5A826395121157), w=(0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B))


def philox(counter, key, rounds: int = 10, params=PHILOX4x32):
    """Philox4xW-R on integer arrays: counter [..., 4], key [..., 2] -> [..., 4] (Python ints in object arrays
    for W = 64, uint64 holding W-bit values for W = 32).

    Round: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 (double-width products),
    c <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); the key is bumped by the Weyl constants between rounds.
    """
    W = params["bits"]
    mask = (1 << W) - 1
    dt = object if W == 64 else np.uint64
    c = [np.asarray(counter, dtype=dt)[..., i] for i in range(4)]
    k = [np.asarray(key, dtype=dt)[..., i] for i in range(2)]
    m0, m1 = (dt(x) if dt is not object else x for x in params["m"])
    w0, w1 = (dt(x) if dt is not object else x for x in params["w"])
    sh = dt(W) if dt is not object else W
    msk = dt(mask) if dt is not object else mask
    for r in range(rounds):
        if r > 0:
            k = [(k[0] + w0) & msk, (k[1] + w1) & msk]
        p0 = m0 * c[0]
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> sh, p0 & msk
        hi1, lo1 = p1 >> sh, p1 & msk
        c = [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]
    if dt is object:  # keep W-bit Python integers (numpy would promote a mix of int64 / uint64 to float)
        return np.stack([np.asarray(x, dtype=object) for x in c], axis=-1)
    return np.stack(c, axis=-1)


def dropout_p8(p: float) -> int:
    """The byte threshold floor(256 p + 1/2) for dropout probability p in [0, 1), p taken as float32."""
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    p32 = float(np.float32(p))
    return min(255, int(math.floor(256.0 * p32 + 0.5)))


def dropout_keep(B: int, H: int, Nq: int, Nk: int, p8: int, seed: int, offset: int = 0,
                 rows=None, b_only=None, h_only=None) -> np.ndarray:
    """Boolean keep mask [B, H, Nq, Nk] (or [len(rows), Nk] for one (b_only, h_only) head and rows)."""
    seed = int(seed)
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    heads = [(b, h) for b in range(B) for h in range(H)] if b_only is None else [(b_only, h_only)]
    qrows = np.arange(Nq) if rows is None else np.asarray(rows)
    keys = np.arange(Nk)
    out = np.zeros((len(heads), len(qrows), Nk), dtype=bool)
    for n, (b, h) in enumerate(heads):
        I, J = np.meshgrid(qrows // 4, keys // 4, indexing="ij")
        ctr = np.stack([J, I, np.full_like(I, b * H + h), np.full_like(I, offset)], axis=-1).astype(np.uint64)
        words = philox(ctr, key)                                  # [rows, keys, 4]
        word = np.take_along_axis(words, (qrows % 4)[:, None, None].repeat(Nk, 1), axis=-1)[..., 0]
        byte = (word >> (8 * (keys % 4)).astype(np.uint64)[None, :]) & np.uint64(0xFF)
        out[n] = byte >= np.uint64(p8)
    if b_only is not None:
        return out[0]
    return out.reshape(B, H, len(qrows), Nk)


def broadcast_bias(bias, B: int, H: int) -> np.ndarray:
    """[Bb, Hb, Nq, Nk] -> [B, H, Nq, Nk] (float64)."""
    bias = np.asarray(bias, dtype=np.float64)
    return np.broadcast_to(bias, (B, H) + bias.shape[2:])


def _scores(q, k, bias, scale, causal):
    s = scale * (q @ k.T)
    if bias is not None:
        s = s + bias
    if causal:
        s = np.where(A.causal_visible(q.shape[0], k.shape[0]), s, -np.inf)
    return s


def attention_forward_head(q, k, v, bias, scale: float, causal: bool, keep=None, p8: int = 0):
    """O = (softmax(scale q k^T + bias [+ causal]) o keep) v * 256 / (256 - p8), LSE before dropout."""
    s = _scores(q, k, bias, scale, causal)
    p, lse = A.softmax_rows(s)
    if keep is not None:
        p = p * keep * (256.0 / (256.0 - p8))
    return p @ v, lse


def attention_forward(q, k, v, bias, scale: float, causal: bool, keep=None, p8: int = 0):
    """Batched forward: q [B, H, Nq, d], k, v [B, H, Nk, d], bias broadcastable [Bb, Hb, Nq, Nk] or None,
    keep [B, H, Nq, Nk] bool or None."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    B, H, Nq, d = q.shape
    bb = None if bias is None else broadcast_bias(bias, B, H)
    o = np.zeros((B, H, Nq, v.shape[-1]))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_head(q[b, h], k[b, h], v[b, h], None if bb is None else bb[b, h],
                                                        scale, causal, None if keep is None else keep[b, h], p8)
    return o, lse


def attention_backward_head(q, k, v, do, bias, scale: float, causal: bool, keep=None, p8: int = 0):
    """dQ, dK, dV of <dO, O> for the forward above (bias and keep mask held constant).

    With Z = keep * 256 / (256 - p8): O = (P o Z) v, so dV = (P o Z)^T dO, the gradient reaching P is
    (dO v^T) o Z, and the row softmax gives dS = P o ((dO v^T) o Z - D) with D_i = sum_c dO_ic O_ic.
    """
    s = _scores(q, k, bias, scale, causal)
    p, _ = A.softmax_rows(s)
    z = np.ones_like(p) if keep is None else keep * (256.0 / (256.0 - p8))
    pz = p * z
    o = pz @ v
    dv = pz.T @ do
    dp = (do @ v.T) * z
    dvec = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - dvec)
    return scale * ds @ k, scale * ds.T @ q, dv


def attention_backward(q, k, v, do, bias, scale: float, causal: bool, keep=None, p8: int = 0):
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    B, H = q.shape[:2]
    bb = None if bias is None else broadcast_bias(bias, B, H)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = attention_backward_head(
                q[b, h], k[b, h], v[b, h], do[b, h], None if bb is None else bb[b, h], scale, causal,
                None if keep is None else keep[b, h], p8)
    return dq, dk, dv
