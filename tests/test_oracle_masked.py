"""Pins for the bias / dropout oracle (CPU only).

What pins it, other than itself:
* Philox: the shared round function in its 4x64 instance against numpy's Philox bit generator (a
  library routine; numpy advances the counter by one before each block), and the 4x32 instance
  the kernels use against the known-answer vectors published with the Random123 library
  (Salmon et al., SC 2011).
* The dropout decisions: the kept fraction against the binomial law, a hand-traced element, and
  independence of the rows requested.
* The forward with a bias: torch's float64 scaled_dot_product_attention with the same float
  mask (a library routine); rows masked entirely give O = 0 and LSE = -inf.
* The forward with dropout: the mean over seeds of O approaches the output without dropout
  (dropout with 1 / (1 - p) scaling is unbiased); p8 = 0 leaves the result unchanged.
* The backward: torch float64 autograd of the forward with the same bias and keep mask, and central
  finite differences of <dO, O>.
The mutation tests at the end plant plausible mistakes and check that a pin rejects each.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import masked as M


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ----------------------------------------------------------------------------------------
# pin functions
# ----------------------------------------------------------------------------------------
def pin_philox(philox):
    for key, ctr in (((1, 2), (5, 0, 0, 0)), ((0xFFFFFFFFFFFFFFFF, 7), (0xFFFFFFFFFFFFFFFE, 3, 0, 9)),
                     ((123456789, 987654321), (42, 43, 44, 45))):
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64))
        st = bg.state
        st["state"]["counter"] = np.array(ctr, dtype=np.uint64)
        bg.state = st
        want = [int(x) for x in bg.random_raw(4)]
        nxt = list(ctr)
        nxt[0] = (nxt[0] + 1) & 0xFFFFFFFFFFFFFFFF
        if nxt[0] == 0:
            nxt[1] += 1
        got = philox(np.array(nxt, dtype=object), np.array(key, dtype=object), params=M.PHILOX4x64)
        assert [int(x) for x in got] == want
    kat = [((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
           ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
           ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
            (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1))]
    for ctr, key, want in kat:
        got = philox(np.array(ctr, dtype=np.uint64), np.array(key, dtype=np.uint64))
        assert tuple(int(x) for x in got) == want


def pin_keep(keep_fn):
    B, H, Nq, Nk = 2, 3, 67, 130
    for p8 in (0, 26, 128, 230):
        k = keep_fn(B, H, Nq, Nk, p8, seed=0x1234_5678_9ABC, offset=5)
        n = k.size
        want = 1 - p8 / 256
        assert abs(k.mean() - want) <= 5 * math.sqrt(want * (1 - want) / n) + 1e-12, (p8, k.mean())
        if p8 == 0:
            assert k.all()
    # One element traced by hand: (b, h) = (1, 2) of H = 3, query 13, key 70, seed 77, offset 9:
    # counter (70 // 4, 13 // 4, 1 * 3 + 2, 9), key (77, 0), word 13 % 4 = 1, byte 70 % 4 = 2.
    words = M.philox(np.array([17, 3, 5, 9], dtype=np.uint64), np.array([77, 0], dtype=np.uint64))
    byte = (int(words[1]) >> 16) & 0xFF
    k = keep_fn(B, H, Nq, Nk, byte, seed=77, offset=9)
    assert k[1, 2, 13, 70]
    k = keep_fn(B, H, Nq, Nk, byte + 1, seed=77, offset=9)
    assert not k[1, 2, 13, 70]
    # Rows requested one head at a time agree with the whole tensor.
    full = keep_fn(B, H, Nq, Nk, 100, seed=3, offset=0)
    rows = np.array([0, 5, 66])
    assert np.array_equal(keep_fn(B, H, Nq, Nk, 100, seed=3, offset=0, rows=rows, b_only=1, h_only=0), full[1, 0, rows])
    assert not np.array_equal(full, keep_fn(B, H, Nq, Nk, 100, seed=4, offset=0))
    assert not np.array_equal(full, keep_fn(B, H, Nq, Nk, 100, seed=3, offset=1))


def make_bias(B, H, Nq, Nk, seed, hidden=0.2):
    rng = np.random.default_rng(seed)
    bias = rng.standard_normal((B, H, Nq, Nk))
    bias[rng.random((B, H, Nq, Nk)) < hidden] = -np.inf
    return bias


def pin_forward_bias(fwd):
    rng = np.random.default_rng(1)
    B, H, Nq, Nk, d = 2, 2, 13, 21, 8
    q, k, v = rng.standard_normal((B, H, Nq, d)), rng.standard_normal((B, H, Nk, d)), rng.standard_normal((B, H, Nk, d))
    for bshape in ((B, H), (1, H), (B, 1), (1, 1)):
        bias = make_bias(*bshape, Nq, Nk, 2)
        bias[..., 3, :] = -np.inf  # one row masked entirely
        for causal in (False, True):
            o, lse = fwd(q, k, v, bias, 0.3, causal)
            tb = torch.from_numpy(np.broadcast_to(bias, (B, H, Nq, Nk)).copy())
            if causal:
                tb = tb.masked_fill(~torch.from_numpy(A.causal_visible(Nq, Nk)), -math.inf)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=tb, scale=0.3).numpy()
            dead = np.isneginf(tb.numpy()).all(axis=-1)
            assert np.allclose(o[~dead], ref[~dead], atol=1e-12)
            assert np.all(o[dead] == 0) and np.all(np.isneginf(lse[dead]))
            assert dead[..., 3].all()
            s = 0.3 * np.einsum("bhqd,bhkd->bhqk", q, k) + np.where(np.isfinite(tb.numpy()), tb.numpy(), 0)
            s = np.where(np.isneginf(tb.numpy()), -np.inf, s)
            with np.errstate(divide="ignore"):
                want_lse = np.log(np.exp(s).sum(-1))
            fin = ~dead
            assert np.allclose(lse[fin], want_lse[fin], atol=1e-12)


def pin_forward_dropout(fwd):
    rng = np.random.default_rng(3)
    B, H, N, d = 1, 1, 24, 8
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    bias = make_bias(B, H, N, N, 4, hidden=0.1)
    base, lse0 = fwd(q, k, v, bias, 0.4, True)
    keep0 = M.dropout_keep(B, H, N, N, 0, seed=1)
    o0, l0 = fwd(q, k, v, bias, 0.4, True, keep0, 0)
    assert np.allclose(o0, base, atol=1e-12) and np.allclose(l0, lse0, atol=1e-12)
    p8 = 77
    acc = np.zeros_like(base)
    n = 4000
    for s in range(n):
        keep = M.dropout_keep(B, H, N, N, p8, seed=s)
        o, l = fwd(q, k, v, bias, 0.4, True, keep, p8)
        assert np.allclose(l, lse0, atol=1e-12)  # LSE is that of the weights before dropout
        acc += o
    assert np.abs(acc / n - base).max() < 0.05, np.abs(acc / n - base).max()


def pin_backward(bwd):
    rng = np.random.default_rng(5)
    B, H, N, d = 1, 2, 10, 6
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    bias = make_bias(1, H, N, N, 6, hidden=0.15)
    bias[..., np.arange(N), np.arange(N)] = 0.0  # every row keeps a key (torch's autograd is NaN otherwise)
    p8 = 64
    keep = M.dropout_keep(B, H, N, N, p8, seed=11)
    for causal in (False, True):
        for kp, pp in ((None, 0), (keep, p8)):
            dq, dk, dv = bwd(q, k, v, do, bias, 0.5, causal, kp, pp)
            tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
            s = 0.5 * tq @ tk.transpose(-1, -2) + torch.from_numpy(np.broadcast_to(bias, (B, H, N, N)).copy())
            if causal:
                s = s.masked_fill(~torch.from_numpy(A.causal_visible(N, N)), -math.inf)
            pr = torch.softmax(s, dim=-1)
            if kp is not None:
                pr = pr * torch.from_numpy(kp.astype(np.float64)) * (256.0 / (256.0 - pp))
            (pr @ tv).backward(torch.from_numpy(do))
            assert np.allclose(dq, tq.grad.numpy(), atol=1e-10)
            assert np.allclose(dk, tk.grad.numpy(), atol=1e-10)
            assert np.allclose(dv, tv.grad.numpy(), atol=1e-10)
    # Central finite differences of <dO, O> for a few entries of q and k (dropout on, causal).
    dq, dk, _ = bwd(q, k, v, do, bias, 0.5, True, keep, p8)
    eps = 1e-6
    for arr, grad in ((q, dq), (k, dk)):
        for idx in ((0, 0, 3, 1), (0, 1, 7, 5), (0, 1, 9, 0)):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = lambda a: (a, k, v) if arr is q else (q, a, v)
            fp = (M.attention_forward(*args(plus), bias, 0.5, True, keep, p8)[0] * do).sum()
            fm = (M.attention_forward(*args(minus), bias, 0.5, True, keep, p8)[0] * do).sum()
            assert abs((fp - fm) / (2 * eps) - grad[idx]) < 1e-6


# ----------------------------------------------------------------------------------------
# the pins
# ----------------------------------------------------------------------------------------
def test_philox_matches_library_and_known_answers():
    pin_philox(M.philox)


def test_dropout_decisions():
    pin_keep(M.dropout_keep)


def test_forward_with_bias_matches_library():
    pin_forward_bias(M.attention_forward)


def test_forward_with_dropout_is_unbiased():
    pin_forward_dropout(M.attention_forward)


def test_backward_matches_autograd_and_finite_differences():
    pin_backward(M.attention_backward)


def test_without_bias_and_dropout_equals_plain_oracle():
    rng = np.random.default_rng(8)
    q, k, v, do = (rng.standard_normal((1, 2, 33, 16)) for _ in range(4))
    for causal in (False, True):
        o, lse = M.attention_forward(q, k, v, None, 0.25, causal)
        ro, rl = A.attention_forward(q, k, v, 0.25, causal)
        assert np.allclose(o, ro, atol=1e-12) and np.allclose(lse, rl, atol=1e-12)
        g = M.attention_backward(q, k, v, do, None, 0.25, causal)
        rg = A.attention_backward(q, k, v, do, 0.25, causal)
        for a, b in zip(g, rg):
            assert np.allclose(a, b, atol=1e-12)


# ----------------------------------------------------------------------------------------
# mutation tests
# ----------------------------------------------------------------------------------------
def _philox_no_bump(counter, key, rounds=10, params=M.PHILOX4x32):
    return M.philox(counter, key, rounds=1, params=params) if rounds == 1 else \
        _philox_fixed_key(counter, key, rounds, params)


def _philox_fixed_key(counter, key, rounds, params):
    W = params["bits"]
    mask = (1 << W) - 1
    obj = W == 64
    c = [np.asarray(counter, dtype=object if obj else np.uint64)[..., i] for i in range(4)]
    k = [np.asarray(key, dtype=object if obj else np.uint64)[..., i] for i in range(2)]
    m0, m1 = (x if obj else np.uint64(x) for x in params["m"])
    sh, msk = (W, mask) if obj else (np.uint64(W), np.uint64(mask))
    for _ in range(rounds):
        p0, p1 = m0 * c[0], m1 * c[2]
        c = [(p1 >> sh) ^ c[1] ^ k[0], p1 & msk, (p0 >> sh) ^ c[3] ^ k[1], p0 & msk]
    return np.stack([np.asarray(x, dtype=object) for x in c], axis=-1) if obj else np.stack(c, axis=-1)


def _keep_transposed(B, H, Nq, Nk, p8, seed, offset=0, rows=None, b_only=None, h_only=None):
    """Query and key roles swapped in the counter."""
    full = M.dropout_keep(B, H, max(Nq, Nk), max(Nq, Nk), p8, seed, offset)
    full = np.swapaxes(full, -1, -2)[:, :, :Nq, :Nk]
    if b_only is not None:
        return full[b_only, h_only][np.arange(Nq) if rows is None else rows]
    return full


def _keep_strict(B, H, Nq, Nk, p8, seed, offset=0, rows=None, b_only=None, h_only=None):
    """u > p8 instead of u >= p8."""
    return M.dropout_keep(B, H, Nq, Nk, min(p8 + 1, 256), seed, offset, rows, b_only, h_only)


def _fwd_unscaled_dropout(q, k, v, bias, scale, causal, keep=None, p8=0):
    return M.attention_forward(q, k, v, bias, scale, causal, keep, 0 if keep is None else 0)


def _fwd_lse_after_dropout(q, k, v, bias, scale, causal, keep=None, p8=0):
    o, lse = M.attention_forward(q, k, v, bias, scale, causal, keep, p8)
    if keep is not None and p8 > 0:
        lse = lse + np.log(256.0 / (256.0 - p8))
    return o, lse


def _fwd_bias_after_softmax(q, k, v, bias, scale, causal, keep=None, p8=0):
    o, lse = M.attention_forward(q, k, v, None, scale, causal, keep, p8)
    if bias is not None:
        B, H = np.asarray(q).shape[:2]
        bb = np.where(np.isfinite(M.broadcast_bias(bias, B, H)), M.broadcast_bias(bias, B, H), 0)
        o = o + 0.01 * np.einsum("bhqk,bhkd->bhqd", bb, np.asarray(v, np.float64))
    return o, lse


def _bwd_dv_without_dropout(q, k, v, do, bias, scale, causal, keep=None, p8=0):
    dq, dk, dv = M.attention_backward(q, k, v, do, bias, scale, causal, keep, p8)
    _, _, dv0 = M.attention_backward(q, k, v, do, bias, scale, causal, None, 0)
    return dq, dk, dv0


def _bwd_dp_without_dropout(q, k, v, do, bias, scale, causal, keep=None, p8=0):
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    B, H = q.shape[:2]
    bb = None if bias is None else M.broadcast_bias(bias, B, H)
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)]
    for b in range(B):
        for h in range(H):
            s = M._scores(q[b, h], k[b, h], None if bb is None else bb[b, h], scale, causal)
            p, _ = A.softmax_rows(s)
            z = np.ones_like(p) if keep is None else keep[b, h] * (256.0 / (256.0 - p8))
            o = (p * z) @ v[b, h]
            dvec = (do[b, h] * o).sum(axis=1, keepdims=True)
            ds = p * (do[b, h] @ v[b, h].T - dvec)
            out[0][b, h], out[1][b, h], out[2][b, h] = scale * ds @ k[b, h], scale * ds.T @ q[b, h], (p * z).T @ do[b, h]
    return tuple(out)


@pytest.mark.parametrize("pin,impl", [
    (pin_philox, _philox_no_bump),
    (pin_keep, _keep_transposed),
    (pin_keep, _keep_strict),
    (pin_forward_dropout, _fwd_unscaled_dropout),
    (pin_forward_dropout, _fwd_lse_after_dropout),
    (pin_forward_bias, _fwd_bias_after_softmax),
    (pin_backward, _bwd_dv_without_dropout),
    (pin_backward, _bwd_dp_without_dropout),
])
def test_pins_reject_planted_mistakes(pin, impl):
    with pytest.raises(AssertionError):
        pin(impl)


def test_dropout_threshold_rounding():
    """p8 = floor(256 p + 1/2) of the float32 p: worked by hand, ties included.  A tie is a p whose
    256 p is an odd multiple of 1/2 and exact in float32 (p = 2.5 / 256 gives 3, not Python's
    round-half-even 2)."""
    cases = {0.0: 0, 0.1: 26, 0.5: 128, 0.9: 230, 2.5 / 256: 3, 3.5 / 256: 4, 0.5 / 256: 1,
             254.5 / 256: 255, 255.4 / 256: 255, 0.99: 253}
    for p, want in cases.items():
        assert M.dropout_p8(p) == want, (p, M.dropout_p8(p), want)
    with pytest.raises(ValueError):
        M.dropout_p8(1.0)
