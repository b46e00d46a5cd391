"""Pins for the float64 oracle (CPU only).

Each check ties the oracle to something other than itself: hand-derived
values, closed forms, invariants of the definition, finite differences, or a
library routine (torch's float64 CPU attention).  The mutation tests at the end
plant plausible mistakes in copies of the oracle and assert that the pins
reject each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(x):
    """Evaluate a golden-file entry: a number or a small expression in ln2/ln3/..."""
    if isinstance(x, (int, float)):
        return float(x)
    env = {"ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4), "ln5": math.log(5)}
    return float(eval(x, {"__builtins__": {}}, env))


def _arr(a):
    return np.array([[_val(e) for e in row] if isinstance(row, list) else _val(row) for row in a])


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ----------------------------------------------------------------------------------------
# pin functions (take an implementation so the mutation tests can reuse them)
# ----------------------------------------------------------------------------------------

def pin_golden_forward(fwd):
    g = json.load(open(os.path.join(GOLDEN, "hand_d1_n2.json")))
    q, k, v = _arr(g["inputs"]["q"]), _arr(g["inputs"]["k"]), _arr(g["inputs"]["v"])
    ok = True
    for mode, causal in (("noncausal", False), ("causal", True)):
        o, lse = fwd(q, k, v, g["inputs"]["scale"], causal)
        ok &= np.allclose(o, _arr(g[mode]["o"]), rtol=0, atol=1e-13)
        ok &= np.allclose(lse, _arr(g[mode]["lse"]), rtol=0, atol=1e-13)
    return bool(ok)


def pin_golden_backward(bwd):
    g = json.load(open(os.path.join(GOLDEN, "hand_d1_n2.json")))
    q, k, v, do = (_arr(g["inputs"][n]) for n in ("q", "k", "v", "do"))
    dq, dk, dv = bwd(q, k, v, do, g["inputs"]["scale"], False)
    exp = g["noncausal"]
    return bool(np.allclose(dq, _arr(exp["dq"]), atol=1e-13) and
                np.allclose(dk, _arr(exp["dk"]), atol=1e-13) and
                np.allclose(dv, _arr(exp["dv"]), atol=1e-13))


def pin_q_zero(fwd):
    """Q = 0: every visible key gets equal weight -> mean of visible V rows; LSE = ln(#visible)."""
    n, d = 9, 5
    k, v = _rand((n, d), 1), _rand((n, d), 2)
    q = np.zeros((n, d))
    o, lse = fwd(q, k, v, 0.37, False)
    ok = np.allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-13)
    ok &= np.allclose(lse, np.log(n), atol=1e-13)
    o, lse = fwd(q, k, v, 0.37, True)
    cum = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
    ok &= np.allclose(o, cum, atol=1e-13)
    ok &= np.allclose(lse, np.log(np.arange(1, n + 1)), atol=1e-13)
    return bool(ok)


def pin_identical_keys(fwd):
    n, d = 7, 4
    q, v = _rand((5, d), 3), _rand((n, d), 4)
    k = np.broadcast_to(_rand((1, d), 5), (n, d)).copy()
    o, _ = fwd(q, k, v, 0.5, False)
    return bool(np.allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-12))


def pin_causal_row0(fwd):
    n, d = 6, 3
    q, k, v = _rand((n, d), 6), _rand((n, d), 7), _rand((n, d), 8)
    o, lse = fwd(q, k, v, 0.9, True)
    return bool(np.array_equal(o[0], v[0]) and abs(lse[0] - 0.9 * q[0] @ k[0]) < 1e-13)


def pin_permutation(fwd):
    n, d = 8, 4
    q, k, v = _rand((5, d), 9), _rand((n, d), 10), _rand((n, d), 11)
    perm = np.random.default_rng(12).permutation(n)
    o1, l1 = fwd(q, k, v, 0.7, False)
    o2, l2 = fwd(q, k[perm], v[perm], 0.7, False)
    return bool(np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13))


def pin_key_shift(fwd):
    """Adding c to every key row leaves O unchanged and shifts LSE_i by scale * q_i . c."""
    n, d = 8, 4
    q, k, v = _rand((6, d), 13), _rand((n, d), 14), _rand((n, d), 15)
    c = _rand((d,), 16)
    for causal in (False, True):
        o1, l1 = fwd(q, k, v, 0.6, causal)
        o2, l2 = fwd(q, k + c, v, 0.6, causal)
        if not (np.allclose(o1, o2, atol=1e-12) and np.allclose(l2 - l1, 0.6 * q @ c, atol=1e-12)):
            return False
    return True


def pin_torch_sdpa(fwd):
    """Library cross-check: torch's attention on CPU in float64 (explicit bottom-right mask)."""
    ok = True
    for (nq, nk, causal) in ((7, 7, False), (7, 7, True), (5, 11, True), (11, 5, False)):
        d = 6
        q, k, v = _rand((nq, d), 17), _rand((nk, d), 18), _rand((nk, d), 19)
        o, lse = fwd(q, k, v, 0.41, causal)
        tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
        mask = None
        if causal:
            mask = torch.ones(nq, nk, dtype=torch.bool).tril(diagonal=nk - nq)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.41)
        s = 0.41 * (tq @ tk.transpose(-1, -2))
        if causal:
            s = s.masked_fill(~mask, float("-inf"))
        ref_lse = torch.logsumexp(s, dim=-1)
        ok &= np.allclose(o, ref[0, 0].numpy(), atol=1e-12)
        ok &= np.allclose(lse, ref_lse[0, 0].numpy(), atol=1e-12)
    return bool(ok)


def pin_bottom_right(fwd):
    """Nq < Nk causal equals the last Nq rows of the square causal problem."""
    nk, nq, d = 10, 4, 3
    qf, k, v = _rand((nk, d), 20), _rand((nk, d), 21), _rand((nk, d), 22)
    o_full, l_full = fwd(qf, k, v, 0.8, True)
    o, l = fwd(qf[-nq:], k, v, 0.8, True)
    return bool(np.allclose(o, o_full[-nq:], atol=1e-13) and np.allclose(l, l_full[-nq:], atol=1e-13))


def pin_rows_sum(fwd):
    """O for V = identity is P itself: rows non-negative and summing to one."""
    n, d = 6, 6
    q, k = _rand((n, d), 23), _rand((n, d), 24)
    ok = True
    for causal in (False, True):
        p, _ = fwd(q, k, np.eye(n), 0.5, causal)
        ok &= bool(np.all(p >= 0)) and np.allclose(p.sum(1), 1.0, atol=1e-14)
        if causal:
            ok &= bool(np.all(np.triu(p, 1) == 0))
    return bool(ok)


FORWARD_PINS = [pin_golden_forward, pin_q_zero, pin_identical_keys, pin_causal_row0,
                pin_permutation, pin_key_shift, pin_torch_sdpa, pin_bottom_right, pin_rows_sum]


def finite_difference_grads(fwd, q, k, v, do, scale, causal, h=1e-6):
    """Central differences of L = <dO, O(q, k, v)> with respect to every input entry."""
    def loss(qq, kk, vv):
        return float(np.sum(do * fwd(qq, kk, vv, scale, causal)[0]))
    grads = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros_like(base[which])
        for idx in np.ndindex(g.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


def pin_finite_differences(bwd, fwd=A.attention_forward_head):
    ok = True
    for (nq, nk, d, causal) in ((4, 4, 3, False), (4, 4, 3, True), (3, 5, 2, True), (5, 3, 2, False)):
        q, k, v, do = _rand((nq, d), 30), _rand((nk, d), 31), _rand((nk, d), 32), _rand((nq, d), 33)
        fd = finite_difference_grads(fwd, q, k, v, do, 0.55, causal)
        an = bwd(q, k, v, do, 0.55, causal)
        for a, b in zip(an, fd):
            ok &= np.allclose(a, b, rtol=1e-7, atol=1e-8)
    return bool(ok)


def pin_torch_autograd(bwd):
    ok = True
    for (nq, nk, causal) in ((6, 6, False), (6, 6, True), (4, 9, True)):
        d = 5
        q, k, v, do = _rand((nq, d), 40), _rand((nk, d), 41), _rand((nk, d), 42), _rand((nq, d), 43)
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        mask = torch.ones(nq, nk, dtype=torch.bool).tril(diagonal=nk - nq) if causal else None
        o = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None],
                                                             attn_mask=mask, scale=0.3)[0]
        o.backward(torch.from_numpy(do))
        dq, dk, dv = bwd(q, k, v, do, 0.3, causal)
        ok &= np.allclose(dq, tq.grad.numpy(), atol=1e-12)
        ok &= np.allclose(dk, tk.grad.numpy(), atol=1e-12)
        ok &= np.allclose(dv, tv.grad.numpy(), atol=1e-12)
    return bool(ok)


def pin_grad_sums(bwd):
    """sum_j dK_j = 0 (each dS row sums to zero) and sum_j dV_j = sum_i dO_i."""
    n, d = 9, 4
    q, k, v, do = _rand((n, d), 50), _rand((n, d), 51), _rand((n, d), 52), _rand((n, d), 53)
    ok = True
    for causal in (False, True):
        dq, dk, dv = bwd(q, k, v, do, 0.45, causal)
        ok &= np.allclose(dk.sum(0), 0.0, atol=1e-12)
        ok &= np.allclose(dv.sum(0), do.sum(0), atol=1e-12)
    return bool(ok)


BACKWARD_PINS = [pin_golden_backward, pin_finite_differences, pin_torch_autograd, pin_grad_sums]


# ----------------------------------------------------------------------------------------
# the oracle passes every pin
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("pin", FORWARD_PINS, ids=lambda f: f.__name__)
def test_forward_pin(pin):
    assert pin(A.attention_forward_head)


@pytest.mark.parametrize("pin", BACKWARD_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    assert pin(A.attention_backward_head)


def test_golden_two_block_merge():
    g = json.load(open(os.path.join(GOLDEN, "hand_two_block_merge.json")))
    x1 = np.array([_val(e) for e in g["x1"]])
    x2 = np.array([_val(e) for e in g["x2"]])
    m1, f1, l1 = A.safe_softmax_stats(x1)
    m2, f2, l2 = A.safe_softmax_stats(x2)
    assert abs(m1 - _val(g["block1"]["m"])) < 1e-15 and abs(l1 - _val(g["block1"]["l"])) < 1e-15
    assert np.allclose(f1, [_val(e) for e in g["block1"]["f"]], atol=1e-15)
    assert abs(m2 - _val(g["block2"]["m"])) < 1e-15 and abs(l2 - _val(g["block2"]["l"])) < 1e-15
    m, f, l = A.merge_two_blocks(m1, f1, l1, m2, f2, l2)
    assert abs(m - _val(g["merged"]["m"])) < 1e-15
    assert np.allclose(f, [_val(e) for e in g["merged"]["f"]], atol=1e-15)
    assert abs(l - _val(g["merged"]["l"])) < 1e-15
    assert np.allclose(f / l, [_val(e) for e in g["merged"]["softmax"]], atol=1e-15)


@pytest.mark.parametrize("split", [1, 2, 7, 15])
def test_merge_identity_random(split):
    x = _rand((5, 16), 60) * 4
    x[1, :split] = -np.inf           # a fully masked first block in row 1
    x[2, split:] = -np.inf           # a fully masked second block in row 2
    m, f, l = A.safe_softmax_stats(x)
    mm, ff, ll = A.merge_two_blocks(*A.safe_softmax_stats(x[:, :split]), *A.safe_softmax_stats(x[:, split:]))
    assert np.array_equal(m, mm)
    assert np.allclose(f, ff, rtol=1e-14, atol=0)
    assert np.allclose(l, ll, rtol=1e-14, atol=0)
    sm = np.exp(x - x.max(1, keepdims=True))
    assert np.allclose(ff / ll[:, None], sm / sm.sum(1, keepdims=True), rtol=1e-14, atol=1e-300)


def test_scale_equivalence():
    q, k, v = _rand((5, 4), 70), _rand((6, 4), 71), _rand((6, 4), 72)
    o1, l1 = A.attention_forward_head(q, k, v, 0.5, True)
    o2, l2 = A.attention_forward_head(2.0 * q, k, v, 0.25, True)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)


def test_fully_masked_rows():
    """Causal with Nq > Nk: the first Nq - Nk rows see no key -> O = 0, LSE = -inf."""
    nq, nk, d = 7, 4, 3
    q, k, v = _rand((nq, d), 80), _rand((nk, d), 81), _rand((nk, d), 82)
    o, lse = A.attention_forward_head(q, k, v, 0.5, True)
    assert np.all(o[:3] == 0) and np.all(np.isneginf(lse[:3]))
    o_sq, l_sq = A.attention_forward_head(q[3:], k, v, 0.5, True)
    assert np.allclose(o[3:], o_sq, atol=1e-14) and np.allclose(lse[3:], l_sq, atol=1e-14)
    do = _rand((nq, d), 83)
    dq, dk, dv = A.attention_backward_head(q, k, v, do, 0.5, True)
    assert np.all(dq[:3] == 0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


def test_empty_keys():
    q = _rand((3, 4), 90)
    o, lse = A.attention_forward_head(q, np.zeros((0, 4)), np.zeros((0, 4)), 0.5, False)
    assert o.shape == (3, 4) and np.all(o == 0) and np.all(np.isneginf(lse))


def test_batched_matches_heads():
    q, k, v, do = (_rand((2, 3, 5, 4), s) for s in (100, 101, 102, 103))
    o, lse = A.attention_forward(q, k, v, 0.5, True)
    dq, dk, dv = A.attention_backward(q, k, v, do, 0.5, True)
    for b in range(2):
        for h in range(3):
            oh, lh = A.attention_forward_head(q[b, h], k[b, h], v[b, h], 0.5, True)
            assert np.array_equal(o[b, h], oh) and np.array_equal(lse[b, h], lh)
            g = A.attention_backward_head(q[b, h], k[b, h], v[b, h], do[b, h], 0.5, True)
            assert np.array_equal(dq[b, h], g[0]) and np.array_equal(dk[b, h], g[1])
            assert np.array_equal(dv[b, h], g[2])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(37, 37), (20, 45), (45, 20)])
def test_restricted_functions_match_full(causal, nq, nk):
    d = 8
    q, k, v, do = _rand((nq, d), 110), _rand((nk, d), 111), _rand((nk, d), 112), _rand((nq, d), 113)
    o, lse = A.attention_forward_head(q, k, v, 0.3, causal)
    dq, dk, dv = A.attention_backward_head(q, k, v, do, 0.3, causal)
    rows = np.array([0, 3, nq - 1])
    o_r, l_r = A.attention_forward_rows(q, k, v, rows, 0.3, causal, block=2)
    assert np.allclose(o_r, o[rows], atol=1e-13)
    assert np.allclose(l_r, lse[rows], atol=1e-13, equal_nan=False) or np.array_equal(l_r, lse[rows])
    assert np.allclose(A.attention_backward_q_rows(q, k, v, do, rows, 0.3, causal, block=2), dq[rows], atol=1e-12)
    keys = np.array([nk - 5, nk - 2, nk - 1])
    dk_r, dv_r = A.attention_backward_kv_rows(q, k, v, do, keys, 0.3, causal, block=3)
    assert np.allclose(dk_r, dk[keys], atol=1e-12)
    assert np.allclose(dv_r, dv[keys], atol=1e-12)


def test_decode_oracle():
    """Decode equals the Nq = 1 forward on the first L_b keys; slots beyond L_b are never read."""
    B, H, L, d = 3, 2, 12, 4
    q = _rand((B, H, 1, d), 120)
    kc, vc = _rand((B, H, L, d), 121), _rand((B, H, L, d), 122)
    lens = np.array([1, 7, 12])
    for b in range(B):
        kc[b, :, lens[b]:] = np.nan
        vc[b, :, lens[b]:] = np.nan
    o, lse = A.decode_forward(q, kc, vc, lens, 0.5)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    for b in range(B):
        for h in range(H):
            oh, lh = A.attention_forward_head(q[b, h], kc[b, h, :lens[b]], vc[b, h, :lens[b]], 0.5, False)
            assert np.allclose(o[b, h], oh[0], atol=1e-14) and abs(lse[b, h] - lh[0]) < 1e-14
    assert np.allclose(o[0], vc[0, :, 0], atol=0)   # one key: O = V[0]


# ----------------------------------------------------------------------------------------
# mutation tests: each planted mistake must fail at least one pin
# ----------------------------------------------------------------------------------------

def _fwd_mutant(kind):
    def f(q, k, v, scale, causal):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        sc = 1.0 if kind == "no_scale" else scale
        s = sc * (q @ k.T)
        if causal:
            nq, nk = s.shape
            off = 0 if kind == "top_left_mask" else nk - nq
            if kind == "strict_mask":
                vis = np.arange(nk)[None, :] < np.arange(nq)[:, None] + off
            else:
                vis = np.arange(nk)[None, :] <= np.arange(nq)[:, None] + off
            s = np.where(vis, s, -np.inf)
        m = s.max(axis=0 if kind == "softmax_wrong_axis" else 1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0)
        e = np.exp(s - m)
        l = e.sum(axis=0 if kind == "softmax_wrong_axis" else 1, keepdims=True)
        p = e / np.where(l > 0, l, 1)
        if kind == "lse_log2":
            lse = (m + np.log2(np.where(l > 0, l, 1)))[:, 0]
        elif kind == "lse_without_max":
            lse = np.log(np.where(l > 0, l, 1))[:, 0]
        else:
            lse = (m + np.log(np.where(l > 0, l, 1)))[:, 0]
        lse = np.where(l[:, 0] > 0, lse, -np.inf) if kind != "softmax_wrong_axis" else lse
        o = (p.T @ v) if (kind == "transposed_p" and p.shape[0] == p.shape[1]) else p @ v
        return o, lse
    return f


def _bwd_mutant(kind):
    def g(q, k, v, do, scale, causal):
        q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
        s = A.scaled_scores(q, k, scale, causal)
        p, _ = A.softmax_rows(s)
        o = p @ v
        dv = p.T @ do
        dp = do @ v.T
        drow = np.sum(do * o, axis=-1)
        if kind == "missing_d":
            ds = p * dp
        elif kind == "wrong_sign":
            ds = p * (drow[:, None] - dp)
        elif kind == "d_from_p":
            ds = p * (dp - p.sum(1)[:, None])
        else:
            ds = p * (dp - drow[:, None])
        dq = (1.0 if kind == "dq_no_scale" else scale) * (ds @ k)
        dk = scale * ((ds if kind == "dk_untransposed" and ds.shape[0] == ds.shape[1] else ds.T) @ q)
        if kind == "dv_untransposed" and p.shape[0] == p.shape[1]:
            dv = p @ do
        return dq, dk, dv
    return g


@pytest.mark.parametrize("kind", ["no_scale", "top_left_mask", "strict_mask", "softmax_wrong_axis",
                                  "lse_log2", "lse_without_max", "transposed_p"])
def test_forward_mutant_is_caught(kind):
    mutant = _fwd_mutant(kind)
    assert not all(pin(mutant) for pin in FORWARD_PINS), kind


@pytest.mark.parametrize("kind", ["missing_d", "wrong_sign", "d_from_p", "dq_no_scale",
                                  "dk_untransposed", "dv_untransposed"])
def test_backward_mutant_is_caught(kind):
    mutant = _bwd_mutant(kind)
    assert not all(pin(mutant) for pin in BACKWARD_PINS), kind


def test_correct_mutant_template_passes():
    """The mutant templates with no planted mistake pass every pin (the pins are not vacuous)."""
    assert all(pin(_fwd_mutant("none")) for pin in FORWARD_PINS)
    assert all(pin(_bwd_mutant("none")) for pin in BACKWARD_PINS)


# ----------------------------------------------------------------------------------------
# the whole-head backward by row blocks (used for full-size gradient parity) is pinned by the
# same pins as the plain backward: finite differences, torch autograd, the gradient sums and the
# hand-worked golden, at block sizes that cut the rows (and, under the causal mask, the key
# range each block keeps) at every position
# ----------------------------------------------------------------------------------------
def _full_head_bwd(block, workers):
    def bwd(q, k, v, do, scale, causal):
        return A.attention_backward_full_head(q, k, v, do, scale, causal, block=block, workers=workers)[2:]
    return bwd


def _full_head_fwd(block):
    def fwd(q, k, v, scale, causal):
        do = np.zeros((q.shape[0], v.shape[1]))
        return A.attention_backward_full_head(q, k, v, do, scale, causal, block=block)[:2]
    return fwd


@pytest.mark.parametrize("block,workers", [(1, 1), (2, 1), (3, 2), (64, 1)])
@pytest.mark.parametrize("pin", BACKWARD_PINS, ids=lambda f: f.__name__)
def test_full_head_backward_pin(pin, block, workers):
    assert pin(_full_head_bwd(block, workers))


@pytest.mark.parametrize("block", [1, 2, 5])
@pytest.mark.parametrize("pin", FORWARD_PINS, ids=lambda f: f.__name__)
def test_full_head_forward_pin(pin, block):
    assert pin(_full_head_fwd(block))


def test_full_head_rows_with_no_key():
    """Causal, Nq > Nk: blocks whose rows see no key give O = 0, LSE = -inf, dQ = 0."""
    nq, nk, d = 9, 4, 3
    q, k, v, do = _rand((nq, d), 130), _rand((nk, d), 131), _rand((nk, d), 132), _rand((nq, d), 133)
    o, lse, dq, dk, dv = A.attention_backward_full_head(q, k, v, do, 0.5, True, block=2)
    ro, rl = A.attention_forward_head(q, k, v, 0.5, True)
    rq, rk, rv = A.attention_backward_head(q, k, v, do, 0.5, True)
    assert np.all(o[:5] == 0) and np.all(np.isneginf(lse[:5])) and np.all(dq[:5] == 0)
    assert np.allclose(o, ro, atol=1e-14) and np.array_equal(np.isneginf(lse), np.isneginf(rl))
    assert np.allclose(dq, rq, atol=1e-13) and np.allclose(dk, rk, atol=1e-13) and np.allclose(dv, rv, atol=1e-13)


def test_full_head_mutant_dropping_the_last_visible_key_is_caught():
    """A plausible slip in the causal key range of a row block (one key short) fails the autograd pin."""
    real = A.attention_row_block

    def short(q_head, k_head, v_head, do_head, r0, r1, scale, causal):
        nq, nk = q_head.shape[0], k_head.shape[0]
        kend = nk if not causal else max(0, min(nk, (r1 - 1) + (nk - nq)))   # one key short
        q, k, v, do = q_head[r0:r1], k_head[:kend], v_head[:kend], do_head[r0:r1]
        s = scale * (q @ k.T)
        if causal:
            s = np.where(A.causal_visible(nq, nk, rows=np.arange(r0, r1), cols=np.arange(kend)), s, -np.inf)
        p, lse = A.softmax_rows(s)
        o = p @ v
        ds = p * (do @ v.T - np.sum(do * o, axis=-1)[:, None])
        return o, lse, scale * (ds @ k), scale * (ds.T @ q), p.T @ do

    A.attention_row_block = short
    try:
        assert not pin_torch_autograd(_full_head_bwd(2, 1))
    finally:
        A.attention_row_block = real
