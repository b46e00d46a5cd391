"""Additive bias and dropout (fa_fwd_ext / fa_bwd_ext) against the oracle.

* The dropout decisions are integer work: with Q = 0 the weights are uniform, and one-hot V rows
  (forward) or one-hot dO rows (backward, through dV) make each kept / dropped entry readable, so
  the pattern is compared with the oracle's Philox decisions exactly.
* Outputs use the forward and backward tolerances of the plain path (max |dO| <= 1e-2 or within
  half a bf16 ulp beyond it, |dLSE| <= 1e-3, gradients relative L2 <= 2e-2) against the float64
  oracle given the same bias values and the same keep mask.
"""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
from oracle import masked as M
import gpu_common as gc
from tolerances import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu

SEED, OFFSET = 0x5EED_1234_ABCD, 7


def make_bias(bB, bH, Nq, Nk, seed, hidden=0.1, dead_rows=()):
    g = torch.Generator().manual_seed(seed)
    b = torch.randn(bB, bH, Nq, Nk, generator=g) * 2.0
    b[torch.rand(bB, bH, Nq, Nk, generator=g) < hidden] = -math.inf
    for r in dead_rows:
        b[:, :, r, :] = -math.inf
    return b.to(torch.bfloat16)


def run_ext(x, bias, causal, scale, p, with_bwd=True):
    qd, kd, vd, dod = gc.to_dev(x["q"], x["k"], x["v"], x["do"])
    bd = bias.to(gc.DEV) if bias is not None else None
    B, H, Nq, d = qd.shape
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, Nq, dtype=torch.float32, device=gc.DEV)
    fa.fa_fwd_ext(qd, kd, vd, o, lse, bd, causal, scale, p, SEED, OFFSET)
    grads = None
    if with_bwd:
        dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        ws = torch.empty(max(fa.fa_bwd_workspace_size(B, H, Nq, d), 256), dtype=torch.uint8, device=gc.DEV)
        fa.fa_bwd_ext(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, bd, causal, scale, p, SEED, OFFSET)
        grads = (dq, dk, dv)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return o, lse, grads


CASES = [
    # B, H, Nq, Nk, d, causal, bias dims (None = no bias), dropout p
    (1, 2, 128, 128, 64, False, (1, 2), 0.0),
    (2, 4, 512, 512, 128, True, (1, 4), 0.0),
    (1, 2, 300, 520, 64, True, (1, 2), 0.1),      # ragged query and key tiles
    (2, 2, 256, 256, 64, False, None, 0.2),       # dropout only
    (1, 2, 1024, 1024, 128, True, (1, 1), 0.15),
    (2, 3, 200, 128, 64, True, (2, 3), 0.0),      # Nq > Nk: leading rows see no key
    (1, 2, 384, 640, 128, False, (1, 2), 0.3),    # rows masked entirely by the bias
    (4, 16, 1024, 1024, 64, True, (1, 16), 0.1),  # two query tiles per CTA
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,bdims,p", CASES)
def test_ext_matches_oracle(B, H, Nq, Nk, d, causal, bdims, p):
    x = W.make_attention_inputs(B, H, Nq, Nk, d, 60 + Nq + Nk + d)
    bias = make_bias(*bdims, Nq, Nk, 5 + Nq, dead_rows=(3, 77) if Nq == 384 else ()) if bdims else None
    scale = 1.0 / math.sqrt(d)
    o, lse, (dq, dk, dv) = run_ext(x, bias, causal, scale, p)
    p8 = M.dropout_p8(p)
    keep = M.dropout_keep(B, H, Nq, Nk, p8, SEED, OFFSET) if p8 else None
    bb = None if bias is None else bias.double().numpy()
    q, k, v, do = (gc.f64(x[n]) for n in ("q", "k", "v", "do"))
    ro, rl = M.attention_forward(q, k, v, bb, scale, causal, keep, p8)
    check_o(gc.f64(o), ro)
    check_lse(gc.f64(lse), rl)
    rq, rk, rv = M.attention_backward(q, k, v, do, bb, scale, causal, keep, p8)
    check_grad(gc.f64(dq), rq, "dQ")
    check_grad(gc.f64(dk), rk, "dK")
    check_grad(gc.f64(dv), rv, "dV")


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9, 2.5 / 256])   # 2.5 / 256: a rounding tie (p8 = 3)
def test_dropout_pattern_is_the_oracle_one(p):
    """Q = 0 (uniform weights, no bias), one-hot rows: the forward's O and the backward's dV show each
    decision of every (batch, head) exactly."""
    B, H, N, d = 2, 3, 64, 64
    p8 = M.dropout_p8(p)
    eye = torch.eye(N, d, dtype=torch.bfloat16).expand(B, H, N, d).contiguous()
    x = {"q": torch.zeros(B, H, N, d, dtype=torch.bfloat16), "k": W.make_attention_inputs(B, H, N, N, d, 3)["k"],
         "v": eye, "do": eye}
    o, _, (_, _, dv) = run_ext(x, None, False, 0.125, p)
    keep = M.dropout_keep(B, H, N, N, p8, SEED, OFFSET)
    fwd_kept = gc.f64(o) != 0          # O[i, j] = keep_ij * (256 / (256 - p8)) / N
    bwd_kept = gc.f64(dv).transpose(0, 1, 3, 2) != 0  # dV[j, i] = keep_ij * (256 / (256 - p8)) / N
    assert np.array_equal(fwd_kept, keep), int((fwd_kept != keep).sum())
    assert np.array_equal(bwd_kept, keep), int((bwd_kept != keep).sum())
    want = 256.0 / (256 - p8) / N
    assert np.allclose(gc.f64(o)[keep], want, rtol=2 ** -8)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (2, 32, 600, 128, True),   # enough CTAs for two 128-row query tiles per CTA; ragged last tile
    (1, 2, 600, 64, False),    # one query tile per CTA, its key tiles split between the two groups
    (1, 3, 384, 128, False),
])
def test_dropout_pattern_across_tiles(B, H, N, d, causal):
    """Every decision of an N x N pattern, across query-tile and key-tile boundaries, equals the oracle's.

    Q = 0 makes the weights uniform over the visible keys.  V one-hot on a window of d keys makes the
    forward's O show the decisions of those keys (O[i, c] != 0 iff key w0 + c is kept and visible),
    and dO one-hot on a window of d queries makes the backward's dV show the decisions of those
    queries (dV[j, c] != 0 iff entry (w0 + c, j) is kept and visible); windows cover every key and
    every query."""
    p = 0.3
    p8 = M.dropout_p8(p)
    keep = M.dropout_keep(B, H, N, N, p8, SEED, OFFSET)
    vis = A.causal_visible(N, N) if causal else np.ones((N, N), dtype=bool)
    want = keep & vis[None, None]
    k = W.make_attention_inputs(B, H, N, N, d, 3, with_do=False)["k"]
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    fwd_seen = np.zeros((B, H, N, N), dtype=bool)
    bwd_seen = np.zeros((B, H, N, N), dtype=bool)
    for w0 in range(0, N, d):
        kw = min(d, N - w0)
        onehot = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
        onehot[:, :, torch.arange(w0, w0 + kw), torch.arange(kw)] = 1.0
        o, _, (_, _, dv) = run_ext({"q": q, "k": k, "v": onehot, "do": onehot}, None, causal, 0.125, p)
        fwd_seen[:, :, :, w0:w0 + kw] = gc.f64(o)[..., :kw] != 0
        bwd_seen[:, :, w0:w0 + kw, :] = (gc.f64(dv)[..., :kw] != 0).transpose(0, 1, 3, 2)
    assert np.array_equal(fwd_seen, want), int((fwd_seen != want).sum())
    assert np.array_equal(bwd_seen, want), int((bwd_seen != want).sum())


def test_without_bias_or_dropout_matches_the_plain_path():
    B, H, N, d = 2, 2, 300, 128
    x = W.make_attention_inputs(B, H, N, N, d, 17)
    scale = 1.0 / math.sqrt(d)
    o, lse, (dq, dk, dv) = run_ext(x, None, True, scale, 0.0)
    qd, kd, vd, dod = gc.to_dev(x["q"], x["k"], x["v"], x["do"])
    o2, lse2 = fa.attention_forward(qd, kd, vd, causal=True, scale=scale)
    g2 = fa.attention_backward(qd, kd, vd, o2, lse2, dod, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 2 ** -7
    assert (lse - lse2).abs().max().item() <= 1e-5
    for a, b in zip((dq, dk, dv), g2):
        assert (a.float() - b.float()).norm().item() <= 1e-2 * b.float().norm().item()


def test_other_seed_or_offset_changes_the_pattern():
    B, H, N, d = 1, 1, 64, 64
    eye = torch.eye(N, d, dtype=torch.bfloat16).expand(B, H, N, d).contiguous()
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device=gc.DEV)
    k = torch.randn(B, H, N, d, device=gc.DEV).to(torch.bfloat16)
    v = eye.to(gc.DEV)
    outs = []
    for seed, off in ((1, 0), (2, 0), (1, 1)):
        o = torch.empty_like(q)
        lse = torch.empty(B, H, N, device=gc.DEV)
        fa.fa_fwd_ext(q, k, v, o, lse, None, False, 0.125, 0.5, seed, off)
        outs.append(o != 0)
    torch.cuda.synchronize()
    assert not torch.equal(outs[0], outs[1]) and not torch.equal(outs[0], outs[2])
    want = M.dropout_keep(B, H, N, N, 128, 2, 0)
    assert np.array_equal(outs[1].cpu().numpy(), want)
