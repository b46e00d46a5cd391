"""Backward parity: dQ, dK, dV from the CUDA path against the float64 oracle.

The CUDA backward consumes the CUDA forward's O and LSE (that is the method:
the backward recomputes P from the saved LSE).  The oracle recomputes
everything from the inputs in float64.
"""
import math
import os

import numpy as np
import pytest
import torch

from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
import gpu_common as gc
from tolerances import check_grad, check_lse, check_o, rel_l2

pytestmark = pytest.mark.gpu


def _full_check(B, H, Nq, Nk, d, causal, seed, peaked=0.0):
    x = W.make_attention_inputs(B, H, Nq, Nk, d, seed, peaked_frac=peaked)
    scale = 1.0 / math.sqrt(d)
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], causal, scale)
    dq, dk, dv = gc.gpu_backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal, scale)
    q, k, v, do = (gc.f64(x[n]) for n in ("q", "k", "v", "do"))
    rq, rk, rv = A.attention_backward(q, k, v, do, scale, causal)
    return (check_grad(gc.f64(dq), rq, "dQ"), check_grad(gc.f64(dk), rk, "dK"),
            check_grad(gc.f64(dv), rv, "dV"))


def test_tiny():
    c = W.TINY
    for causal in c.causal:
        _full_check(c.B, c.H, c.Nq, c.Nk, c.d, causal, c.seed)


@pytest.mark.parametrize("causal", [True, False])
def test_b2_h8_n1024_d64(causal):
    c = W.C2
    _full_check(c.B, c.H, c.Nq, c.Nk, c.d, causal, c.seed)


RAGGED = [
    (1, 1, 1, 1, 64, False),
    (1, 2, 127, 127, 64, True),
    (1, 1, 129, 129, 128, True),
    (2, 1, 300, 300, 128, False),
    (1, 3, 1000, 1000, 64, True),
    (1, 1, 200, 500, 128, True),
    (1, 1, 500, 200, 64, True),
    (1, 1, 500, 200, 128, False),
    (1, 2, 384, 640, 64, False),
    (3, 2, 256, 256, 128, True),
    (1, 1, 513, 1025, 128, True),
    (2, 40, 700, 1300, 128, True),
    (2, 40, 1300, 700, 64, True),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", RAGGED)
def test_ragged_and_edge_shapes(B, H, Nq, Nk, d, causal):
    _full_check(B, H, Nq, Nk, d, causal, seed=23 + Nq + Nk + d)


def test_per_row_errors_small():
    """Per-row relative error of dQ and per-key error of dK/dV stay small, not only the aggregate."""
    x = W.make_attention_inputs(1, 2, 640, 640, 128, 31)
    scale = 1 / math.sqrt(128)
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], True, scale)
    dq, dk, dv = gc.gpu_backward(x["q"], x["k"], x["v"], o, lse, x["do"], True, scale)
    q, k, v, do = (gc.f64(x[n]) for n in ("q", "k", "v", "do"))
    rq, rk, rv = A.attention_backward(q, k, v, do, scale, True)
    for g, r, name in ((gc.f64(dq), rq, "dQ"), (gc.f64(dk), rk, "dK"), (gc.f64(dv), rv, "dV")):
        num = np.linalg.norm(g - r, axis=-1)
        den = np.linalg.norm(r, axis=-1).mean()
        assert num.max() / den < 0.1, name


def test_peaked_keys_small():
    _full_check(1, 2, 1024, 1024, 128, True, seed=8, peaked=0.02)


def test_workspace_reuse_and_determinism_of_dk_dv():
    """dK/dV have no atomics: two runs agree bit for bit; dQ agrees within rounding."""
    x = W.make_attention_inputs(1, 4, 512, 512, 64, 41)
    scale = 0.125
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], True, scale)
    a = gc.gpu_backward(x["q"], x["k"], x["v"], o, lse, x["do"], True, scale)
    b = gc.gpu_backward(x["q"], x["k"], x["v"], o, lse, x["do"], True, scale)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert rel_l2(gc.f64(a[0]), gc.f64(b[0])) < 1e-2


def _oracle_workers():
    return max(1, min(16, os.cpu_count() or 1))


def _full_head_check(cfg, b, h, x, o_dev, lse_dev, grads_dev, scale, causal):
    """Whole head (b, h): O, LSE, dQ, dK and dV against the float64 oracle, every element.

    Returns the per-tensor relative L2 errors, the worst per-row dQ error (relative to the mean row
    norm of the oracle's dQ) and the errors of the first and last 64 keys' dK / dV rows (the first
    keys are seen by every query row: their key-block CTAs run the longest accumulation loops)."""
    from threadpoolctl import threadpool_limits
    q, k, v, do = (gc.f64(x[n][b, h]) for n in ("q", "k", "v", "do"))
    with threadpool_limits(1):
        ro, rl, rq, rk, rv = A.attention_backward_full_head(q, k, v, do, scale, causal, block=256,
                                                            workers=_oracle_workers())
    dq, dk, dv = (gc.f64(g[b, h]) for g in grads_dev)
    check_o(gc.f64(o_dev[b, h]), ro, f"O[{b},{h}]")
    check_lse(gc.f64(lse_dev[b, h]), rl, f"LSE[{b},{h}]")
    res = {"dQ": check_grad(dq, rq, f"dQ [{b},{h}]"), "dK": check_grad(dk, rk, f"dK [{b},{h}]"),
           "dV": check_grad(dv, rv, f"dV [{b},{h}]")}
    n = min(64, k.shape[0])
    for name, g, r in (("dK", dk, rk), ("dV", dv, rv)):
        res[f"{name}_first64"] = check_grad(g[:n], r[:n], f"{name} first keys [{b},{h}]")
        res[f"{name}_last64"] = check_grad(g[-n:], r[-n:], f"{name} last keys [{b},{h}]")
    row_err = np.linalg.norm(dq - rq, axis=-1)
    res["dQ_worst_row"] = float(row_err.max() / max(np.linalg.norm(rq, axis=-1).mean(), 1e-30))
    res["dQ_worst_row_index"] = int(row_err.argmax())
    return res


def _sampled_head_check(cfg, b, h, x, grads_dev, scale, causal, rows_per_head, seed, last_keys=64):
    """A head checked on samples: every one of the first 256 dQ rows (few visible keys, so they carry
    most of the norm under the causal mask) plus a uniform sample of the rest, weighted by the rows it
    stands for (an estimate of the whole-tensor relative L2), and the last keys' dK / dV rows."""
    q, k, v, do = (gc.f64(x[n][b, h]) for n in ("q", "k", "v", "do"))
    dq_h, dk_h, dv_h = (gc.f64(g[b, h]) for g in grads_dev)
    head_rows = min(256, cfg.Nq)
    first = np.arange(head_rows)
    rest = np.random.default_rng(seed + 97 * b + h).choice(
        np.arange(head_rows, cfg.Nq), size=min(rows_per_head, cfg.Nq - head_rows), replace=False)
    r_first = A.attention_backward_q_rows(q, k, v, do, first, scale, causal)
    r_rest = A.attention_backward_q_rows(q, k, v, do, np.sort(rest), scale, causal)
    w = (cfg.Nq - head_rows) / max(len(rest), 1)
    num = np.sum((dq_h[first] - r_first) ** 2) + w * np.sum((dq_h[np.sort(rest)] - r_rest) ** 2)
    den = np.sum(r_first ** 2) + w * np.sum(r_rest ** 2)
    est = math.sqrt(num / den)
    assert est <= 2e-2, f"dQ [{b},{h}]: estimated whole-tensor rel L2 {est:.3e}"
    keys = np.arange(cfg.Nk - last_keys, cfg.Nk)
    rk, rv = A.attention_backward_kv_rows(q, k, v, do, keys, scale, causal)
    check_grad(dk_h[keys], rk, f"dK last keys [{b},{h}]")
    check_grad(dv_h[keys], rv, f"dV last keys [{b},{h}]")
    # Properties at any size: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i.
    rms_k = math.sqrt(np.sum(dk_h ** 2))
    assert np.linalg.norm(dk_h.sum(0)) <= 0.05 * rms_k + 1e-6
    rms_v = math.sqrt(np.sum(dv_h ** 2))
    assert np.linalg.norm(dv_h.sum(0) - do.sum(0)) <= 0.02 * rms_v + 1e-6


def _full_size_check(cfg, causal, rows_per_head, seed):
    """Heads (0, 0) and (B-1, H-1) whole, every element; every other head on samples."""
    x = W.make_config_inputs(cfg)
    scale = cfg.scale
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], causal, scale)
    grads = gc.gpu_backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal, scale)
    for g in grads:
        assert torch.isfinite(g).all()
    full = [(0, 0), (cfg.B - 1, cfg.H - 1)]
    for b, h in full:
        res = _full_head_check(cfg, b, h, x, o, lse, grads, scale, causal)
        print(f"GRAD-PARITY {cfg.name} b={b} h={h} " + " ".join(
            f"{k}={v:.3e}" if isinstance(v, float) else f"{k}={v}" for k, v in res.items()))
    for b in range(cfg.B):
        for h in range(cfg.H):
            if (b, h) not in full:
                _sampled_head_check(cfg, b, h, x, grads, scale, causal, rows_per_head, seed)


@pytest.mark.parametrize("cfg", W.SWEEP, ids=lambda c: c.name)
def test_sweep_full_size(cfg):
    _full_size_check(cfg, True, rows_per_head=64, seed=13)


def test_long_context_full_size():
    _full_size_check(W.LONG, True, rows_per_head=64, seed=17)


def test_no_query_rows_gives_zero_dk_dv():
    """Nq = 0 with keys: no score touches any key, so dK = dV = 0 (and nothing else is read)."""
    B, H, Nk, d = 1, 2, 200, 64
    k = torch.randn(B, H, Nk, d, device=gc.DEV).bfloat16()
    v = torch.randn(B, H, Nk, d, device=gc.DEV).bfloat16()
    q = torch.empty(B, H, 0, d, device=gc.DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, H, 0, device=gc.DEV, dtype=torch.float32)
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    ws = torch.empty(256, dtype=torch.uint8, device=gc.DEV)
    gc.fa.fa_bwd(q, k, v, q, q, lse, torch.empty_like(q), dk, dv, ws, causal=True)
    torch.cuda.synchronize()
    assert gc.fa.fa_get_device_error() == 0
    assert torch.all(dk == 0) and torch.all(dv == 0)
