"""Forward parity: the CUDA path (through the C ABI) against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
import gpu_common as gc
from tolerances import check_lse, check_o

pytestmark = pytest.mark.gpu


def _full_check(B, H, Nq, Nk, d, causal, seed, peaked=0.0):
    x = W.make_attention_inputs(B, H, Nq, Nk, d, seed, peaked_frac=peaked, with_do=False)
    scale = 1.0 / math.sqrt(d)
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], causal, scale)
    o_ref, lse_ref = A.attention_forward(gc.f64(x["q"]), gc.f64(x["k"]), gc.f64(x["v"]), scale, causal)
    err, n_over = check_o(gc.f64(o), o_ref)
    check_lse(gc.f64(lse), lse_ref)
    return err, n_over


def test_tiny():
    c = W.TINY
    for causal in c.causal:
        _full_check(c.B, c.H, c.Nq, c.Nk, c.d, causal, c.seed)


@pytest.mark.parametrize("causal", [True, False])
def test_b2_h8_n1024_d64(causal):
    c = W.C2
    _full_check(c.B, c.H, c.Nq, c.Nk, c.d, causal, c.seed)


RAGGED = [
    # B, H, Nq, Nk, d, causal
    (1, 1, 1, 1, 64, False),
    (1, 1, 1, 1, 128, True),
    (1, 2, 127, 127, 64, True),
    (1, 1, 129, 129, 128, True),
    (2, 1, 300, 300, 128, False),
    (1, 3, 1000, 1000, 64, True),
    (1, 1, 200, 500, 128, True),    # Nq < Nk: bottom-right causal alignment
    (1, 1, 500, 200, 64, True),     # Nq > Nk: the first 300 rows see no key
    (1, 1, 500, 200, 128, False),
    (1, 1, 77, 1, 64, True),
    (1, 2, 384, 640, 64, False),
    (3, 2, 256, 256, 128, True),
    (1, 1, 513, 1025, 128, True),
    # Enough 256-row units for the persistent two-tile grid (several units per CTA): Nq < Nk, Nq > Nk
    # (whole units whose rows see no key), and a last unit whose second tile lies past Nq.
    (2, 40, 700, 1300, 128, True),
    (2, 40, 1300, 700, 64, True),
    (1, 160, 300, 300, 128, False),
    (1, 160, 300, 300, 64, True),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", RAGGED)
def test_ragged_and_edge_shapes(B, H, Nq, Nk, d, causal):
    _full_check(B, H, Nq, Nk, d, causal, seed=11 + Nq + Nk + d)


def test_peaked_keys_small():
    """1% of key rows scaled by 8: large jumps of the running max (rescaling path)."""
    _full_check(1, 4, 2048, 2048, 128, True, seed=5, peaked=0.01)
    _full_check(1, 2, 1024, 1024, 64, False, seed=6, peaked=0.05)


def test_empty_keys_and_queries():
    dev = gc.DEV
    q = torch.randn(1, 2, 5, 64, device=dev).bfloat16()
    k = torch.empty(1, 2, 0, 64, device=dev, dtype=torch.bfloat16)
    o, lse = gc.fa.attention_forward(q, k, k, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    q0 = torch.empty(1, 2, 0, 64, device=dev, dtype=torch.bfloat16)
    o0, l0 = gc.fa.attention_forward(q0, q, q, causal=True)
    assert o0.numel() == 0 and l0.numel() == 0


def _sampled_check(cfg, causal, rows_per_head, seed):
    x = W.make_config_inputs(cfg, with_do=False)
    scale = cfg.scale
    o, lse = gc.gpu_forward(x["q"], x["k"], x["v"], causal, scale)
    o_h, lse_h = gc.f64(o), gc.f64(lse)
    q, k, v = x["q"], x["k"], x["v"]
    worst = 0.0
    for b in range(cfg.B):
        for h in range(cfg.H):
            must = []
            if x["peaks"].numel():
                must = x["peaks"][b, h][:8].tolist()   # queries at peaked positions
            rows = gc.sample_rows(cfg.Nq, rows_per_head, seed + 131 * b + h, must)
            o_ref, l_ref = A.attention_forward_rows(gc.f64(q[b, h]), gc.f64(k[b, h]), gc.f64(v[b, h]),
                                                    rows, scale, causal)
            err, _ = check_o(o_h[b, h, rows], o_ref, f"O[{b},{h}]")
            check_lse(lse_h[b, h, rows], l_ref, f"LSE[{b},{h}]")
            worst = max(worst, err)
    return worst


@pytest.mark.parametrize("cfg", W.SWEEP, ids=lambda c: c.name)
def test_sweep_full_size_sampled(cfg):
    _sampled_check(cfg, True, rows_per_head=64, seed=7)


def test_long_context_sampled():
    """512 sampled rows of every head (rows 0, 1 and N-1 and queries at peaked key positions among
    them); the whole of heads 0 and 15 is compared in tests/test_parity_bwd.py."""
    _sampled_check(W.LONG, True, rows_per_head=512, seed=9)
