"""Split-KV decode parity against the float64 oracle (no splitting, plain definition)."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
import gpu_common as gc
from tolerances import check_lse, check_o, rel_l2

pytestmark = pytest.mark.gpu


def _run(x, num_splits=0, poison=False):
    q, kc, vc = gc.to_dev(x["q"], x["k_cache"], x["v_cache"])
    seq = x["seqlens"].to(gc.DEV)
    if poison:
        # Slots at or beyond L_b must never be read: fill them with NaN.
        for b, L in enumerate(x["seqlens"].tolist()):
            kc[b, :, L:] = float("nan")
            vc[b, :, L:] = float("nan")
    o, lse = fa.decode_splitkv(q, kc, vc, seq, scale=1 / math.sqrt(q.shape[-1]), num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return gc.f64(o)[:, :, 0], gc.f64(lse)


def _oracle(x):
    d = x["q"].shape[-1]
    return A.decode_forward(gc.f64(x["q"]), gc.f64(x["k_cache"]), gc.f64(x["v_cache"]),
                            x["seqlens"].numpy(), 1 / math.sqrt(d))


def test_decode_config_full():
    c = W.DECODE
    x = W.make_decode_inputs(c.B, c.H, c.Lmax, c.d, c.lmin, c.seed)
    o_ref, l_ref = _oracle(x)
    o, lse = _run(x, poison=True)
    check_o(o, o_ref)
    check_lse(lse, l_ref)


@pytest.mark.parametrize("splits", [1, 3, 8, 64, 256])
def test_split_count_invariance(splits):
    x = W.make_decode_inputs(4, 8, 4096, 128, 1, seed=21)
    o_ref, l_ref = _oracle(x)
    o, lse = _run(x, num_splits=splits, poison=True)
    check_o(o, o_ref)
    check_lse(lse, l_ref)
    o0, _ = _run(x, num_splits=0)
    assert rel_l2(o, o0) < 1e-2


@pytest.mark.parametrize("B,H,Lmax,d,lmin", [(3, 2, 1, 64, 1), (5, 3, 37, 128, 1), (2, 4, 1000, 64, 500),
                                             (7, 1, 3000, 128, 1), (1, 2, 65536, 128, 60000)])
def test_decode_shapes(B, H, Lmax, d, lmin):
    x = W.make_decode_inputs(B, H, Lmax, d, lmin, seed=B + H + Lmax)
    o_ref, l_ref = _oracle(x)
    o, lse = _run(x, poison=True)
    check_o(o, o_ref)
    check_lse(lse, l_ref)


def test_decode_matches_forward_with_one_query():
    """One split over the full cache equals the prefill path with Nq = 1."""
    x = W.make_decode_inputs(2, 4, 640, 128, 640, seed=3)
    o, _ = _run(x, num_splits=1)
    qd, kd, vd = gc.to_dev(x["q"], x["k_cache"], x["v_cache"])
    of, _ = fa.attention_forward(qd, kd, vd, causal=False, scale=1 / math.sqrt(128))
    assert np.max(np.abs(o - gc.f64(of)[:, :, 0])) < 1e-2
