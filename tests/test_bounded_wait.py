"""The give-up path of the kernels' bounded waits, exercised without any fault.

Every wait in the kernels gives up after a time limit (2 s by default): the CTA
records FA_ERR_TIMEOUT in the device status word, the other warps of the CTA
see its abort flag and stop, and the teardown still waits (with the fixed 2 s
limit) for the CTA's own copies and MMAs in flight before it frees its tensor
memory and exits.  Here the test hook fa_debug_set_wait_limit lowers the
limit to 300 ns, so the waits of a healthy causal forward, backward (both
head dims) or split-KV decode run out; each test checks that
fa_get_device_error reports the timeout, restores the limit, and checks that
the next call on the same device matches the float64 oracle (nothing was left
allocated or half-written that it could trip over).
"""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A
import gpu_common as gc
from tolerances import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = 6


def test_waits_give_up_and_the_device_stays_usable():
    B, H, N, d = 1, 16, 4096, 128
    x = W.make_attention_inputs(B, H, N, N, d, seed=91, with_do=False)
    q, k, v = gc.to_dev(x["q"], x["k"], x["v"])
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=gc.DEV)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    fa.fa_debug_set_wait_limit(300)
    try:
        fa.fa_fwd(q, k, v, o, lse, True, scale)
        torch.cuda.synchronize()
        status = fa.fa_get_device_error()
    finally:
        fa.fa_debug_set_wait_limit(0)
    assert status == FA_ERR_TIMEOUT, status

    o2, lse2 = fa.attention_forward(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    rows = gc.sample_rows(N, 48, 5)
    for h in (0, H - 1):
        ro, rl = A.attention_forward_rows(gc.f64(x["q"][0, h]), gc.f64(x["k"][0, h]), gc.f64(x["v"][0, h]),
                                          rows, scale, True)
        check_o(gc.f64(o2[0, h, rows]), ro, f"O[{h}]")
        check_lse(gc.f64(lse2[0, h, rows]), rl, f"LSE[{h}]")
    assert np.isfinite(gc.f64(o2)).all()


@pytest.mark.parametrize("d", [64, 128])
def test_backward_waits_give_up_and_the_device_stays_usable(d):
    # d = 64 and d = 128 take different dQ paths (own staging buffer / the block's dO tile).
    B, H, N = 1, 16, 4096
    x = W.make_attention_inputs(B, H, N, N, d, seed=92, with_do=True)
    q, k, v, do = gc.to_dev(x["q"], x["k"], x["v"], x["do"])
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    fa.fa_debug_set_wait_limit(300)
    try:
        fa.attention_backward(q, k, v, o, lse, do, causal=True, scale=scale)
        torch.cuda.synchronize()
        status = fa.fa_get_device_error()
    finally:
        fa.fa_debug_set_wait_limit(0)
    assert status == FA_ERR_TIMEOUT, status

    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    h = H - 1
    _, _, rdq, rdk, rdv = A.attention_backward_full_head(gc.f64(x["q"][0, h]), gc.f64(x["k"][0, h]),
                                                         gc.f64(x["v"][0, h]), gc.f64(x["do"][0, h]),
                                                         scale, True, block=512, workers=4)
    check_grad(gc.f64(dq[0, h]), rdq, "dQ")
    check_grad(gc.f64(dk[0, h]), rdk, "dK")
    check_grad(gc.f64(dv[0, h]), rdv, "dV")


def test_decode_waits_give_up_and_the_device_stays_usable():
    x = W.make_decode_inputs(8, 8, 4096, 128, 1024, seed=93)
    q, kc, vc = gc.to_dev(x["q"], x["k_cache"], x["v_cache"])
    seq = x["seqlens"].to(gc.DEV)
    scale = 1.0 / math.sqrt(128)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    fa.fa_debug_set_wait_limit(300)
    try:
        fa.decode_splitkv(q, kc, vc, seq, scale=scale)
        torch.cuda.synchronize()
        status = fa.fa_get_device_error()
    finally:
        fa.fa_debug_set_wait_limit(0)
    assert status == FA_ERR_TIMEOUT, status

    o, lse = fa.decode_splitkv(q, kc, vc, seq, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    o_ref, l_ref = A.decode_forward(gc.f64(x["q"]), gc.f64(x["k_cache"]), gc.f64(x["v_cache"]),
                                    x["seqlens"].numpy(), scale)
    check_o(gc.f64(o)[:, :, 0], o_ref)
    check_lse(gc.f64(lse), l_ref)
