"""The allocation-free decode entry point against the workspace entry point.

fa_decode_splitkv_noalloc serves callers that cannot allocate device memory
(for instance a plugin whose host framework owns all device memory through
its own pool, or a latency-critical loop where an allocation could
synchronise the device).  It keeps the split partials in the library's own
fixed device array instead of a caller workspace.  Here it is called through
the C ABI twice in a row, on different problems (so the second call starts
from the first call's leftovers in the shared array), and each result is
compared with fa_decode_splitkv on the same inputs within the decode
tolerances used elsewhere (|dO| <= 1e-2, |dLSE| <= 1e-3).

This file sorts last so that a run stopping at the first failure has already
run every other test; it passes alone in a fresh process too.
"""
import ctypes
import math

import pytest
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import build
from io_aware_exact_32_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20  # FA_DECODE_NOALLOC_SCRATCH_BYTES in include/fa.h


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _with_workspace(x, dev, splits):
    q, kc, vc = (x[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    seq = x["seqlens"].to(dev)
    d = q.shape[-1]
    return fa.decode_splitkv(q, kc, vc, seq, scale=1 / math.sqrt(d), num_splits=splits)


def _noalloc(L, x, dev, splits):
    q, kc, vc = (x[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    seq = x["seqlens"].to(dev)
    B, H, _, d = q.shape
    o = torch.full((B, H, 1, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device=dev)
    st = L.fa_decode_splitkv_noalloc(_ptr(q), _ptr(kc), _ptr(vc), _ptr(seq), kc.shape[2], _ptr(o), _ptr(lse),
                                     B, H, d, 1 / math.sqrt(d), splits,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fa.fa_status_string(st)
    return o, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    L = fa.lib()
    dev = torch.device("cuda:0")
    problems = [
        (W.make_decode_inputs(4, 8, 3000, 128, 1, seed=71), 0),
        (W.make_decode_inputs(3, 5, 1000, 64, 1, seed=72), 7),
    ]
    for x, splits in problems:
        B, H = x["q"].shape[:2]
        assert fa.fa_decode_workspace_size(B, H, x["k_cache"].shape[2], x["q"].shape[-1], splits) <= SCRATCH_BYTES
        o_ref, lse_ref = _with_workspace(x, dev, splits)
        o, lse = _noalloc(L, x, dev, splits)
        torch.cuda.synchronize()
        assert fa.fa_get_device_error() == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert (o.float() - o_ref.float()).abs().max().item() <= 1e-2
        assert (lse - lse_ref).abs().max().item() <= 1e-3


def test_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = fa.lib()
    dev = torch.device("cuda:0")
    B, H, Lmax, d = 64, 64, 8192, 128          # 64*64*8 splits of (128 + 2) floats > 8 MiB
    assert fa.fa_decode_workspace_size(B, H, Lmax, d, 0) > SCRATCH_BYTES
    t = torch.empty(16, dtype=torch.bfloat16, device=dev)
    seq = torch.ones(B, dtype=torch.int32, device=dev)
    st = L.fa_decode_splitkv_noalloc(_ptr(t), _ptr(t), _ptr(t), _ptr(seq), Lmax, _ptr(t), ctypes.c_void_p(0),
                                     B, H, d, 0.088, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 4   # FA_ERR_WORKSPACE, nothing launched
