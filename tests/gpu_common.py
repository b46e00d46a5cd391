"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, and turn the same seeded bf16 inputs into float64 for the oracle."""
import numpy as np
import torch

import io_aware_exact_32_b200 as fa
from io_aware_exact_32_b200 import build

build.build()
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(*ts):
    return [t.to(DEV).contiguous() if t is not None else None for t in ts]


def gpu_forward(q, k, v, causal, scale):
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.attention_forward(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return o, lse


def gpu_backward(q, k, v, o_dev, lse_dev, do, causal, scale):
    qd, kd, vd, dod = to_dev(q, k, v, do)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o_dev, lse_dev, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return dq, dk, dv


def sample_rows(n, count, seed, must=()):
    rng = np.random.default_rng(seed)
    base = set(int(m) for m in must if 0 <= m < n)
    base |= {0, min(1, n - 1), n - 1}
    extra = rng.choice(n, size=min(count, n), replace=False)
    return np.array(sorted(base | set(int(x) for x in extra)))
