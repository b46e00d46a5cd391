"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2).

The path shards (batch, head) units across ranks with no collective on the
data path; the only exchange is the max over ranks of the timed duration.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = bench.dist_env()
        my_time = 1.5 + r                      # rank 1 is the slow one
        t = bench.reduce_max(my_time, w)
        seed = bench.shard_seed(7, r)
        from io_aware_exact_32_b200 import workloads as W
        x = W.make_attention_inputs(1, 2, 8, 8, 64, seed, with_do=False)
        q.put((r, t, seed, float(x["q"].float().sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_shards_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]          # every rank sees the max over ranks
    assert res[0][2] != res[1][2]                     # distinct shards
    assert res[0][3] != res[1][3]
    assert bench.whole_job_rate(10.0, world, 2.5) == 8.0


def test_single_process_defaults(monkeypatch):
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.reduce_max(3.0, 1) == 3.0


def test_measured_peaks_read():
    p = bench.measured_peaks()
    assert p["bf16_tflops"] > 100 and p["hbm_gbs"] > 1000


def test_long_context_measurement_host_logic():
    """bench.py's long-context block with a stand-in for the library (no GPU call): it allocates the
    right shapes and turns times into the FLOP-rate fields."""
    import types

    import torch

    import bench
    from io_aware_exact_32_b200 import workloads as W

    calls = []
    fake = types.SimpleNamespace(
        attention_forward=lambda q, k, v, causal, scale: (torch.empty_like(q), torch.empty(q.shape[:3])),
        fa_bwd_workspace_size=lambda B, H, N, d: 256,
        fa_fwd=lambda *a: calls.append("fwd"),
        fa_bwd=lambda *a: calls.append("bwd"),
        fa_get_device_error=lambda stream: 0)
    small = W.AttnConfig("long_small", 1, 2, 256, 256, 128, (True,), seed=3, peaked_frac=0.01)
    out = bench.long_context_measurement(fake, W, torch.device("cpu"), None, {"bf16_tflops": 1000.0},
                                         lambda fn: (fn(), 1e-3)[1], cfg=small)
    assert calls == ["fwd", "bwd"]
    ff = W.flops_forward(1, 2, 256, 256, 128, True)
    assert abs(out["fwd_tflops"] - ff / 1e-3 / 1e12) < 1e-12
    assert abs(out["fwd_bwd_tflops"] - 3.5 * ff / 2e-3 / 1e12) < 1e-12
    assert out["device_status"] == 0 and out["N"] == 256
