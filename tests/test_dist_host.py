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


def test_attn_point_host_logic():
    """bench.py's per-workload block with a stand-in for the library (no GPU call): it allocates the
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
    out = bench.attn_point(fake, W, torch.device("cpu"), None, {"bf16_tflops": 1000.0},
                           lambda fn: (fn(), 1e-3)[1], small)
    assert calls == ["fwd", "bwd"]
    ff = W.flops_forward(1, 2, 256, 256, 128, True)
    assert abs(out["fwd_tflops"] - ff / 1e-3 / 1e12) < 1e-12
    assert abs(out["fwd_bwd_tflops"] - 3.5 * ff / 2e-3 / 1e12) < 1e-12
    assert out["device_status"] == 0 and out["N"] == 256


def test_visible_pairs_and_cpu_sample_flops():
    """The CPU baseline counts FLOPs over the visible (query, key) pairs of its row blocks: summed over
    all blocks that is N (N + 1) / 2 pairs under the causal mask (the convention's N^2 / 2, up to N / 2)."""
    import bench
    from io_aware_exact_32_b200 import workloads as W
    n = 1024
    assert sum(bench.visible_keys(r, r + 256, n, n, True) for r in range(0, n, 256)) == n * (n + 1) // 2
    assert bench.visible_keys(0, 4, 10, 10, False) == 40
    assert bench.visible_keys(0, 3, 5, 3, True) == 0 + 0 + 1      # bottom-right: rows 0, 1 see nothing
    cfg = W.AttnConfig("t", 1, 1, 512, 512, 64, (True,), seed=0)
    x = W.make_config_inputs(cfg)
    flops, el, nblk, _ = bench.cpu_oracle_blocks(0.0, cfg, x, steps=2)
    assert nblk == 2 and el > 0
    want = sum(3.5 * 4 * 64 * bench.visible_keys(r0, r0 + 256, 512, 512, True)
               for r0 in ((0 * 7919) % 2 * 256, (1 * 7919) % 2 * 256))
    assert flops == want


def test_clock_summary():
    import bench
    rows = ["0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1800, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 300, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    s = bench.summarize_clocks(rows)
    assert s["sm_mhz"] == (1965 + 1800) / 2 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3
    assert bench.summarize_clocks([])["reasons"] == ["unsampled"]
