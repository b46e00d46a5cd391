#!/usr/bin/env python
"""Benchmark of the exact fused attention path on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (per GPU): the long-context case B=1, H=16, Nq=Nk=65536,
d=128, causal, bf16 Q, K, V, dO iid N(0,1) with 1% of key rows x8 (peaked
softmax).  One step = fa_fwd + fa_bwd through the C ABI (every row of the hot
path: tiled forward with the online softmax, D preprocessing, the key-block
backward with its dQ reduce-adds, dQ conversion).  `value` is whole-job
TFLOP/s by the convention 4*B*H*Nq*Nk*d per forward, halved when causal, and
2.5x that per backward.  Every operand (268 MB each) is larger than the
126 MB L2, so no flush is needed between steps.

Alongside: `e2e` (the same step through the public binding from pinned host
buffers, host<->device copies inside the timed region), the roofline of the
dominant kernel (fa_bwd_main_kernel<128>), a CPU-oracle baseline, and `extra`:
the 12 points of the sequence sweep (N 512..16384 x d 64/128, causal, forward
and forward+backward), the B=2 H=8 N=1024 d=64 step, the FP8 and bias /
dropout variants, the deterministic backward and split-KV decode (HBM GB/s).

With N > 1 (torchrun, one process per GPU) every rank runs its own shard of
(batch, head) units (weak scaling, no collective on the data path); times are
the max over ranks.  `--impl reference` times the float64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20
METRIC = "attention fwd+bwd TFLOP/s (causal, d=128, N=65536)"


# --------------------------------------------------------------------------------- host logic
def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process when absent)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own shard of (batch, head) units: distinct inputs, no exchange."""
    return base_seed + 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one process)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(per_rank_units: float, world: int, max_seconds: float) -> float:
    return per_rank_units * world / max_seconds


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def captured_traffic(key):
    """DRAM bytes per launch of a kernel, from the committed record of its ncu capture
    (profiles/traffic.json), or (None, None) once the kernel's sources differ from the captured ones."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[key]
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["sources_sha256"]:
            return None, None
        return int(rec["dram_bytes_per_launch"]), rec["capture"]
    except Exception:
        return None, None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None, period_ms: int = 100):
        self.gpu = str(gpu_index)
        self.proc = None
        self.period_ms = period_ms
        # The raw samples are kept where --clock-log asks (else a temporary file); the summary
        # goes into the JSON line either way.
        self.path = path or os.path.join(tempfile.gettempdir(), f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", str(self.period_ms), "-i", self.gpu], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)  # let the sampler start before the timed region
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        return summarize_clocks(open(self.path).read().splitlines())


def summarize_clocks(lines):
    """Median SM clock under load, the max clock and the throttle reasons seen, from nvidia-smi CSV rows."""
    sm, smax, reasons = [], [], set()
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
    busy = [s for s in sm if s > 0.5 * max(sm)] or sm
    return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
            "samples": len(sm)}


def visible_keys(r0: int, r1: int, nq: int, nk: int, causal: bool) -> int:
    """Number of (query, key) pairs of query rows [r0, r1) that the mask leaves visible."""
    if not causal:
        return (r1 - r0) * nk
    tot = 0
    for i in range(r0, r1):
        tot += max(0, min(nk, i + (nk - nq) + 1))
    return tot


# --------------------------------------------------------------------------------- CPU oracle
def cpu_oracle_blocks(seconds: float, cfg, x, steps: int | None = None, block: int = 256):
    """Time the float64 oracle on 256-row blocks of head 0 of ``cfg`` (forward + backward of those rows,
    each row with its whole visible score row); FLOPs counted by the forward / backward convention
    over the visible pairs, 4 d per pair forward and 2.5 x that backward.

    Runs until ``seconds`` have passed (or for ``steps`` blocks).  Returns (flops, elapsed, blocks, threads)."""
    import numpy as np
    from oracle import attention as A
    q, k, v, do = (x[n][0, 0].double().numpy() for n in ("q", "k", "v", "do"))
    nblk = cfg.Nq // block
    causal = True in cfg.causal
    flops, t0, n = 0.0, time.perf_counter(), 0
    while True:
        r0 = ((n * 7919) % nblk) * block
        A.attention_row_block(q, k, v, do, r0, r0 + block, cfg.scale, causal)
        flops += 3.5 * 4.0 * cfg.d * visible_keys(r0, r0 + block, cfg.Nq, cfg.Nk, causal)
        n += 1
        el = time.perf_counter() - t0
        if (steps is not None and n >= steps) or (steps is None and el >= seconds):
            break
    return flops, el, n, blas_threads()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def workload_config(cfg, world: int) -> dict:
    return {"workload": f"{cfg.name} causal fwd+bwd (B={cfg.B} H={cfg.H} N={cfg.Nq} d={cfg.d}, 1% of key rows x8)",
            "global_batch": cfg.B * world, "seq_len": cfg.Nq, "heads": cfg.H, "head_dim": cfg.d,
            "parallelism": f"dp{world} over (batch, head)" if world > 1 else "single GPU",
            "l2": "no flush: every operand (268 MB) is larger than the 126 MB L2"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from io_aware_exact_32_b200 import workloads as W
    c = W.LONG
    x = W.make_config_inputs(c)
    cpu_oracle_blocks(0.0, c, x, steps=args.warmup)
    flops, secs, n, threads = cpu_oracle_blocks(0.0, c, x, steps=args.steps)
    value = flops / secs / 1e12
    sample = (f"{args.steps} steps, each a 256-row block of head 0 of B={c.B} H={c.H} N={c.Nq} d={c.d} causal: "
              f"forward + backward of those rows in float64 numpy (every row with its whole visible score row)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(c, 1), parallelism="none (host cores)"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------- GPU path
def run_ours(args):
    import torch
    import torch.distributed as dist

    import io_aware_exact_32_b200 as fa
    from io_aware_exact_32_b200 import build, workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    fa.lib()
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()

    c = W.LONG
    x = W.make_attention_inputs(c.B, c.H, c.Nq, c.Nk, c.d, shard_seed(c.seed, rank), c.peaked_frac, c.peak_factor)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, N, d = c.B, c.H, c.Nq, c.d
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    f_fwd = W.flops_forward(B, H, N, N, d, True)
    f_bwd = W.flops_backward(B, H, N, N, d, True)
    step_flops = f_fwd + f_bwd
    launches_per_step = 1 + 3  # fa_fwd: 1 kernel; fa_bwd: preprocess + main + dQ convert

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.fa_fwd(q, k, v, o, lse, True, c.scale, stream)
        if ev is not None:
            ev[1].record(stream)
        fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, True, c.scale, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(dev.index if world == 1 else local, args.clock_log).start() if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(K):
        step(ev[s])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    status = fa.fa_get_device_error()
    fwd_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    bwd_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K)]
    step_total_s = sum(ev[s][0].elapsed_time(ev[s][2]) for s in range(K)) / 1e3
    total_s = reduce_max(step_total_s, world, dev)
    value = whole_job_rate(step_flops * K, world, total_s) / 1e12

    # ---------------------------------------------------------------- end to end from host buffers
    # Every step copies its inputs (q, k, v, dO) from pinned host memory and reads all its outputs
    # (o, lse, dq, dk, dv) back; the copies of one step overlap the compute of its neighbours (upload
    # stream -> compute stream -> read-back stream, device buffers double-buffered).
    # e2e.serial_value: the same step with copies and compute in sequence.
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
    names_out = ("o", "lse", "dq", "dk", "dv")
    shapes_out = {"o": (q.shape, torch.bfloat16), "lse": (lse.shape, torch.float32), "dq": (q.shape, torch.bfloat16),
                  "dk": (k.shape, torch.bfloat16), "dv": (v.shape, torch.bfloat16)}
    dev_in = [tuple(torch.empty_like(t) for t in (q, k, v, do)) for _ in range(2)]
    dev_out = [{n: torch.empty(s, dtype=dt, device=dev) for n, (s, dt) in shapes_out.items()} for _ in range(2)]
    host_out = [{n: torch.empty(s, dtype=dt, pin_memory=True) for n, (s, dt) in shapes_out.items()} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    wse = torch.empty_like(ws)

    def compute(buf, dst):
        q_, k_, v_, do_ = buf
        fa.fa_fwd(q_, k_, v_, dst["o"], dst["lse"], True, c.scale, stream)
        fa.fa_bwd(q_, k_, v_, dst["o"], do_, dst["lse"], dst["dq"], dst["dk"], dst["dv"], wse, True, c.scale, stream)

    def e2e_serial_step():
        buf, dst, hst = dev_in[0], dev_out[0], host_out[0]
        for d_, h_ in zip(buf, (hq, hk, hv, hdo)):
            d_.copy_(h_, non_blocking=True)
        compute(buf, dst)
        for n in names_out:
            hst[n].copy_(dst[n], non_blocking=True)

    def e2e_pipelined(n_steps):
        mk = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, computed, read_back = [], [], []
        for st in range(n_steps):
            slot = st % 2
            with torch.cuda.stream(up):
                if st >= 2:
                    up.wait_event(computed[st - 2])  # that step is done with this input buffer
                for d_, h_ in zip(dev_in[slot], (hq, hk, hv, hdo)):
                    d_.copy_(h_, non_blocking=True)
                in_ready.append(mk())
                in_ready[-1].record(up)
            stream.wait_event(in_ready[st])
            if st >= 2:
                stream.wait_event(read_back[st - 2])  # that step's outputs are on the host
            compute(dev_in[slot], dev_out[slot])
            computed.append(mk())
            computed[-1].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[st])
                for n in names_out:
                    host_out[slot][n].copy_(dev_out[slot][n], non_blocking=True)
                read_back.append(mk())
                read_back[-1].record(down)
        return read_back[-1]

    e2e_serial_step()
    e2e_pipelined(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(up)
    last = e2e_pipelined(K)
    down.wait_event(last)
    t1.record(down)
    torch.cuda.synchronize()
    e2e_s = reduce_max(t0.elapsed_time(t1) / 1e3, world, dev)
    e2e_value = whole_job_rate(step_flops * K, world, e2e_s) / 1e12
    n_ser = min(K, 5)
    ser_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ser)]
    if world > 1:
        dist.barrier()
    for a_, b_ in ser_ev:
        a_.record(stream)
        e2e_serial_step()
        b_.record(stream)
    torch.cuda.synchronize()
    ser_s = reduce_max(sum(a_.elapsed_time(b_) for a_, b_ in ser_ev) / 1e3, world, dev)
    e2e_serial_value = whole_job_rate(step_flops * n_ser, world, ser_s) / 1e12
    e2e_status = fa.fa_get_device_error()
    del dev_in, dev_out, host_out, hq, hk, hv, hdo, wse

    # ---------------------------------------------------------------- dominant kernel roofline
    # fa_bwd_main_kernel<128> carries about three quarters of the step (ncu launch list); it is timed
    # per fa_bwd call in the timed region above.  The call also holds the D preprocessing and the dQ
    # conversion (together ~0.5% of it), so the achieved rate understates the main kernel slightly.
    bwd_mean_s = statistics.mean(bwd_ms) / 1e3
    dom_tflops = f_bwd / bwd_mean_s / 1e12
    roofline = {"bound": "tensor", "kernel": "fa_bwd_main_kernel<128>, timed per fa_bwd call (with its D "
                                             "preprocessing and dQ-conversion kernels)",
                "achieved": dom_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": dom_tflops / peaks["bf16_tflops"], "traffic": None,
                "peak_source": (f"measured bf16 burst (MEASURED_PEAKS.json); of the sustained "
                                f"{peaks['bf16_tflops_sustained']:.0f}: "
                                f"{dom_tflops / peaks['bf16_tflops_sustained']:.3f}")
                if peaks["source"] == "measured" else "fallback 1590 TFLOP/s",
                "algorithmic_flops_per_launch": f_bwd}
    roofline["traffic"], roofline["traffic_source"] = captured_traffic("fa_bwd_main_kernel<128> long_n65536_d128")
    if roofline["traffic"] is not None:
        roofline["traffic_unit"] = "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)"
    fwd_mean_s = statistics.mean(fwd_ms) / 1e3
    del q, k, v, do, o, lse, dq, dk, dv, ws

    extra = {}
    if not args.no_extra and world == 1:  # single-GPU kernel measurements; the N > 1 line is the headline alone
        extra = extra_measurements(fa, W, dev, stream, peaks)

    if world > 1:
        dist.barrier()
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu:
            f, el, nblk, threads = cpu_oracle_blocks(args.cpu_seconds, c, x)
            cpu = {"value": f / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                   "sample": f"{nblk} blocks of 256 query rows of head 0 of the headline workload, forward + "
                             f"backward of those rows in float64 numpy ({el:.1f} s)"}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (iid N(0,1) bf16, 1% of key rows x8, seeded per rank)",
            "config": dict(workload_config(c, world), launch="eager, one fa_fwd + one fa_bwd per step"),
            "frac_of_peak": value / world / peaks["bf16_tflops"],
            "fwd_tflops": f_fwd / fwd_mean_s / 1e12, "bwd_tflops": f_bwd / bwd_mean_s / 1e12,
            "fwd_ms": 1e3 * fwd_mean_s, "bwd_ms": 1e3 * bwd_mean_s,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "overlapped with the neighbouring steps' compute (upload, compute and read-back streams)",
                    "serial_value": e2e_serial_value, "device_status": e2e_status},
            "gpu_launches": launches_per_step * K,
            "clocks": clk,
            "device_status": status,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def attn_point(fa, W, dev, stream, peaks, timed, cfg, causal=True):
    """Forward and forward+backward of one attention workload; ``timed(fn)`` returns seconds per call."""
    import torch
    x = W.make_config_inputs(cfg)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    del x
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=cfg.scale)
    ws = torch.empty(max(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), 256), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    t_f = timed(lambda: fa.fa_fwd(q, k, v, o, lse, causal, cfg.scale, stream))
    t_b = timed(lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, causal, cfg.scale, stream))
    ff = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal)
    fb = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal)
    f1, f2 = ff / t_f / 1e12, (ff + fb) / (t_f + t_b) / 1e12
    return {"B": cfg.B, "H": cfg.H, "N": cfg.Nq, "d": cfg.d, "fwd_tflops": f1, "fwd_frac": f1 / peaks["bf16_tflops"],
            "bwd_tflops": fb / t_b / 1e12, "fwd_bwd_tflops": f2, "fwd_bwd_frac": f2 / peaks["bf16_tflops"],
            "fwd_frac_of_2250": f1 / 2250.0, "fwd_bwd_frac_of_2250": f2 / 2250.0,
            "fwd_ms": 1e3 * t_f, "bwd_ms": 1e3 * t_b, "device_status": fa.fa_get_device_error(stream)}


def extra_measurements(fa, W, dev, stream, peaks, iters=10):
    """The sequence sweep (12 points), the B=2 H=8 N=1024 d=64 step, FP8 and bias / dropout at causal
    d=128, the deterministic backward and split-KV decode bandwidth."""
    import torch
    res = {"peak_note": "fractions are of the measured bf16 burst peak (MEASURED_PEAKS.json); *_of_2250 of the "
                        "datasheet dense bf16 figure (HGX B200: 36 PFLOPS per 8 GPUs with 2:4 sparsity)"}
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(iters):
            flush_buf.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ts) / 1e3

    sweep = {}
    for cfg in W.SWEEP:
        try:
            sweep[f"n{cfg.Nq}_d{cfg.d}"] = attn_point(fa, W, dev, stream, peaks, timed, cfg)
        except Exception as e:  # noqa: BLE001 - reported in the JSON line
            sweep[f"n{cfg.Nq}_d{cfg.d}"] = {"error": f"{type(e).__name__}: {e}"}
    res["sweep_causal_16384_tokens_h16"] = sweep
    res["b2_h8_n1024_d64_step"] = small_step(fa, W, dev, stream, peaks, flush_buf)

    for n in (4096, 8192, 16384):
        cfg = next(c for c in W.SWEEP if c.Nq == n and c.d == 128)
        x = W.make_config_inputs(cfg)
        q, k, v, do = (x[nm].to(dev) for nm in ("q", "k", "v", "do"))
        o, lse = fa.attention_forward(q, k, v, causal=True, scale=cfg.scale)
        ff = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, True)
        fb = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, True)
        t_f = sweep[f"n{n}_d128"]["fwd_ms"] / 1e3
        t_b = sweep[f"n{n}_d128"]["bwd_ms"] / 1e3
        # FP8 forward on the same inputs: Q and K rotated (random-sign Hadamard) and quantised, V quantised.
        signs = W.make_hadamard_signs(cfg.d, 11).to(dev)
        q8, dsq = fa.quantize_fp8(q, signs, True, stream)
        k8, dsk = fa.quantize_fp8(k, signs, True, stream)
        v8, dsv = fa.quantize_fp8(v, None, False, stream)
        o8 = torch.empty_like(o)
        lse8 = torch.empty_like(lse)
        t_f8 = timed(lambda: fa.fa_fwd_fp8(q8, k8, v8, dsq, dsk, dsv, o8, lse8, True, cfg.scale, stream))

        def quantize_all():
            fa.fa_quantize_fp8(q, signs, q8, dsq, True, stream)
            fa.fa_quantize_fp8(k, signs, k8, dsk, True, stream)
            fa.fa_quantize_fp8(v, None, v8, dsv, False, stream)

        t_q8 = timed(quantize_all)
        f8_t = ff / t_f8 / 1e12
        qbytes = 3 * q.numel() * 3  # algorithmic: read bf16 (2 B) and write E4M3 (1 B) for Q, K, V
        res[f"fp8_causal_n{n}_d128"] = {
            "fwd_tflops": f8_t, "fwd_ms": 1e3 * t_f8, "vs_bf16_fwd": t_f / t_f8,
            "fwd_frac_of_fp8_peak": f8_t / (2.0 * peaks["bf16_tflops"]), "fwd_frac_of_4500": f8_t / 4500.0,
            "fp8_peak_note": "2 x measured bf16 (the nominal fp8 / bf16 ratio)",
            "quantize_qkv_ms": 1e3 * t_q8, "quantize_gbs_algorithmic": qbytes / t_q8 / 1e9,
            "quantize_frac_of_hbm": qbytes / t_q8 / 1e9 / peaks["hbm_gbs"],
            "fwd_incl_quantize_tflops": ff / (t_f8 + t_q8) / 1e12}
        del q8, k8, v8, dsq, dsk, dsv, o8, lse8
        if n == 4096:
            ws = torch.empty(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), dtype=torch.uint8, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            # Bias (one [Nq, Nk] plane per head, broadcast over the batch) and dropout p = 0.1.
            gb = torch.Generator().manual_seed(9)
            bias = (torch.randn(1, cfg.H, cfg.Nq, cfg.Nk, generator=gb) * 0.5).to(torch.bfloat16).to(dev)
            oe, lsee = torch.empty_like(o), torch.empty_like(lse)
            t_fe = timed(lambda: fa.fa_fwd_ext(q, k, v, oe, lsee, bias, True, cfg.scale, 0.1, 1234, 0, stream))
            t_be = timed(lambda: fa.fa_bwd_ext(q, k, v, oe, do, lsee, dq, dk, dv, ws, bias, True, cfg.scale, 0.1, 1234,
                                               0, stream))
            res["bias_dropout_causal_n4096_d128"] = {
                "fwd_tflops": ff / t_fe / 1e12, "bwd_tflops": fb / t_be / 1e12,
                "fwd_bwd_tflops": (ff + fb) / (t_fe + t_be) / 1e12, "fwd_ms": 1e3 * t_fe, "bwd_ms": 1e3 * t_be,
                "vs_plain_fwd": t_f / t_fe, "vs_plain_bwd": t_b / t_be,
                "note": "bias [1, H, N, N] bf16, dropout p = 0.1"}
            # Each extension alone: the bias without dropout, and dropout 0.1 without a bias.
            for name, bias_, p_ in (("bias_only", bias, 0.0), ("dropout_only", None, 0.1)):
                t_f1 = timed(lambda: fa.fa_fwd_ext(q, k, v, oe, lsee, bias_, True, cfg.scale, p_, 1234, 0, stream))
                t_b1 = timed(lambda: fa.fa_bwd_ext(q, k, v, oe, do, lsee, dq, dk, dv, ws, bias_, True, cfg.scale, p_,
                                                   1234, 0, stream))
                res[f"{name}_causal_n4096_d128"] = {
                    "fwd_tflops": ff / t_f1 / 1e12, "bwd_tflops": fb / t_b1 / 1e12, "fwd_ms": 1e3 * t_f1,
                    "bwd_ms": 1e3 * t_b1, "vs_plain_fwd": t_f / t_f1, "vs_plain_bwd": t_b / t_b1}
            del bias, oe, lsee
            t_bd = timed(lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, True, cfg.scale, stream,
                                           deterministic=True))
            res["deterministic_bwd_causal_n4096_d128"] = {"bwd_tflops": fb / t_bd / 1e12, "bwd_ms": 1e3 * t_bd,
                                                          "vs_default_bwd": t_b / t_bd}
            del ws, dq, dk, dv
        del q, k, v, do, o, lse, x
    dc = W.DECODE
    xd = W.make_decode_inputs(dc.B, dc.H, dc.Lmax, dc.d, dc.lmin, dc.seed)
    qd, kc, vc = (xd[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    seq = xd["seqlens"].to(dev)
    od = torch.empty_like(qd)
    lsed = torch.empty(dc.B, dc.H, device=dev, dtype=torch.float32)
    wsd = torch.empty(fa.fa_decode_workspace_size(dc.B, dc.H, dc.Lmax, dc.d, 0), dtype=torch.uint8, device=dev)
    t_d = timed(lambda: fa.fa_decode_splitkv(qd, kc, vc, seq, od, lsed, wsd, dc.scale, 0, stream))
    nbytes = W.decode_bytes(xd["seqlens"], dc.H, dc.d)
    res["decode_b32_h32_l8192_d128"] = {"gbs": nbytes / t_d / 1e9, "frac_of_measured_hbm": nbytes / t_d / 1e9 /
                                        peaks["hbm_gbs"], "frac_of_8000": nbytes / t_d / 1e9 / 8000.0,
                                        "ms": 1e3 * t_d, "algorithmic_bytes": nbytes,
                                        "device_status": fa.fa_get_device_error(stream)}
    return res


def small_step(fa, W, dev, stream, peaks, flush_buf, reps=200):
    """The B=2 H=8 N=1024 d=64 step (forward + backward causal, then non-causal), captured once as a
    CUDA graph and replayed, with a 256 MiB L2 flush before each replay."""
    import torch
    c = W.C2
    x = W.make_attention_inputs(c.B, c.H, c.Nq, c.Nk, c.d, c.seed)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, N, d = c.B, c.H, c.Nq, c.d
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    out = {cz: dict(o=torch.empty_like(q), lse=torch.empty(B, H, N, device=dev, dtype=torch.float32),
                    dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v)) for cz in (True, False)}
    flops = sum(W.flops_forward(B, H, N, N, d, cz) + W.flops_backward(B, H, N, N, d, cz) for cz in (True, False))

    def step(st):
        for cz in (True, False):
            t = out[cz]
            fa.fa_fwd(q, k, v, t["o"], t["lse"], cz, c.scale, st)
            fa.fa_bwd(q, k, v, t["o"], do, t["lse"], t["dq"], t["dk"], t["dv"], ws, cz, c.scale, st)

    for _ in range(3):
        step(stream)
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        step(cap)
    stream.wait_stream(cap)
    evs = []
    for i in range(reps + 5):
        flush_buf.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        if i >= 5:
            evs.append((a, b))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    del graph
    return {"tflops": flops / (ms / 1e3) / 1e12, "frac": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "ms_per_step": ms, "launch": "CUDA graph of one step (8 launches), replayed; L2 flushed before each",
            "device_status": fa.fa_get_device_error(stream)}


CASES = ("fwd_c2", "bwd_c2", "fwd_n4096_d128", "bwd_n4096_d128", "fwd_fp8_n4096_d128", "fwd_ext_n4096_d128",
         "bwd_ext_n4096_d128", "fwd_bias_n4096_d128", "bwd_bias_n4096_d128", "fwd_drop_n4096_d128",
         "bwd_drop_n4096_d128", "decode", "fwd_long", "bwd_long", "bwd_n16384_d128", "fwd_n16384_d128",
         "bwd_n4096_d64", "fwd_n4096_d64", "bwd_det_n4096_d128", "quant_n4096_d128")


def run_case(args):
    """One C-ABI call on one workload, repeated; used for single-kernel profiling."""
    import torch

    import io_aware_exact_32_b200 as fa
    from io_aware_exact_32_b200 import build, workloads as W

    build.build()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream()
    name = args.case
    if name == "decode":
        dc = W.DECODE
        xd = W.make_decode_inputs(dc.B, dc.H, dc.Lmax, dc.d, dc.lmin, dc.seed)
        qd, kc, vc = (xd[n].to(dev) for n in ("q", "k_cache", "v_cache"))
        seq = xd["seqlens"].to(dev)
        od = torch.empty_like(qd)
        lsed = torch.empty(dc.B, dc.H, device=dev, dtype=torch.float32)
        wsd = torch.empty(fa.fa_decode_workspace_size(dc.B, dc.H, dc.Lmax, dc.d, 0), dtype=torch.uint8, device=dev)
        fn = lambda: fa.fa_decode_splitkv(qd, kc, vc, seq, od, lsed, wsd, dc.scale, 0, stream)
        units, unit = W.decode_bytes(xd["seqlens"], dc.H, dc.d) / 1e9, "GB/s"
    else:
        if name.endswith("c2"):
            cfg = W.C2
        elif name.endswith("long"):
            cfg = W.LONG
        else:
            n, d = (int(t[1:]) for t in name.split("_")[-2:])
            cfg = next(c for c in W.SWEEP if c.Nq == n and c.d == d)
        causal = True
        x = W.make_config_inputs(cfg)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
        del x
        o, lse = fa.attention_forward(q, k, v, causal=causal, scale=cfg.scale)
        ff = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal)
        fb = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal)
        if name.startswith("bwd"):
            ws = torch.empty(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), dtype=torch.uint8, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        if name.startswith("quant"):
            # Q and K rotated (random-sign Hadamard) and quantised, V quantised; algorithmic bytes: read
            # bf16 and write E4M3 once (3 bytes an element).
            signs = W.make_hadamard_signs(cfg.d, 11).to(dev)
            q8, dsq = fa.quantize_fp8(q, signs, True, stream)
            k8, dsk = fa.quantize_fp8(k, signs, True, stream)
            v8, dsv = fa.quantize_fp8(v, None, False, stream)

            def fn():
                fa.fa_quantize_fp8(q, signs, q8, dsq, True, stream)
                fa.fa_quantize_fp8(k, signs, k8, dsk, True, stream)
                fa.fa_quantize_fp8(v, None, v8, dsv, False, stream)

            units, unit = 3 * q.numel() * 3 / 1e9, "GB/s"
        elif name.startswith("fwd_fp8"):
            signs = W.make_hadamard_signs(cfg.d, 11).to(dev)
            q8, dsq = fa.quantize_fp8(q, signs, True, stream)
            k8, dsk = fa.quantize_fp8(k, signs, True, stream)
            v8, dsv = fa.quantize_fp8(v, None, False, stream)
            fn = lambda: fa.fa_fwd_fp8(q8, k8, v8, dsq, dsk, dsv, o, lse, causal, cfg.scale, stream)
            units = ff / 1e12
        elif "_ext_" in name or "_bias_" in name or "_drop_" in name:
            # bias [1, H, N, N] and / or dropout p = 0.1 (ext: both)
            bias = None
            if "_drop_" not in name:
                gb = torch.Generator().manual_seed(9)
                bias = (torch.randn(1, cfg.H, cfg.Nq, cfg.Nk, generator=gb) * 0.5).to(torch.bfloat16).to(dev)
            pd = 0.0 if "_bias_" in name else 0.1
            fa.fa_fwd_ext(q, k, v, o, lse, bias, causal, cfg.scale, pd, 1234, 0, stream)
            if name.startswith("fwd"):
                fn = lambda: fa.fa_fwd_ext(q, k, v, o, lse, bias, causal, cfg.scale, pd, 1234, 0, stream)
                units = ff / 1e12
            else:
                fn = lambda: fa.fa_bwd_ext(q, k, v, o, do, lse, dq, dk, dv, ws, bias, causal, cfg.scale, pd, 1234, 0,
                                           stream)
                units = fb / 1e12
        elif name.startswith("fwd"):
            fn = lambda: fa.fa_fwd(q, k, v, o, lse, causal, cfg.scale, stream)
            units = ff / 1e12
        else:
            det = name.startswith("bwd_det")
            fn = lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, causal, cfg.scale, stream, deterministic=det)
            units = fb / 1e12
        if not name.startswith("quant"):
            unit = "TFLOP/s"
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ts)
    print(json.dumps({"case": name, "ms": ms, "rate": units / (ms / 1e3), "unit": unit,
                      "device_status": fa.fa_get_device_error()}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--clock-log", default=None, help="CSV file for the raw nvidia-smi clock samples")
    ap.add_argument("--no-extra", action="store_true", help="skip the side measurements (sweep, variants, decode)")
    ap.add_argument("--case", choices=CASES, default=None,
                    help="time one C-ABI call on one workload (single-kernel profiling), not the contract line")
    args = ap.parse_args(argv)
    if args.case:
        return run_case(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
