#!/usr/bin/env python
"""Benchmark of the exact fused attention path on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (per GPU): B=2, H=8, Nq=Nk=1024, d=64, bf16 inputs iid N(0,1);
one step = forward + backward with the causal mask, then forward + backward
without it, all through the C ABI, captured once as a CUDA graph and replayed
for every timed step (`--no-graph`: eager launches; the eager rate is reported
beside it either way).  `value` is whole-job TFLOP/s by the
FLOP convention 4*B*H*Nq*Nk*d per forward (halved when causal) and 2.5x that
per backward.  L2 is flushed (a 256 MiB write) before every timed step.

Alongside: `e2e` (the same step through the C ABI from pinned host buffers,
host<->device copies inside the timed region), the roofline of the dominant
kernel, a CPU-oracle baseline, and `extra` measurements of the d=128 causal
N=4096 forward / forward+backward and of split-KV decode (HBM GB/s).

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

    def __init__(self, gpu_index: int, path: str | None = None):
        self.gpu = str(gpu_index)
        self.proc = None
        # The raw samples are kept where --clock-log asks (else a temporary file); the summary
        # goes into the JSON line either way.
        self.path = path or os.path.join(tempfile.gettempdir(), f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", self.gpu], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
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


# --------------------------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(seconds: float, seed: int = 1):
    """Time the float64 oracle on whole (batch, head) slices of the headline workload.

    Returns (flops_done, elapsed, heads_done, threads)."""
    import numpy as np
    from io_aware_exact_32_b200 import workloads as W
    from oracle import attention as A
    c = W.C2
    x = W.make_attention_inputs(c.B, c.H, c.Nq, c.Nk, c.d, seed)
    q, k, v, do = (x[n].double().numpy() for n in ("q", "k", "v", "do"))
    per_head = sum(W.flops_forward(1, 1, c.Nq, c.Nk, c.d, cz) + W.flops_backward(1, 1, c.Nq, c.Nk, c.d, cz)
                   for cz in (True, False))
    t0 = time.perf_counter()
    heads = 0
    while True:
        b, h = divmod(heads % (c.B * c.H), c.H)
        for causal in (True, False):
            A.attention_forward_head(q[b, h], k[b, h], v[b, h], c.scale, causal)
            A.attention_backward_head(q[b, h], k[b, h], v[b, h], do[b, h], c.scale, causal)
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return per_head * heads, el, heads, blas_threads()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from io_aware_exact_32_b200 import workloads as W
    c = W.C2
    for _ in range(args.warmup):
        cpu_oracle_sample(0.0)
    flops, secs = 0.0, 0.0
    for _ in range(args.steps):
        f, el, _, threads = cpu_oracle_sample(0.0)
        flops += f
        secs += el
    value = flops / secs / 1e12
    sample = (f"{args.steps} steps, each one (batch, head) slice of B={c.B} H={c.H} N={c.Nq} d={c.d}: "
              f"forward+backward causal and non-causal in float64 numpy")
    line = {
        "impl": "reference", "metric": "attention fwd+bwd TFLOP/s (causal + non-causal step)", "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"b{c.B}_h{c.H}_n{c.Nq}_d{c.d} fwd+bwd causal+noncausal (one head per step)",
                   "global_batch": c.B, "seq_len": c.Nq, "parallelism": "none (host cores)"},
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

    c = W.C2
    x = W.make_attention_inputs(c.B, c.H, c.Nq, c.Nk, c.d, shard_seed(c.seed, rank))
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, N, d = c.B, c.H, c.Nq, c.d
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    out = {}
    for causal in (True, False):
        out[causal] = dict(o=torch.empty_like(q), lse=torch.empty(B, H, N, device=dev, dtype=torch.float32),
                           dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v))
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    step_flops = sum(W.flops_forward(B, H, N, N, d, cz) + W.flops_backward(B, H, N, N, d, cz) for cz in (True, False))
    calls = [("fwd_causal", True, "fwd"), ("bwd_causal", True, "bwd"), ("fwd_noncausal", False, "fwd"),
             ("bwd_noncausal", False, "bwd")]
    call_flops = {name: (W.flops_forward if kind == "fwd" else W.flops_backward)(B, H, N, N, d, cz)
                  for name, cz, kind in calls}
    launches_per_step = 2 * (1 + 3)  # fa_fwd: 1 kernel; fa_bwd: preprocess + main + dQ convert

    def step(events=None, st=None):
        st = stream if st is None else st
        for i, (name, cz, kind) in enumerate(calls):
            o = out[cz]
            if events is not None:
                events[i][0].record(st)
            if kind == "fwd":
                fa.fa_fwd(q, k, v, o["o"], o["lse"], cz, c.scale, st)
            else:
                fa.fa_bwd(q, k, v, o["o"], do, o["lse"], o["dq"], o["dk"], o["dv"], ws, cz, c.scale, st)
            if events is not None:
                events[i][1].record(st)

    for _ in range(args.warmup):
        flush_buf.zero_()
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    # One step captured as a CUDA graph (the launch-bound inner loop: 8 small kernel launches);
    # every timed iteration replays it, with the L2 flush and the events outside the graph.
    graph = None
    if not args.no_graph:
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            step(st=cap)
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            flush_buf.zero_()
            graph.replay()
        torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(dev.index if world == 1 else local, args.clock_log).start() if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(K):
        flush_buf.zero_()
        ev[s][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    status = fa.fa_get_device_error()
    step_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    total_s = reduce_max(sum(step_ms) / 1e3, world, dev)
    value = whole_job_rate(step_flops * K, world, total_s) / 1e12

    # Per-call device times (eager launches, events around each C-ABI call) for the roofline.
    Kc = min(K, 500)
    call_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
               for _ in range(Kc)]
    eager_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Kc)]
    for s in range(Kc):
        flush_buf.zero_()
        eager_ev[s][0].record(stream)
        step(call_ev[s])
        eager_ev[s][1].record(stream)
    torch.cuda.synchronize()
    call_ms = {name: statistics.mean(call_ev[s][i][0].elapsed_time(call_ev[s][i][1]) for s in range(Kc))
               for i, (name, _, _) in enumerate(calls)}
    eager_s = reduce_max(sum(a.elapsed_time(b) for a, b in eager_ev) / 1e3, world, dev)
    value_eager = whole_job_rate(step_flops * Kc, world, eager_s) / 1e12

    # ---------------------------------------------------------------- end to end from host buffers
    # Every step copies its inputs from pinned host memory and reads all its outputs back; the
    # copies of one step overlap the compute of its neighbours (upload stream -> compute stream ->
    # read-back stream, device buffers double-buffered).  The L2 flush stays on the compute stream,
    # inside the timed region.  e2e_serial: the same step with copies and compute in sequence.
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
    dev_in = [tuple(torch.empty_like(t) for t in (q, k, v, do)) for _ in range(2)]
    dev_out = [{cz: {n: torch.empty_like(t) for n, t in out[cz].items()} for cz in (True, False)} for _ in range(2)]
    host_out = [{cz: {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in out[cz].items()}
                 for cz in (True, False)} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for cz in (True, False) for t in host_out[0][cz].values())
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def compute(buf, dst):
        dq_, dk_, dv_, dd_ = buf
        for name, cz, kind in calls:
            o = dst[cz]
            if kind == "fwd":
                fa.fa_fwd(dq_, dk_, dv_, o["o"], o["lse"], cz, c.scale, stream)
            else:
                fa.fa_bwd(dq_, dk_, dv_, o["o"], dd_, o["lse"], o["dq"], o["dk"], o["dv"], ws, cz, c.scale, stream)

    def e2e_serial_step():
        buf, dst, hst = dev_in[0], dev_out[0], host_out[0]
        for d_, h_ in zip(buf, (hq, hk, hv, hdo)):
            d_.copy_(h_, non_blocking=True)
        compute(buf, dst)
        for cz in (True, False):
            for n, t in dst[cz].items():
                hst[cz][n].copy_(t, non_blocking=True)

    def e2e_pipelined(n_steps, flush):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, computed, read_back = [], [], []
        for st in range(n_steps):
            slot = st % 2
            with torch.cuda.stream(up):
                if st >= 2:
                    up.wait_event(computed[st - 2])  # that step is done with this input buffer
                for d_, h_ in zip(dev_in[slot], (hq, hk, hv, hdo)):
                    d_.copy_(h_, non_blocking=True)
                in_ready.append(ev())
                in_ready[-1].record(up)
            stream.wait_event(in_ready[st])
            if flush:
                flush_buf.zero_()
            if st >= 2:
                stream.wait_event(read_back[st - 2])  # that step's outputs are on the host
            compute(dev_in[slot], dev_out[slot])
            computed.append(ev())
            computed[-1].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[st])
                for cz in (True, False):
                    for n, t in dev_out[slot][cz].items():
                        host_out[slot][cz][n].copy_(t, non_blocking=True)
                read_back.append(ev())
                read_back[-1].record(down)
        return read_back[-1]

    for _ in range(max(1, args.warmup)):
        e2e_serial_step()
    e2e_pipelined(4, True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(up)
    last = e2e_pipelined(K, True)
    down.wait_event(last)
    t1.record(down)
    torch.cuda.synchronize()
    e2e_s = reduce_max(t0.elapsed_time(t1) / 1e3, world, dev)
    e2e_value = whole_job_rate(step_flops * K, world, e2e_s) / 1e12
    ser_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(min(K, 200))]
    if world > 1:
        dist.barrier()
    for a_, b_ in ser_ev:
        flush_buf.zero_()
        a_.record(stream)
        e2e_serial_step()
        b_.record(stream)
    torch.cuda.synchronize()
    ser_s = reduce_max(sum(a_.elapsed_time(b_) for a_, b_ in ser_ev) / 1e3, world, dev)
    e2e_serial_value = whole_job_rate(step_flops * len(ser_ev), world, ser_s) / 1e12

    # ---------------------------------------------------------------- dominant kernel roofline
    # The kernel with the most time per step (fa_bwd_main_kernel, in both mask modes) is timed per
    # fa_bwd call; the call also holds the two small preprocess / dQ-convert kernels, so the
    # achieved rate understates the main kernel slightly.
    kind_ms = {k: sum(call_ms[n] for n, _, kk in calls if kk == k) for k in ("fwd", "bwd")}
    dom = max(kind_ms, key=lambda k: kind_ms[k])
    dom_flops = sum(call_flops[n] for n, _, kk in calls if kk == dom)
    dom_tflops = dom_flops / (kind_ms[dom] / 1e3) / 1e12
    roofline = {"bound": "tensor",
                "kernel": ("fa_bwd_main_kernel<64>, timed per fa_bwd call (with its preprocess and dQ-convert "
                           "kernels), causal + non-causal" if dom == "bwd"
                           else "fa_fwd_kernel<64>, causal + non-causal"),
                "achieved": dom_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": dom_tflops / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                else "fallback 1590 TFLOP/s"}

    if dom == "bwd":
        roofline["traffic"], roofline["traffic_source"] = captured_traffic("fa_bwd_main_kernel<64> b2_h8_n1024_d64")
        if roofline["traffic"] is not None:
            roofline["traffic_unit"] = "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)"

    extra = {}
    if not args.no_extra and world == 1:  # single-GPU kernel measurements; the N > 1 line is the headline alone
        extra = extra_measurements(fa, W, dev, stream, flush_buf, peaks)

    if world > 1:
        dist.barrier()
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu:
            f, el, heads, threads = cpu_oracle_sample(args.cpu_seconds)
            cpu = {"value": f / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                   "sample": f"{heads} (batch, head) slices of the headline workload, fwd+bwd causal and "
                             f"non-causal, float64 numpy, {el:.1f} s"}
        line = {
            "metric": "attention fwd+bwd TFLOP/s (causal + non-causal step)", "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (iid N(0,1) bf16, seeded per rank)",
            "config": {"workload": f"b{B}_h{H}_n{N}_d{d} fwd+bwd causal+noncausal", "global_batch": B * world,
                       "seq_len": N, "heads": H, "head_dim": d, "parallelism": f"dp{world} over (batch, head)",
                       "l2": "flushed before every timed step (256 MiB write)",
                       "launch": "CUDA graph of one step, replayed" if graph is not None else "eager"},
            "value_eager_launches": value_eager,
            "frac_of_peak": value / world / peaks["bf16_tflops"],
            "per_call_ms": call_ms,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "overlapped with the neighbouring steps' compute (upload, compute and read-back streams)",
                    "serial_value": e2e_serial_value},
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


def long_context_measurement(fa, W, dev, stream, peaks, timed, cfg=None):
    """Causal forward and forward+backward on the long-context case (B=1, H=16, N=65536, d=128, 1% of
    key rows x8); ``timed(fn)`` returns seconds per call."""
    import torch
    c = cfg or W.LONG
    x = W.make_config_inputs(c)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    del x
    o, lse = fa.attention_forward(q, k, v, causal=True, scale=c.scale)
    ws = torch.empty(fa.fa_bwd_workspace_size(c.B, c.H, c.Nq, c.d), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    t_f = timed(lambda: fa.fa_fwd(q, k, v, o, lse, True, c.scale, stream))
    t_b = timed(lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, True, c.scale, stream))
    ff = W.flops_forward(c.B, c.H, c.Nq, c.Nk, c.d, True)
    fb = W.flops_backward(c.B, c.H, c.Nq, c.Nk, c.d, True)
    f1, f2 = ff / t_f / 1e12, (ff + fb) / (t_f + t_b) / 1e12
    return {"B": c.B, "H": c.H, "N": c.Nq, "fwd_tflops": f1, "fwd_frac": f1 / peaks["bf16_tflops"],
            "fwd_frac_of_2250": f1 / 2250.0, "bwd_tflops": fb / t_b / 1e12, "fwd_bwd_tflops": f2,
            "fwd_bwd_frac": f2 / peaks["bf16_tflops"], "fwd_bwd_frac_of_2250": f2 / 2250.0, "fwd_ms": 1e3 * t_f,
            "bwd_ms": 1e3 * t_b, "device_status": fa.fa_get_device_error(stream)}


def extra_measurements(fa, W, dev, stream, flush_buf, peaks, iters=10):
    """d=128 causal forward and forward+backward at N = 4096, 8192, 16384 (the sweep's B*N = 16384
    tokens, H=16), the FP8 and bias / dropout variants, the deterministic backward, split-KV decode
    bandwidth, and the 65536-token causal case."""
    import torch
    res = {}

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

    for n in (4096, 8192, 16384):
        cfg = next(c for c in W.SWEEP if c.Nq == n and c.d == 128)
        x = W.make_config_inputs(cfg)
        q, k, v, do = (x[nm].to(dev) for nm in ("q", "k", "v", "do"))
        o, lse = fa.attention_forward(q, k, v, causal=True, scale=cfg.scale)
        ws = torch.empty(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        t_f = timed(lambda: fa.fa_fwd(q, k, v, o, lse, True, cfg.scale, stream))
        t_b = timed(lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, True, cfg.scale, stream))
        ff = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, True)
        fb = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, True)
        fwd_t, fb_t = ff / t_f / 1e12, (ff + fb) / (t_f + t_b) / 1e12
        res[f"causal_n{n}_d128"] = {"B": cfg.B, "H": cfg.H, "fwd_tflops": fwd_t, "fwd_frac": fwd_t / peaks["bf16_tflops"],
                                    "fwd_frac_of_2250": fwd_t / 2250.0, "bwd_tflops": fb / t_b / 1e12,
                                    "fwd_bwd_tflops": fb_t, "fwd_bwd_frac": fb_t / peaks["bf16_tflops"],
                                    "fwd_bwd_frac_of_2250": fb_t / 2250.0, "fwd_ms": 1e3 * t_f, "bwd_ms": 1e3 * t_b}
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
            "fwd_incl_quantize_tflops": ff / (t_f8 + t_q8) / 1e12}
        del q8, k8, v8, dsq, dsk, dsv, o8, lse8
        if n == 4096:
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
                "note": "bias [1, H, N, N] bf16 (read once per query tile), dropout p = 0.1"}
            del bias, oe, lsee
            t_bd = timed(lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, True, cfg.scale, stream,
                                           deterministic=True))
            res["deterministic_bwd_causal_n4096_d128"] = {"bwd_tflops": fb / t_bd / 1e12, "bwd_ms": 1e3 * t_bd,
                                                          "vs_default_bwd": t_b / t_bd}
        del q, k, v, do, o, lse, dq, dk, dv, ws, x
    # Its failure is recorded rather than raised, so that the lines above are still reported.
    try:
        res["long_n65536_d128_causal_peaked"] = long_context_measurement(fa, W, dev, stream, peaks, timed)
    except Exception as e:  # noqa: BLE001 - reported in the JSON line
        res["long_n65536_d128_causal_peaked"] = {"error": f"{type(e).__name__}: {e}"}
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
                                        "ms": 1e3 * t_d, "algorithmic_bytes": nbytes}
    return res


CASES = ("fwd_c2", "bwd_c2", "fwd_n4096_d128", "bwd_n4096_d128", "fwd_fp8_n4096_d128", "fwd_ext_n4096_d128",
         "bwd_ext_n4096_d128", "decode")


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
        cfg = W.C2 if name.endswith("c2") else next(c for c in W.SWEEP if c.Nq == 4096 and c.d == 128)
        causal = True
        x = W.make_config_inputs(cfg)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
        o, lse = fa.attention_forward(q, k, v, causal=causal, scale=cfg.scale)
        if name.startswith("fwd_fp8"):
            signs = W.make_hadamard_signs(cfg.d, 11).to(dev)
            q8, dsq = fa.quantize_fp8(q, signs, True, stream)
            k8, dsk = fa.quantize_fp8(k, signs, True, stream)
            v8, dsv = fa.quantize_fp8(v, None, False, stream)
            fn = lambda: fa.fa_fwd_fp8(q8, k8, v8, dsq, dsk, dsv, o, lse, causal, cfg.scale, stream)
            units = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal) / 1e12
        elif name.endswith("ext_n4096_d128"):
            gb = torch.Generator().manual_seed(9)
            bias = (torch.randn(1, cfg.H, cfg.Nq, cfg.Nk, generator=gb) * 0.5).to(torch.bfloat16).to(dev)
            fa.fa_fwd_ext(q, k, v, o, lse, bias, causal, cfg.scale, 0.1, 1234, 0, stream)
            if name.startswith("fwd"):
                fn = lambda: fa.fa_fwd_ext(q, k, v, o, lse, bias, causal, cfg.scale, 0.1, 1234, 0, stream)
                units = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal) / 1e12
            else:
                ws = torch.empty(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), dtype=torch.uint8, device=dev)
                dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
                fn = lambda: fa.fa_bwd_ext(q, k, v, o, do, lse, dq, dk, dv, ws, bias, causal, cfg.scale, 0.1, 1234, 0,
                                           stream)
                units = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal) / 1e12
        elif name.startswith("fwd"):
            fn = lambda: fa.fa_fwd(q, k, v, o, lse, causal, cfg.scale, stream)
            units = W.flops_forward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal) / 1e12
        else:
            ws = torch.empty(fa.fa_bwd_workspace_size(cfg.B, cfg.H, cfg.Nq, cfg.d), dtype=torch.uint8, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            fn = lambda: fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, causal, cfg.scale, stream)
            units = W.flops_backward(cfg.B, cfg.H, cfg.Nq, cfg.Nk, cfg.d, causal) / 1e12
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
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--clock-log", default=None, help="CSV file for the raw nvidia-smi clock samples")
    ap.add_argument("--no-extra", action="store_true", help="skip the d=128 and decode side measurements")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of a replayed CUDA graph")
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
