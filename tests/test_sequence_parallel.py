"""Sequence-parallel decode (key positions split across ranks).

CPU, gloo, world size 2: the host logic of io_aware_exact_32_b200.sequence_parallel (slicing,
the all-gather of partials, the merge over ranks) with per-rank partials and the merge computed on
the CPU from the oracle's definitions.  GPU (one device): two ranks emulated in one process through
fa_decode_partials and fa_decode_merge, against the oracle's full decode.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_exact_32_b200 import sequence_parallel as sp
from io_aware_exact_32_b200 import workloads as W
from oracle import attention as A

LOG2E = 1.0 / math.log(2.0)


def test_slices_cover_every_position_once():
    for Lmax, world in ((100, 2), (8192, 8), (7, 3), (5, 8)):
        covered = []
        for r in range(world):
            start, Ls = sp.slice_bounds(Lmax, r, world)
            covered += [p for p in range(start, start + Ls) if p < Lmax]
        assert covered == list(range(Lmax))
    lens = torch.tensor([0, 1, 50, 51, 100])
    got = [sp.local_lengths(lens, r, 2, 100).tolist() for r in range(2)]
    assert got == [[0, 1, 50, 50, 50], [0, 0, 0, 1, 50]]


def cpu_partials(q, k, v, lens, part_o, part_ml, scale=None, num_splits=0, stream=None):
    """Per split of the slice: m in log2 units of scale * q.k, l = sum 2^(x - m), unnormalised O."""
    B, H, S, d = part_o.shape
    Ls = k.shape[2]
    C = math.ceil(Ls / S)
    qq = q.double()[:, :, 0, :]
    for b in range(B):
        for h in range(H):
            for s in range(S):
                lo, hi = s * C, min((s + 1) * C, int(lens[b]))
                if hi <= lo:
                    part_o[b, h, s] = 0.0
                    part_ml[b, h, s] = torch.tensor([-math.inf, 0.0])
                    continue
                x = (k.double()[b, h, lo:hi] @ qq[b, h]) * scale * LOG2E
                m = x.max()
                w = torch.exp2(x - m)
                part_o[b, h, s] = (w[:, None] * v.double()[b, h, lo:hi]).sum(0).float()
                part_ml[b, h, s] = torch.tensor([float(m), float(w.sum())])


def cpu_merge(all_o, all_ml, o, lse, stream=None):
    """Pairwise merges with the oracle's two-block identity (natural-log units)."""
    R, B, H, S, d = all_o.shape
    for b in range(B):
        for h in range(H):
            ms = all_ml[:, b, h, :, 0].double().reshape(-1).numpy() / LOG2E
            ls = all_ml[:, b, h, :, 1].double().reshape(-1).numpy()
            os_ = all_o[:, b, h].double().reshape(-1, d).numpy()
            m, l, acc = -np.inf, 0.0, np.zeros(d)
            for mi, li, oi in zip(ms, ls, os_):
                m_new, f, l = A.merge_two_blocks(np.array(m), np.array([1.0]), np.array(l),
                                                 np.array(mi), np.array([1.0]), np.array(li))
                acc = f[0] * acc + f[1] * oi
                m = float(m_new)
            o[b, h, 0] = torch.tensor(acc / l if l > 0 else np.zeros(d)).to(o.dtype)
            lse[b, h] = float(m + np.log(l)) if l > 0 else -math.inf


def _worker(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, Lmax, d = 2, 2, 37, 8
        x = W.make_decode_inputs(B, H, Lmax, d, 5, 11)
        start, Ls = sp.slice_bounds(Lmax, rank, world)
        kl = torch.zeros(B, H, Ls, d, dtype=torch.bfloat16)
        vl = torch.zeros(B, H, Ls, d, dtype=torch.bfloat16)
        n = min(Ls, Lmax - start)
        kl[:, :, :n] = x["k_cache"][:, :, start:start + n]
        vl[:, :, :n] = x["v_cache"][:, :, start:start + n]
        lens = sp.local_lengths(x["seqlens"], rank, world, Lmax)
        o, lse = sp.decode_sequence_parallel(x["q"], kl, vl, lens, scale=1.0 / math.sqrt(d), num_splits=3,
                                             partials_fn=cpu_partials, merge_fn=cpu_merge)
        q_out.put((rank, o.float().numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.timeout(120)
def test_two_ranks_match_full_decode():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=100) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    B, H, Lmax, d = 2, 2, 37, 8
    x = W.make_decode_inputs(B, H, Lmax, d, 5, 11)
    ro, rl = A.decode_forward(x["q"].double().numpy(), x["k_cache"].double().numpy(), x["v_cache"].double().numpy(),
                              x["seqlens"].numpy(), 1.0 / math.sqrt(d))
    for _, o, lse in res:
        assert np.max(np.abs(o[:, :, 0] - ro)) < 1e-2
        assert np.max(np.abs(lse - rl)) < 1e-4
    assert np.array_equal(res[0][1], res[1][1])       # every rank holds the same result


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_gpu_two_slices_merge_to_full_decode(d):
    import io_aware_exact_32_b200 as fa
    B, H, Lmax, world = 4, 8, 3000, 2
    x = W.make_decode_inputs(B, H, Lmax, d, 200, 19 + d)
    x["seqlens"][0] = 1200                              # the second slice of sequence 0 is empty
    dev = torch.device("cuda:0")
    scale = 1.0 / math.sqrt(d)
    qd = x["q"].to(dev)
    parts_o, parts_ml = [], []
    for r in range(world):
        start, Ls = sp.slice_bounds(Lmax, r, world)
        n = min(Ls, Lmax - start)
        kl = torch.zeros(B, H, Ls, d, dtype=torch.bfloat16, device=dev)
        vl = torch.zeros(B, H, Ls, d, dtype=torch.bfloat16, device=dev)
        kl[:, :, :n] = x["k_cache"][:, :, start:start + n].to(dev)
        vl[:, :, :n] = x["v_cache"][:, :, start:start + n].to(dev)
        lens = sp.local_lengths(x["seqlens"], r, world, Lmax).to(torch.int32).to(dev)
        S = fa.fa_decode_num_splits(Ls)
        po = torch.empty(B, H, S, d, dtype=torch.float32, device=dev)
        pm = torch.empty(B, H, S, 2, dtype=torch.float32, device=dev)
        fa.fa_decode_partials(qd, kl, vl, lens, po, pm, scale=scale)
        parts_o.append(po)
        parts_ml.append(pm)
    o = torch.empty(B, H, 1, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    fa.fa_decode_merge(torch.stack(parts_o), torch.stack(parts_ml), o, lse)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    ro, rl = A.decode_forward(x["q"].double().numpy(), x["k_cache"].double().numpy(), x["v_cache"].double().numpy(),
                              x["seqlens"].numpy(), scale)
    assert np.max(np.abs(o[:, :, 0].double().cpu().numpy() - ro)) < 1e-2
    assert np.max(np.abs(lse.double().cpu().numpy() - rl)) < 1e-3
