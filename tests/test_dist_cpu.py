"""The multi-rank plumbing of bench.py on CPU with gloo (world size 2):
per-rank sites differ, timings reduce to the max over ranks, and the
whole-job value counts every rank's elements once."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from fp4_quantization_aware_trace_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        times = [10.0 + rank, 1.0 * (world - rank), 3.0]
        got = bench.max_over_ranks(times, dist, "cpu")
        site = inputs.attention_input(seed=bench.site_seed(rank), rows=64, cols=128)
        digest = float(site.x_roll.float().abs().sum())
        dig = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(dig, torch.tensor([digest], dtype=torch.float64))
        q.put((rank, got, [float(d) for d in dig]))
    finally:
        dist.destroy_process_group()


def test_two_rank_plumbing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, dig in res:
        assert got == [11.0, 2.0, 3.0]          # element-wise max over ranks
        assert dig[0] != dig[1]                 # each rank has its own site


def test_job_value_counts_every_rank():
    import bench
    one = bench.job_gbs(1, 1000, 17.3125, 2.0)
    assert bench.job_gbs(4, 1000, 17.3125, 2.0) == pytest.approx(4 * one)
    assert bench.job_gbs(2, 1000, 17.3125, 4.0) == pytest.approx(one)
    assert bench.max_over_ranks([1.5, 2.5], None, "cpu") == [1.5, 2.5]


def _amax_worker(rank, world, port, q):
    """Each rank holds a row shard; the per-group amax (bf16 bit patterns in
    int32, as trace_capture_amax writes them) is all-reduced with MAX."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(100 + rank)
        vals = np.abs(rng.standard_normal(7).astype(np.float32)) * 10.0 ** rng.integers(-30, 30, 7)
        vals[rank] = 0.0                                     # a group empty on this shard
        bits = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).to(torch.int32)
        local = bits.clone()
        dist.all_reduce(bits, op=dist.ReduceOp.MAX)
        allv = [torch.zeros(7, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(allv, local)
        q.put((rank, bits.tolist(), [a.tolist() for a in allv]))
    finally:
        dist.destroy_process_group()


def test_sharded_amax_reduction():
    """The one collective of a row-sharded capture: MAX over the bf16 bit
    patterns equals the bit pattern of the largest magnitude, on every rank."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_amax_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, red, allv in res:
        for g in range(7):
            mags = [torch.tensor([a[g]], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float().item()
                    for a in allv]
            want = torch.tensor([max(mags)]).to(torch.bfloat16).view(torch.int16).item()
            assert red[g] == want
