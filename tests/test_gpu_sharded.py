"""Row-sharded capture on two ranks (ops.capture_sharded): each rank holds
half of every group's rows, runs the amax pass on its shard, the per-group
maxima are all-reduced (MAX), and each rank quantises its shard with the
global scales of the whole tensor.  Both ranks run on cuda:0 and reduce over
gloo (CUDA tensors), so no peer memory and no NCCL are involved; nothing on
the device waits for the other rank.  Each rank's codes, mantissa bits and
scales must equal the oracle's capture of the whole tensor on that rank's
rows, and its global scales the oracle's whole-tensor ones."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROWS, COLS, G = 512, 256, 4
PER = ROWS // G  # rows per group; each rank holds half of them


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _whole_tensor():
    from fp4_quantization_aware_trace_b200 import inputs
    x = inputs.tiny_site(4321, ROWS, COLS).x_roll.float()
    # the largest magnitude of group 1 sits in rank 1's half, that of group 2
    # in rank 0's half: the reduction has to bring each one across
    x[PER + PER // 2 + 5, 3] = 1000.0
    x[2 * PER + 7, 9] = -2000.0
    x[3 * PER:] *= 1e-3  # a group with much smaller values
    return x.to(torch.bfloat16)


def _shard_rows(rank: int) -> np.ndarray:
    h = PER // 2
    return np.concatenate([np.arange(g * PER + rank * h, g * PER + rank * h + h)
                           for g in range(G)])


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    from fp4_quantization_aware_trace_b200 import ops
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rows = _shard_rows(rank)
        xs = _whole_tensor()[torch.from_numpy(rows)].contiguous().cuda()
        offs = torch.arange(0, len(rows) + 1, PER // 2, dtype=torch.int64, device="cuda")
        cap = ops.capture_sharded(xs, offs, group=dist.group.WORLD)
        torch.cuda.synchronize()
        q.put((rank, cap.codes.cpu().numpy(), cap.mbits.cpu().numpy().view(np.uint32),
               cap.scales.cpu().numpy(), cap.gscale.cpu().numpy()))
    except Exception as exc:  # report, so the parent does not wait for nothing
        q.put((rank, repr(exc), None, None, None))
        raise
    finally:
        dist.destroy_process_group()


def test_capture_sharded_two_ranks_matches_whole_tensor(oracle_mod):
    from fp4_quantization_aware_trace_b200 import inputs
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    x = inputs.bits(_whole_tensor())
    offs = np.arange(0, ROWS + 1, PER, dtype=np.int64)
    codes, mbits, scales, gscale = oracle_mod.capture(x, G, offs)
    codes = codes.reshape(ROWS, COLS // 2)
    mbits = mbits.reshape(ROWS, COLS // 32)
    scales = scales.reshape(ROWS, COLS // 16)
    for rank, c, m, s, gs in res:
        assert not isinstance(c, str), c
        rows = _shard_rows(rank)
        assert np.array_equal(gs.view(np.uint32), gscale.view(np.uint32)), rank
        assert np.array_equal(c.reshape(len(rows), -1), codes[rows]), rank
        assert np.array_equal(m.reshape(len(rows), -1), mbits[rows]), rank
        assert np.array_equal(s.reshape(len(rows), -1), scales[rows]), rank
