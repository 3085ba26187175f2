"""Multi-threaded driver of the CPU oracle -- TEST INFRASTRUCTURE.

Only ``tests/`` and ``bench.py``'s CPU legs use it.  It holds no arithmetic
of the method: it cuts a tensor into row chunks, runs the oracle's row entry
points (``group_amax``, ``capture_rows``, ``fake_quant_rows``,
``full_guided_rows``, ``fq_bwd``) on them from a pool of threads (ctypes
releases the GIL during each call, so the chunks run on separate cores), and
puts the pieces back together.  The per-group amax of a tensor is the maximum
of its chunks' maxima (max is exact and independent of order); the global
scale then comes from the oracle's own ``global_scale``.

Every function here returns exactly what the single-threaded whole-tensor
function of the same name in ``oracle`` returns (pinned by
``tests/test_oracle_threaded.py``).
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np

from . import (_as_bf16_bits, _offsets, capture_rows, fake_quant_rows, fq_bwd as _fq_bwd,
               full_guided_rows, global_scale, group_amax)


def cores() -> int:
    """Cores this process may run on (its affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


_pool = None
_pool_threads = 0


def _executor(threads: int) -> cf.ThreadPoolExecutor:
    global _pool, _pool_threads
    if _pool is None or _pool_threads != threads:
        if _pool is not None:
            _pool.shutdown(wait=True)
        _pool = cf.ThreadPoolExecutor(max_workers=threads)
        _pool_threads = threads
    return _pool


def _chunks(rows: int, pieces: int, quantum: int = 1) -> list[tuple[int, int]]:
    """About `pieces` row ranges [a, b) covering 0..rows (no empty range)."""
    if rows == 0:
        return []
    per = max(quantum, -(-rows // max(1, pieces)))
    per = -(-per // quantum) * quantum
    return [(a, min(rows, a + per)) for a in range(0, rows, per)]


def _map(fn, items, threads):
    if threads <= 1 or len(items) <= 1:
        return [fn(*it) for it in items]
    return list(_executor(threads).map(lambda it: fn(*it), items))


def row_gscales(gscale: np.ndarray, rows: int, num_groups: int = 1, offsets=None) -> np.ndarray:
    """The global scale of every row (the group's), f32[rows]."""
    g = np.ascontiguousarray(gscale, dtype=np.float32)
    if num_groups == 1:
        return np.full(rows, g[0], np.float32)
    o = _offsets(offsets, num_groups, rows)
    return np.repeat(g, np.diff(o)).astype(np.float32)


def group_amax_mt(x, num_groups: int = 1, offsets=None, threads: int | None = None) -> np.ndarray:
    """max |x| per group (f32[G]), each group's rows cut into chunks."""
    x = _as_bf16_bits(x)
    rows = x.shape[0]
    threads = threads or cores()
    o = _offsets(offsets, num_groups, rows)
    bounds = [(0, rows)] if o is None else [(int(o[g]), int(o[g + 1])) for g in range(num_groups)]
    work = []
    for g, (a, b) in enumerate(bounds):
        for ca, cb in _chunks(b - a, max(1, threads * 2 * (b - a) // max(1, rows))):
            work.append((g, a + ca, a + cb))
    amax = np.zeros(num_groups, np.float32)
    parts = _map(lambda g, a, b: (g, group_amax(x[a:b])[0]), work, threads)
    for g, m in parts:
        amax[g] = max(amax[g], m)
    return amax


def capture_mt(x, num_groups: int = 1, offsets=None, threads: int | None = None):
    """oracle.capture on row chunks: (codes, mbits, scales, gscale)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    threads = threads or cores()
    amax = group_amax_mt(x, num_groups, offsets, threads)
    gscale = np.array([global_scale(float(a)) for a in amax], np.float32)
    rg = row_gscales(gscale, rows, num_groups, offsets)
    parts = _map(lambda a, b: capture_rows(x[a:b], rg[a:b]), _chunks(rows, 4 * threads), threads)
    if not parts:
        return (np.zeros(0, np.uint8), np.zeros(0, np.uint32),
                np.zeros((0, cols // 16), np.uint8), gscale)
    codes = np.concatenate([p[0] for p in parts])
    mbits = np.concatenate([p[1] for p in parts])
    scales = np.concatenate([p[2] for p in parts])
    return codes, mbits, scales, gscale


def _fq_mt(x, gscale, scales, mbits, num_groups, offsets, threads):
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    threads = threads or cores()
    rg = row_gscales(gscale, rows, num_groups, offsets)
    sc = np.ascontiguousarray(scales, dtype=np.uint8).reshape(rows, cols // 16)
    mb = None if mbits is None else np.ascontiguousarray(mbits, np.uint32).reshape(rows, cols // 32)
    parts = _map(lambda a, b: fake_quant_rows(x[a:b], rg[a:b], sc[a:b],
                                              None if mb is None else mb[a:b]),
                 _chunks(rows, 4 * threads), threads)
    if not parts:
        return np.zeros((0, cols), np.uint16), np.zeros(0, np.uint32)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def guided_fwd_mt(x_train, mbits, scales, gscale, num_groups: int = 1, offsets=None,
                  threads: int | None = None):
    """oracle.guided_fwd on row chunks: (out, mask)."""
    return _fq_mt(x_train, gscale, scales, mbits, num_groups, offsets, threads)


def rtn_fwd_mt(x, scales, gscale, num_groups: int = 1, offsets=None, threads: int | None = None):
    """oracle.rtn_fwd on row chunks: (out, mask)."""
    return _fq_mt(x, gscale, scales, None, num_groups, offsets, threads)


def full_guided_fwd_mt(x_train, rcodes, scales, gscale, num_groups: int = 1, offsets=None,
                       threads: int | None = None):
    """oracle.full_guided_fwd on row chunks: (out, mask)."""
    x = _as_bf16_bits(x_train)
    rows, cols = x.shape
    threads = threads or cores()
    rg = row_gscales(gscale, rows, num_groups, offsets)
    sc = np.ascontiguousarray(scales, dtype=np.uint8).reshape(rows, cols // 16)
    rc = np.ascontiguousarray(rcodes, dtype=np.uint8).reshape(rows, cols // 2)
    parts = _map(lambda a, b: full_guided_rows(x[a:b], rg[a:b], sc[a:b], rc[a:b]),
                 _chunks(rows, 4 * threads), threads)
    if not parts:
        return np.zeros((0, cols), np.uint16), np.zeros(0, np.uint32)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def fq_bwd_mt(grad_out, mask, threads: int | None = None):
    """oracle.fq_bwd on chunks of 32-element words: grad_in bits."""
    g = np.ascontiguousarray(grad_out, dtype=np.uint16)
    shape = g.shape
    g = g.reshape(-1)
    m = np.ascontiguousarray(mask, dtype=np.uint32).reshape(-1)
    threads = threads or cores()
    parts = _map(lambda a, b: _fq_bwd(g[32 * a:32 * b], m[a:b]),
                 _chunks(m.size, 4 * threads), threads)
    if not parts:
        return np.zeros(shape, np.uint16)
    return np.concatenate(parts).reshape(shape)


def capture_rows_mt(x, row_gscale, threads: int | None = None):
    """oracle.capture_rows on row chunks (rows whose global scale is given
    per row): (codes, mbits, scales)."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    threads = threads or cores()
    rg = np.ascontiguousarray(row_gscale, dtype=np.float32)
    parts = _map(lambda a, b: capture_rows(x[a:b], rg[a:b]), _chunks(rows, 4 * threads), threads)
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))


def fake_quant_rows_mt(x, row_gscale, scales, mbits=None, threads: int | None = None):
    """oracle.fake_quant_rows on row chunks: (out, mask); guided when mbits
    is given, round to nearest otherwise."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    threads = threads or cores()
    rg = np.ascontiguousarray(row_gscale, dtype=np.float32)
    sc = np.ascontiguousarray(scales, dtype=np.uint8).reshape(rows, cols // 16)
    mb = None if mbits is None else np.ascontiguousarray(mbits, np.uint32).reshape(rows, cols // 32)
    parts = _map(lambda a, b: fake_quant_rows(x[a:b], rg[a:b], sc[a:b],
                                              None if mb is None else mb[a:b]),
                 _chunks(rows, 4 * threads), threads)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])
