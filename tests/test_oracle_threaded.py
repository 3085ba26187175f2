"""The threaded oracle driver (oracle.threaded) returns exactly what the
single-threaded whole-tensor oracle returns: it only cuts rows into chunks,
runs the oracle's row entry points on a thread pool and joins the pieces.
Checked with few threads (many chunks per group, chunks crossing group
boundaries) on ragged and empty groups, one group, and a tensor whose
largest magnitude sits in a single row of one chunk."""
from __future__ import annotations

import numpy as np
import pytest

from fp4_quantization_aware_trace_b200 import inputs


def _same(a, b, name):
    a, b = np.asarray(a).reshape(-1), np.asarray(b).reshape(-1)
    if a.dtype == np.float32:
        a, b = a.view(np.uint32), b.view(np.uint32)
    assert a.shape == b.shape and np.array_equal(a, b), name


@pytest.mark.parametrize("threads", [1, 3, 8])
@pytest.mark.parametrize("groups", [None, [0, 37, 37, 100, 333, 400]])
def test_threaded_equals_whole_tensor(oracle_mod, threads, groups):
    import oracle.threaded as ot
    site = inputs.tiny_site(77, 400, 256)
    xr, xt, g = (inputs.bits(t) for t in (site.x_roll, site.x_train, site.grad))
    xr = xr.copy()
    xr[211, 5] = 0x4780  # one outlier (65536) in a single row
    G = 1 if groups is None else len(groups) - 1
    offs = None if groups is None else np.array(groups, np.int64)
    ref = oracle_mod.capture(xr, G, offs)
    got = ot.capture_mt(xr, G, offs, threads=threads)
    for name, a, b in zip(("codes", "mbits", "scales", "gscale"), got, ref):
        _same(a, b, name)
    codes, mbits, scales, gscale = ref
    _same(ot.group_amax_mt(xr, G, offs, threads), oracle_mod.group_amax(xr, G, offs), "amax")
    o, m = oracle_mod.guided_fwd(xt, mbits, scales, gscale, G, offs)
    og, mg = ot.guided_fwd_mt(xt, mbits, scales, gscale, G, offs, threads)
    _same(og, o, "guided out")
    _same(mg, m, "guided mask")
    r, rm = oracle_mod.rtn_fwd(xt, scales, gscale, G, offs)
    rg, rmg = ot.rtn_fwd_mt(xt, scales, gscale, G, offs, threads)
    _same(rg, r, "rtn out")
    _same(rmg, rm, "rtn mask")
    f, fm = oracle_mod.full_guided_fwd(xt, codes, scales, gscale, G, offs)
    fg, fmg = ot.full_guided_fwd_mt(xt, codes, scales, gscale, G, offs, threads)
    _same(fg, f, "full out")
    _same(fmg, fm, "full mask")
    _same(ot.fq_bwd_mt(g, m, threads), oracle_mod.fq_bwd(g, m), "grad_in")


def test_chunks_cover_rows_once():
    import oracle.threaded as ot
    for rows in (0, 1, 5, 64, 1000, 4097):
        for pieces in (1, 3, 7, 64):
            for q in (1, 8):
                c = ot._chunks(rows, pieces, q)
                assert [a for a, _ in c] == sorted({a for a, _ in c})
                assert sum(b - a for a, b in c) == rows
                assert all(b > a for a, b in c)
                assert all(a % q == 0 for a, _ in c)
                if c:
                    assert c[0][0] == 0 and c[-1][1] == rows
                    assert all(c[i][1] == c[i + 1][0] for i in range(len(c) - 1))


def test_cores_is_the_affinity_mask():
    import os

    import oracle.threaded as ot
    assert ot.cores() == len(os.sched_getaffinity(0)) >= 1
