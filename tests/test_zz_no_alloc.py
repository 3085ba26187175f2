"""The capture entry point that needs no workspace (trace_capture_static_ws).

Who it is for: callers that may not allocate device memory when they call
the library -- a program whose device memory is fixed at start-up, or a
binding that can only pass along the buffers it received -- and so cannot
hand trace_capture a workspace.  The library keeps that scratch in a static
per-GPU array instead.

This file is collected last on purpose, and it must pass both on its own in
a fresh process (its first call then does the one-time address lookup) and
after every other test.  It checks, through the C ABI, two calls in a row
against the ordinary trace_capture: outputs must be identical bit for bit
(the tolerance the parity tests use), and the second call must not see the
first call's leftovers in the shared array."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _outs(rows, cols, G):
    n = rows * cols
    return dict(codes=torch.full((n // 2,), 0x5A, dtype=torch.uint8, device=DEV),
                mbits=torch.full((n // 32,), -1, dtype=torch.int32, device=DEV),
                scales=torch.full((rows, cols // 16), 0x33, dtype=torch.uint8, device=DEV),
                gscale=torch.full((G,), -7.0, dtype=torch.float32, device=DEV))


def _reference(x, offs, G):
    rows, cols = x.shape
    o = _outs(rows, cols, G)
    ws = torch.zeros(ops.trace_capture_workspace_bytes(rows, cols, G), dtype=torch.uint8, device=DEV)
    ops.trace_capture(x, rows, cols, G, offs, o["codes"], o["mbits"], o["scales"], o["gscale"],
                      ws, ws.numel())
    return o


def _static(x, offs, G):
    rows, cols = x.shape
    o = _outs(rows, cols, G)
    ops.trace_capture_static_ws(x, rows, cols, G, offs, o["codes"], o["mbits"], o["scales"],
                                o["gscale"])
    return o


def _same(a, b):
    for k in a:
        assert torch.equal(a[k].view(torch.uint8), b[k].view(torch.uint8)), k


def test_static_workspace_capture_matches_two_calls_in_a_row():
    # call 1: ragged groups, one of them huge in magnitude so the shared
    # accumulators hold large values afterwards
    s1 = inputs.tiny_site(31, 700, 256)
    x1 = s1.x_roll.float()
    x1[100:200] *= 1e6
    x1 = x1.to(torch.bfloat16).to(DEV)
    offs1 = torch.tensor([0, 100, 200, 200, 650, 700], dtype=torch.int64, device=DEV)
    got1 = _static(x1, offs1, 5)
    ref1 = _reference(x1, offs1, 5)
    # call 2: small values in one group; leftovers from call 1 would show up
    # as a wrong (too large) global scale
    s2 = inputs.tiny_site(32, 512, 128)
    x2 = (s2.x_roll.float() * 1e-3).to(torch.bfloat16).to(DEV)
    got2 = _static(x2, None, 1)
    ref2 = _reference(x2, None, 1)
    torch.cuda.synchronize()
    _same(got1, ref1)
    _same(got2, ref2)
    assert float(got2["gscale"][0]) < 1.0


def test_static_workspace_rejects_too_many_groups():
    lib = ops.library()
    G = ops.TRACE_STATIC_MAX_GROUPS + 1
    x = torch.zeros(G, 32, dtype=torch.bfloat16, device=DEV)
    offs = torch.arange(G + 1, dtype=torch.int64, device=DEV)
    o = _outs(G, 32, G)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.trace_capture_static_ws(P(x), G, 32, G, P(offs), P(o["codes"]), P(o["mbits"]),
                                     P(o["scales"]), P(o["gscale"]), None)
    torch.cuda.synchronize()
    assert st == 4  # TRACE_ERR_WORKSPACE: nothing enqueued
    assert torch.all(o["gscale"] == -7.0)


def test_static_workspace_capture_after_device_reset(tmp_path):
    """cudaDeviceReset unloads the library's module, so the static array may
    come back at another device address; a plain C program (its own process,
    since a reset would also pull the device out from under torch) captures
    without a workspace before and after a reset and compares every output
    with trace_capture given a workspace."""
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "fp4_quantization_aware_trace_b200")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = str(tmp_path / "c_static_ws_reset")
    subprocess.run(["gcc", "-O2", "-std=c11", "-Wall", "-Werror", "-I",
                    os.path.join(root, "include"), "-I", os.path.join(cuda, "include"),
                    os.path.join(root, "tests", "c_static_ws_reset.c"), "-L", pkg, "-ltrace_fp4",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{pkg}:{os.path.join(cuda, 'lib64')}", "-o", exe],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
