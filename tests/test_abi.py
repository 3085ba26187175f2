"""The C-ABI library loads without a GPU, exports every function that
include/*.h declares, and rejects bad arguments on the host before touching
CUDA (no compute call is made here)."""
from __future__ import annotations

import ctypes
import glob
import os
import re
import subprocess

import pytest

from fp4_quantization_aware_trace_b200 import _build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return ops.library()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(trace_\w+)\s*\(", src, re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_abi():
    names = _declared()
    for n in ("trace_capture", "trace_guided_fq_fwd", "trace_fq_bwd", "trace_rtn_fq_fwd",
              "trace_capture_workspace_bytes", "trace_strerror", "trace_abi_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    missing = _declared() - exported
    assert not missing, missing
    for n in _declared():
        assert hasattr(lib, n)


def test_version_and_strings(lib):
    assert lib.trace_abi_version() == 2
    for st in range(7):
        assert lib.trace_strerror(st)
    assert b"unknown" in lib.trace_strerror(99)


def test_workspace_query(lib):
    # four words of barrier state and G accumulators, 4 bytes each, in
    # 256-byte units
    assert ops.trace_capture_workspace_bytes(16, 32, 1) == 256
    assert ops.trace_capture_workspace_bytes(16, 32, 60) == 256
    assert ops.trace_capture_workspace_bytes(16, 32, 61) == 512
    assert ops.trace_capture_workspace_bytes(16, 32, 4096) == 16640
    assert ops.trace_capture_workspace_bytes(16, 33, 1) == 0
    assert ops.trace_capture_workspace_bytes(16, 32, 0) == 0


def test_host_argument_checks(lib):
    P = ctypes.c_void_p
    a = P(1 << 20)          # aligned fake pointers: never dereferenced
    odd = P((1 << 20) + 2)
    # shape errors come first
    assert lib.trace_capture(a, 4, 48, 1, None, a, a, a, a, a, 256, None) == 2
    assert lib.trace_capture(a, -1, 32, 1, None, a, a, a, a, a, 256, None) == 2
    assert lib.trace_capture(a, 4, 32, 0, None, a, a, a, a, a, 256, None) == 2
    assert lib.trace_capture(a, 1 << 33, 32, 1, None, a, a, a, a, a, 256, None) == 2
    # NULLs
    assert lib.trace_capture(None, 4, 32, 1, None, a, a, a, a, a, 256, None) == 1
    assert lib.trace_capture(a, 4, 32, 3, None, a, a, a, a, a, 256, None) == 1
    assert lib.trace_guided_fq_fwd(a, 4, 32, 1, None, None, a, a, a, a, None) == 1
    assert lib.trace_rtn_fq_fwd(a, 4, 32, 1, None, a, a, None, a, None) == 1
    assert lib.trace_fq_bwd(a, None, 32, a, None) == 1
    # alignment
    assert lib.trace_capture(odd, 4, 32, 1, None, a, a, a, a, a, 256, None) == 3
    assert lib.trace_guided_fq_fwd(a, 4, 32, 1, None, a, a, a, odd, a, None) == 3
    assert lib.trace_fq_bwd(a, a, 32, odd, None) == 3
    assert lib.trace_copy_bf16(a, odd, 16, None) == 3
    # workspace
    assert lib.trace_capture(a, 4, 32, 1, None, a, a, a, a, a, 255, None) == 4
    assert lib.trace_capture(a, 4, 32, 65, a, a, a, a, a, a, 256, None) == 4
    # sizes
    assert lib.trace_fq_bwd(a, a, 40, a, None) == 2
    assert lib.trace_copy_bf16(a, a, 12, None) == 2
    # the staged copy yardstick
    assert lib.trace_copy_bf16_staged(a, a, 12, a, None) == 2
    assert lib.trace_copy_bf16_staged(a, a, 16, None, None) == 1
    assert lib.trace_copy_bf16_staged(a, odd, 16, a, None) == 3
    assert lib.trace_copy_bf16_staged(a, a, 16, odd, None) == 3
    assert lib.trace_copy_bf16_staged(a, a, 0, None, None) == 0


def test_binding_rejects_host_tensors(lib):
    import torch
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(ops.TraceError):
        ops.fq_bwd(x, torch.zeros(4, dtype=torch.int32))


def test_scale_bytes_query(lib):
    """Host-only size query of the scale layouts (no GPU needed)."""
    assert lib.trace_scale_bytes(300, 2048, 16, 0) == 300 * 128
    assert lib.trace_scale_bytes(300, 2048, 16, 1) == 3 * 32 * 512
    assert lib.trace_scale_bytes(300, 2048, 32, 1) == 3 * 16 * 512
    assert lib.trace_scale_bytes(1, 32, 16, 1) == 512
    assert lib.trace_scale_bytes(1, 32, 32, 0) == 1
    for bad in [(4, 48, 16, 0), (4, 64, 8, 0), (4, 64, 16, 2), (-1, 64, 16, 0)]:
        assert lib.trace_scale_bytes(*bad) == 0


def test_host_argument_checks_newer_calls(lib):
    """The checks of the calls beyond the core path return before any CUDA
    call (fake, never dereferenced pointers; no GPU needed)."""
    P = ctypes.c_void_p
    a = P(1 << 20)
    odd = P((1 << 20) + 2)
    # full-information guidance
    assert lib.trace_full_guided_fq_fwd(a, 4, 48, 1, None, a, a, a, a, a, None) == 2
    assert lib.trace_full_guided_fq_fwd(a, 4, 32, 1, None, None, a, a, a, a, None) == 1
    assert lib.trace_full_guided_fq_fwd(a, 4, 32, 1, None, odd, a, a, a, a, None) == 3
    # MXFP4 / W4A8
    for cap in (lib.trace_mx_capture, lib.trace_mx8_capture):
        assert cap(a, 4, 48, a, a, a, None) == 2
        assert cap(None, 4, 32, a, a, a, None) == 1
        assert cap(odd, 4, 32, a, a, a, None) == 3
    assert lib.trace_mx8_capture(a, 4, 32, P((1 << 20) + 16), a, a, None) == 3   # codes: 32 B
    for fwd in (lib.trace_mx_guided_fq_fwd, lib.trace_mx8_guided_fq_fwd):
        assert fwd(a, 4, 32, None, a, a, a, None) == 1
        assert fwd(a, 4, 32, a, a, odd, a, None) == 3
    assert lib.trace_mx_rtn_fq_fwd(a, 4, 32, a, a, None, None) == 1
    assert lib.trace_mx8_rtn_fq_fwd(a, -1, 32, a, a, a, None) == 2
    # tiled layout: unknown layout / rule
    assert lib.trace_capture_ex(a, 4, 32, 1, None, a, a, a, a, a, 256, 7, None) == 2
    assert lib.trace_fq_fwd_ex(5, a, 4, 32, 1, None, a, a, a, a, a, a, 0, None) == 2
    assert lib.trace_mx_capture_ex(a, 4, 32, a, a, a, 2, None) == 2
    assert lib.trace_mx8_fq_fwd_ex(0, a, 4, 32, a, a, a, a, a, 3, None) == 2
    # histograms
    assert lib.trace_mismatch_histogram(a, 4, 32, 1, None, a, a, a, None, None) == 1
    assert lib.trace_mismatch_histogram(a, 4, 32, 1, None, a, a, a, P((1 << 20) + 4), None) == 3
    assert lib.trace_mx_mismatch_histogram(a, 4, 32, a, a, None, None) == 1
    assert lib.trace_mx_mismatch_histogram(a, 4, 40, a, a, a, None) == 2
    # capture's two passes
    assert lib.trace_capture_amax(a, 4, 48, 1, None, a, None) == 2
    assert lib.trace_capture_amax(a, 4, 32, 1, None, None, None) == 1
    assert lib.trace_capture_amax_accumulate(a, 4, 32, 1, None, odd, None) == 3
    assert lib.trace_capture_with_amax(a, 4, 32, 1, None, a, a, a, a, a, 9, None) == 2
    assert lib.trace_capture_with_amax(a, 4, 32, 1, None, None, a, a, a, a, 0, None) == 1
    # capture status: NULL / misaligned workspace
    assert lib.trace_capture_status(None, None) == 1
    assert lib.trace_capture_status(P((1 << 20) + 2), None) == 3
    # no-workspace capture: too many groups
    assert lib.trace_capture_static_ws(a, 4, 32, 4097, a, a, a, a, a, None) == 4
    # self-test range: must stay below +inf
    assert lib.trace_selftest_e4m3_sweep(0x7F800000, 1, a, None) == 2
    assert lib.trace_selftest_e4m3_sweep(0, 0, None, None) == 0


def test_validate_offsets_argument_checks(lib):
    P = ctypes.c_void_p
    a = P(1 << 20)
    assert lib.trace_validate_offsets(a, 0, 4, a, None) == 2
    assert lib.trace_validate_offsets(None, 2, 4, a, None) == 1
    assert lib.trace_validate_offsets(P((1 << 20) + 4), 2, 4, a, None) == 3


def test_host_argument_checks_check_calls(lib):
    """The self-test, the offset check and capture without a workspace reject
    bad arguments before any CUDA call (fake, never dereferenced pointers)."""
    P = ctypes.c_void_p
    a = P(1 << 20)
    odd = P((1 << 20) + 2)
    # E4M3 self-test: nothing to do, no output, inputs not below +inf
    assert lib.trace_selftest_e4m3_sweep(0x3F800000, 0, None, None) == 0
    assert lib.trace_selftest_e4m3_sweep(0x3F800000, 16, None, None) == 1
    assert lib.trace_selftest_e4m3_sweep(0x7F800000, 1, a, None) == 2
    assert lib.trace_selftest_e4m3_sweep(0x7F7FFFFF, 2, a, None) == 2
    # offset check: groups, rows, pointers, alignment
    assert lib.trace_validate_offsets(a, 0, 16, a, None) == 2
    assert lib.trace_validate_offsets(a, 1, -1, a, None) == 2
    assert lib.trace_validate_offsets(None, 2, 16, a, None) == 1
    assert lib.trace_validate_offsets(a, 2, 16, None, None) == 1
    assert lib.trace_validate_offsets(P((1 << 20) + 4), 2, 16, a, None) == 3
    assert lib.trace_validate_offsets(a, 2, 16, odd, None) == 3
    # capture without a workspace: more groups than its static scratch holds
    assert lib.trace_capture_static_ws(a, 4, 32, 4097, a, a, a, a, a, None) == 4
