"""The device's E4M3 block-scale rounding against the oracle on every
positive finite fp32 (2^31 - 2^23 values): round to nearest even, the
subnormal range, the 2^-10 -> 0 tie, and saturation at 448 (the band
448 < t < 464 rounds to 448 and everything above saturates)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import ops

pytestmark = pytest.mark.gpu


def test_e4m3_rounding_every_positive_fp32(oracle_mod):
    end = 0x7F800000
    chunk = 1 << 27
    buf = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for first in range(0, end, chunk):
        n = min(chunk, end - first)
        ops.trace_selftest_e4m3_sweep(first, n, buf[:n])
        got = buf[:n].cpu().numpy()
        ref = oracle_mod.e4m3_sweep(first, n)
        bad = np.flatnonzero(got != ref)
        assert bad.size == 0, (f"{bad.size} mismatches from 0x{first:08x}, first at bit pattern "
                               f"0x{first + int(bad[0]):08x}: got {got[bad[0]]} ref {ref[bad[0]]}")


def test_e4m3_sweep_argument_checks():
    out = torch.empty(16, dtype=torch.uint8, device="cuda")
    lib = ops.library()
    assert lib.trace_selftest_e4m3_sweep(0x7F7FFFFF, 2, out.data_ptr(), None) == 2
    assert lib.trace_selftest_e4m3_sweep(0, 4, None, None) == 1
    assert lib.trace_selftest_e4m3_sweep(0, 0, None, None) == 0
