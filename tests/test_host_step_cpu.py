"""Host-side logic of the host-to-host step (no GPU): the row chunks cover
every row once, in order, and every chunk start keeps the byte alignment of
each array's slice (x and outputs 32 B, codes 16 B, mantissa bits and masks
16 B, row-major scales 16 B)."""
from __future__ import annotations

import pytest

from fp4_quantization_aware_trace_b200.host_step import row_chunks


@pytest.mark.parametrize("rows", [0, 1, 7, 8, 31, 64, 100, 1000, 16384, 16389])
@pytest.mark.parametrize("cols", [32, 64, 96, 128, 160, 640, 2048, 4096])
@pytest.mark.parametrize("chunks", [1, 2, 3, 8, 1000])
def test_row_chunks_cover_and_align(rows, cols, chunks):
    cuts = row_chunks(rows, cols, chunks)
    # cover 0..rows exactly once, in order, no empty chunk
    pos = 0
    for a, b in cuts:
        assert a == pos and b > a
        pos = b
    assert pos == rows
    # equal chunks (a multiple of the row quantum) and a shorter tail
    lens = [b - a for a, b in cuts]
    if len(lens) > 1:
        assert len(set(lens[:-1])) == 1 and lens[-1] <= lens[0]
    for a, _ in cuts:
        n = a * cols  # elements before the chunk
        assert (2 * n) % 32 == 0        # bf16 x / outputs
        assert (n // 2) % 16 == 0       # codes, two per byte
        assert (n // 8) % 16 == 0       # mantissa bits / mask words
        assert (n // 16) % 16 == 0      # row-major scales, one byte per block


def test_row_chunks_counts():
    assert row_chunks(0, 2048, 8) == []
    assert row_chunks(16384, 2048, 8) == [(i * 2048, (i + 1) * 2048) for i in range(8)]
    # fewer rows than the quantum: one chunk
    assert row_chunks(5, 32, 8) == [(0, 5)]
