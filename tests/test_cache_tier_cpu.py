"""Host logic of the cache tier: which layers are kept and the layout of a
site's compact-cache record (a host function of the C ABI; no GPU needed)."""
from __future__ import annotations

import pytest

from fp4_quantization_aware_trace_b200 import cache_tier, ops


def test_kept_layers_deeper_half():
    # the post's ablation keeps the latter 20 of 40 layers
    assert list(cache_tier.kept_layers(40)) == list(range(20, 40))
    assert list(cache_tier.kept_layers(40, 5)) == list(range(35, 40))
    assert list(cache_tier.kept_layers(7)) == [3, 4, 5, 6]
    assert list(cache_tier.kept_layers(3, 0)) == []
    with pytest.raises(ValueError):
        cache_tier.kept_layers(4, 5)


@pytest.mark.parametrize("rows,cols,G", [(1, 32, 1), (3, 32, 1), (37, 96, 1), (16384, 2048, 1),
                                         (65536, 128, 1), (5, 64, 3), (0, 64, 2)], ids=str)
def test_record_layout(rows, cols, G):
    lay = cache_tier.RecordLayout.of(rows, cols, G)
    n = rows * cols
    segs = [(lay.mbits_offset, n // 8), (lay.scales_offset, n // 16), (lay.gscale_offset, 4 * G)]
    assert all(o % 16 == 0 for o, _ in segs) and lay.nbytes % 16 == 0
    end = 0
    for o, size in segs:           # in order, disjoint, inside the record
        assert o >= end
        end = o + size
    assert end <= lay.nbytes
    # 1.5 bits per element + 4 bytes per group, plus at most 45 bytes padding
    assert 0 <= lay.nbytes - (n // 8 + n // 16 + 4 * G) <= 45


def test_record_layout_rejects_bad_shapes():
    for shape in [(4, 33, 1), (4, 0, 1), (-1, 32, 1), (4, 32, 0), (1 << 31, 1 << 10, 1)]:
        assert ops.trace_cache_record_bytes(*shape)[0] == 0
        with pytest.raises(ops.TraceError):
            cache_tier.RecordLayout.of(*shape)


def test_compression_against_full_codes():
    """Compact records on the deeper half vs full FP4 records (codes + scales)
    on every layer: about 6x fewer bytes (compact-cache paragraph)."""
    rows, cols, layers = 65536, 4096, 40
    n = rows * cols
    compact = cache_tier.RecordLayout.of(rows, cols).nbytes * len(cache_tier.kept_layers(layers))
    full = (n // 2 + n // 16 + 4) * layers
    assert abs(full / compact - 6.0) < 1e-3
