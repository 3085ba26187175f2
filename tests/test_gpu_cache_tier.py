"""The cache tier on the GPU: records written by the rollout side reach
pinned host memory intact (bit-exact against the oracle's capture), come
back to the device, and drive the guided forward to the oracle's output;
ring slots are not reused before their copy has finished."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import cache_tier, inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _host_parts(lay, rec):
    r = rec.numpy()
    n = lay.rows * lay.cols
    return (r[lay.mbits_offset:lay.mbits_offset + n // 8].view(np.uint32),
            r[lay.scales_offset:lay.scales_offset + n // 16],
            r[lay.gscale_offset:lay.gscale_offset + 4 * lay.num_groups].view(np.float32))


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_roundtrip_bit_exact(oracle_mod):
    tier = cache_tier.CacheTier(num_layers=4, keep=2, ring=2)
    sites = {layer: inputs.tiny_site(100 + layer, 200 + 32 * layer, 256, eps=0.01) for layer in range(4)}
    stream = torch.cuda.Stream()
    caps = {}
    with torch.cuda.stream(stream):
        for layer, s in sites.items():
            caps[layer] = tier.capture(("b0", layer), layer, s.x_roll.to(DEV))
    assert not tier.has(("b0", 0)) and not tier.has(("b0", 1))
    assert tier.has(("b0", 2)) and tier.has(("b0", 3))
    for layer in (2, 3):
        s = sites[layer]
        xr, xt = inputs.bits(s.x_roll), inputs.bits(s.x_train)
        codes, mbits, scales, gscale = oracle_mod.capture(xr)
        lay = cache_tier.RecordLayout.of(*xr.shape)
        hm, hs, hg = _host_parts(lay, tier.host_record(("b0", layer)))
        assert np.array_equal(hm, mbits) and np.array_equal(hs, scales.reshape(-1))
        assert np.array_equal(hg.view(np.uint32), gscale.view(np.uint32))
        # trainer side: fetch on another stream, guided forward
        train = torch.cuda.Stream()
        with torch.cuda.stream(train):
            cache = tier.fetch(("b0", layer))
            out, mask = ops.guided_fq_fwd(s.x_train.to(DEV), cache)
        train.synchronize()
        ro, rm = oracle_mod.guided_fwd(xt, mbits, scales, gscale)
        assert np.array_equal(_bits(out).reshape(-1), ro.reshape(-1))
        assert np.array_equal(mask.cpu().numpy().view(np.uint32), rm)
    # not-kept layers still return a full capture (codes for the rollout's GEMM)
    torch.cuda.synchronize()
    c0, *_ = oracle_mod.capture(inputs.bits(sites[0].x_roll))
    assert np.array_equal(caps[0].codes.cpu().numpy(), c0)


def test_ring_reuse_waits_for_copies(oracle_mod):
    """Many captures of one shape through a 2-slot ring with no host sync in
    between: every host record must hold its own site."""
    tier = cache_tier.CacheTier(num_layers=2, keep=1, ring=2)
    sites = [inputs.tiny_site(300 + i, 2048, 512, eps=0.01) for i in range(7)]
    xs = [s.x_roll.to(DEV) for s in sites]
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        tier.capture(("step", i), 1, x)
    tier.synchronize()
    assert tier.d2h_bytes == 7 * cache_tier.RecordLayout.of(2048, 512).nbytes
    for i, s in enumerate(sites):
        _, mbits, scales, gscale = oracle_mod.capture(inputs.bits(s.x_roll))
        lay = cache_tier.RecordLayout.of(2048, 512)
        hm, hs, hg = _host_parts(lay, tier.host_record(("step", i)))
        assert np.array_equal(hm, mbits), i
        assert np.array_equal(hs, scales.reshape(-1)), i


def test_grouped_site_and_recapture(oracle_mod):
    s = inputs.tiny_site(7, 300, 128, eps=0.01)
    offs = torch.tensor([0, 10, 10, 170, 300], dtype=torch.int64)
    tier = cache_tier.CacheTier(num_layers=1, keep=1)
    tier.capture("k", 0, s.x_roll.to(DEV), offs.to(DEV))
    # the same key again overwrites its host record in place
    x2 = (s.x_roll.float() * 3).to(torch.bfloat16)
    tier.capture("k", 0, x2.to(DEV), offs.to(DEV))
    cache = tier.fetch("k")
    out, mask = ops.guided_fq_fwd(s.x_train.to(DEV), cache)
    torch.cuda.synchronize()
    xb, xt = inputs.bits(x2), inputs.bits(s.x_train)
    codes, mbits, scales, gscale = oracle_mod.capture(xb, 4, offs.numpy())
    ro, rm = oracle_mod.guided_fwd(xt, mbits, scales, gscale, 4, offs.numpy())
    assert np.array_equal(_bits(out).reshape(-1), ro.reshape(-1))
    assert tier.host_nbytes() == cache_tier.RecordLayout.of(300, 128, 4).nbytes
