"""Seeded random cases through every kernel family, bit-exact against the
oracle: random shapes (cols any multiple of 32), ragged groups including
empty ones, values from 1e-30 to 1e30 with zeros, outliers and signs mixed,
and drifted or independent training sides."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _u(t):
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32).reshape(-1)
    if t.dtype == torch.float32:
        return t.numpy().view(np.uint32).reshape(-1)
    return t.numpy().reshape(-1)


def _case(seed):
    rng = np.random.default_rng(seed)
    rows = int(rng.integers(1, 700))
    cols = 32 * int(rng.integers(1, 40))
    scale = 10.0 ** rng.uniform(-30, 30)
    x = rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((1, cols)) * rng.uniform(0, 2))
    x *= scale
    x[rng.random((rows, cols)) < 0.02] = 0.0
    x[rng.random((rows, cols)) < 0.001] *= 1e3
    if rng.random() < 0.3:
        x[: max(1, rows // 7)] *= 1e-12
    x = np.clip(x, -3e38, 3e38).astype(np.float32)
    if rng.random() < 0.25:
        xt = np.clip(rng.standard_normal((rows, cols)) * scale, -3e38, 3e38).astype(np.float32)
    else:
        xt = np.clip(x.astype(np.float64) * (1 + rng.uniform(0.001, 0.05) * rng.standard_normal((rows, cols))),
                     -3e38, 3e38).astype(np.float32)
    g = rng.standard_normal((rows, cols)).astype(np.float32)
    G = int(rng.integers(1, 6))
    offs = None
    if G > 1:
        cuts = np.sort(rng.integers(0, rows + 1, G - 1))
        offs = np.concatenate([[0], cuts, [rows]]).astype(np.int64)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    return bf(x), bf(xt), bf(g), G, offs


@pytest.mark.parametrize("seed", range(24))
def test_fuzz_nvfp4(oracle_mod, seed):
    xr, xt, g, G, offs = _case(seed)
    od = None if offs is None else torch.from_numpy(offs).to(DEV)
    cap = ops.capture(xr.to(DEV), od)
    xtd = xt.to(DEV)
    out, mask = ops.guided_fq_fwd(xtd, cap)
    out_f, mask_f = ops.full_guided_fq_fwd(xtd, cap)
    out_r, mask_r = ops.rtn_fq_fwd(xtd, cap.scales, cap.gscale, od)
    gin = ops.fq_bwd(g.to(DEV), mask)
    hist = ops.mismatch_histogram(xtd, cap)
    torch.cuda.synchronize()
    xb, tb, gb = inputs.bits(xr), inputs.bits(xt), inputs.bits(g)
    codes, mbits, scales, gscale = oracle_mod.capture(xb, G, offs)
    ro, rm = oracle_mod.guided_fwd(tb, mbits, scales, gscale, G, offs)
    rf, rfm = oracle_mod.full_guided_fwd(tb, codes, scales, gscale, G, offs)
    rr, rrm = oracle_mod.rtn_fwd(tb, scales, gscale, G, offs)
    rg = oracle_mod.fq_bwd(gb, rm)
    rh = oracle_mod.mismatch_histogram(tb, codes, scales, gscale, G, offs)
    for name, got, ref in [("codes", cap.codes, codes), ("mbits", cap.mbits, mbits),
                           ("scales", cap.scales, scales), ("gscale", cap.gscale, gscale.view(np.uint32)),
                           ("out", out, ro), ("mask", mask, rm), ("out_full", out_f, rf),
                           ("mask_full", mask_f, rfm), ("out_rtn", out_r, rr), ("mask_rtn", mask_r, rrm),
                           ("grad_in", gin, rg)]:
        assert np.array_equal(_u(got), np.asarray(ref).reshape(-1)), (seed, name)
    assert np.array_equal(hist.cpu().numpy().view(np.uint64), rh), (seed, "hist")


@pytest.mark.parametrize("seed", range(100, 112))
def test_fuzz_mx_formats(oracle_mod, seed):
    xr, xt, _, _, _ = _case(seed)
    xrd, xtd = xr.to(DEV), xt.to(DEV)
    m4 = ops.mx_capture(xrd)
    o4, k4 = ops.mx_guided_fq_fwd(xtd, m4)
    f4, _ = ops.mx_full_guided_fq_fwd(xtd, m4)
    h4 = ops.mx_mismatch_histogram(xtd, m4)
    m8 = ops.mx8_capture(xrd)
    o8, k8 = ops.mx8_guided_fq_fwd(xtd, m8)
    f8, _ = ops.mx8_full_guided_fq_fwd(xtd, m8)
    r8, _ = ops.mx8_rtn_fq_fwd(xtd, m8.scales)
    torch.cuda.synchronize()
    xb, tb = inputs.bits(xr), inputs.bits(xt)
    c4, b4, s4 = oracle_mod.mx_capture(xb)
    c8, b8, s8 = oracle_mod.mx8_capture(xb)
    refs = [("mx codes", m4.codes, c4), ("mx scales", m4.scales, s4),
            ("mx out", o4, oracle_mod.mx_guided_fwd(tb, b4, s4)[0]),
            ("mx mask", k4, oracle_mod.mx_guided_fwd(tb, b4, s4)[1]),
            ("mx full", f4, oracle_mod.mx_full_guided_fwd(tb, c4, s4)[0]),
            ("w4a8 codes", m8.codes, c8), ("w4a8 mbits", m8.mbits, b8), ("w4a8 scales", m8.scales, s8),
            ("w4a8 out", o8, oracle_mod.mx8_guided_fwd(tb, b8, s8)[0]),
            ("w4a8 mask", k8, oracle_mod.mx8_guided_fwd(tb, b8, s8)[1]),
            ("w4a8 full", f8, oracle_mod.mx8_full_guided_fwd(tb, c8, s8)[0]),
            ("w4a8 rtn", r8, oracle_mod.mx8_rtn_fwd(tb, s8)[0])]
    for name, got, ref in refs:
        assert np.array_equal(_u(got), np.asarray(ref).reshape(-1)), (seed, name)
    assert np.array_equal(h4.cpu().numpy().view(np.uint64),
                          oracle_mod.mx_mismatch_histogram(tb, c4, s4)), (seed, "mx hist")
