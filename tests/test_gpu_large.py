"""A tensor past 2^31 elements ([1048704, 2048] bf16, 4.3 GB per activation):
64-bit addressing in every kernel.  The global amax is fixed by construction
(one planted +-1000, everything else clamped below it), so the oracle's
global scale needs no scan of the tensor; sampled rows -- several past
element 2^31 -- are checked bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import ops

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROWS, COLS = (1 << 20) + 128, 2048


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def test_past_2_to_the_31_elements(oracle_mod):
    assert ROWS * COLS > 2 ** 31
    g = torch.Generator(device=DEV)
    g.manual_seed(4242)
    xr = torch.randn(ROWS, COLS, generator=g, device=DEV).mul_(8.0).clamp_(-999.0, 999.0)
    xr[ROWS - 3, 17] = -1000.0                     # the global maximum magnitude
    noise = torch.randn(ROWS, COLS, generator=g, device=DEV)
    xt = (xr * (1.0 + 0.005 * noise)).to(torch.bfloat16)
    del noise
    xr = xr.to(torch.bfloat16)
    grad = torch.randn(ROWS, COLS, generator=g, device=DEV).to(torch.bfloat16)
    cap = ops.capture(xr)
    out, mask = ops.guided_fq_fwd(xt, cap)
    gin = ops.fq_bwd(grad, mask)
    torch.cuda.synchronize()
    gs = np.array([oracle_mod.global_scale(1000.0)], np.float32)
    assert cap.gscale.cpu().numpy().view(np.uint32)[0] == gs.view(np.uint32)[0]
    first_past = (2 ** 31) // COLS                  # first row past element 2^31
    rows = np.array([0, 1, 77, first_past - 1, first_past, first_past + 5, ROWS - 3, ROWS - 1])
    rows = np.unique(np.concatenate([rows, np.random.default_rng(1).integers(0, ROWS, 24)]))
    idx = torch.from_numpy(rows).to(DEV)
    xr_s, xt_s, g_s = _bits(xr[idx]), _bits(xt[idx]), _bits(grad[idx])
    rg = np.full(rows.size, gs[0], np.float32)
    codes, mbits, scales = oracle_mod.capture_rows(xr_s, rg)
    o, m = oracle_mod.fake_quant_rows(xt_s, rg, scales, mbits)
    gi = oracle_mod.fq_bwd(g_s, m)
    got_codes = cap.codes.view(ROWS, COLS // 2)[idx].cpu().numpy()
    got_mbits = cap.mbits.view(ROWS, COLS // 32)[idx].cpu().numpy().view(np.uint32)
    got_scales = cap.scales[idx].cpu().numpy()
    assert np.array_equal(got_codes, codes.reshape(rows.size, -1))
    assert np.array_equal(got_mbits, mbits.reshape(rows.size, -1))
    assert np.array_equal(got_scales, scales.reshape(rows.size, -1))
    assert np.array_equal(_bits(out[idx]), o.reshape(rows.size, -1))
    assert np.array_equal(mask.view(ROWS, COLS // 32)[idx].cpu().numpy().view(np.uint32),
                          m.reshape(rows.size, -1))
    assert np.array_equal(_bits(gin[idx]), gi.reshape(rows.size, -1))
