"""Bit-exact parity of the MXFP4 kernels (through the C ABI) with the
oracle: capture (E8M0 scales, codes, mantissa bits) and the 1-bit guided,
round-to-nearest and full-information guided forwards with their STE masks.
"""
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
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def _eq(name, got, ref):
    got, ref = np.asarray(got).reshape(-1), np.asarray(ref).reshape(-1)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, (f"{name}: {bad.size} mismatches, first at {bad[:8].tolist()}: "
                           f"got {got[bad[:8]].tolist()} ref {ref[bad[:8]].tolist()}")


def run_gpu(xr, xt, g=None):
    cap = ops.mx_capture(xr.to(DEV).contiguous())
    xtd = xt.to(DEV).contiguous()
    out, mask = ops.mx_guided_fq_fwd(xtd, cap)
    out_r, mask_r = ops.mx_rtn_fq_fwd(xtd, cap.scales)
    out_f, mask_f = ops.mx_full_guided_fq_fwd(xtd, cap)
    res = dict(codes=_u(cap.codes), mbits=_u(cap.mbits), scales=_u(cap.scales), out=_u(out),
               mask=_u(mask), out_rtn=_u(out_r), mask_rtn=_u(mask_r), out_full=_u(out_f),
               mask_full=_u(mask_f))
    if g is not None:
        res["grad_in"] = _u(ops.fq_bwd(g.to(DEV).contiguous(), mask))
    torch.cuda.synchronize()
    return res


def run_oracle(oracle_mod, xr, xt, g=None):
    xr, xt = inputs.bits(xr), inputs.bits(xt)
    codes, mbits, scales = oracle_mod.mx_capture(xr)
    out, mask = oracle_mod.mx_guided_fwd(xt, mbits, scales)
    out_r, mask_r = oracle_mod.mx_rtn_fwd(xt, scales)
    out_f, mask_f = oracle_mod.mx_full_guided_fwd(xt, codes, scales)
    res = dict(codes=codes, mbits=mbits, scales=scales, out=out, mask=mask, out_rtn=out_r,
               mask_rtn=mask_r, out_full=out_f, mask_full=mask_f)
    if g is not None:
        res["grad_in"] = oracle_mod.fq_bwd(inputs.bits(g), mask)
    return res


def check(oracle_mod, name, xr, xt, g=None):
    got, ref = run_gpu(xr, xt, g), run_oracle(oracle_mod, xr, xt, g)
    for k in ref:
        _eq(f"{name}.{k}", got[k], ref[k])
    return got


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 32), (37, 96), (129, 160), (513, 2048),
                                       (4099, 128)])
def test_mx_small_shapes(oracle_mod, rows, cols):
    s = inputs.tiny_site(rows * 13 + cols, rows, cols, eps=0.02)
    check(oracle_mod, f"mx{rows}x{cols}", s.x_roll, s.x_train, s.grad)


def test_mx_special_values(oracle_mod):
    rng = np.random.default_rng(19)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x[0, :32] = 0.0
    x[0, 3] = -0.0
    x[1, :32] = 1e-39 * rng.standard_normal(32)       # subnormal block (scale clamps)
    x[2, :] *= 1e30
    x[3, 5] = 3.3e38
    x[4, :32] = 2.0 ** -133
    x[5, :] = np.tile([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], 32)
    x[6, :] *= 1e-30
    x[7, :32] = 2.0 ** -125 * rng.uniform(0.5, 1.99, 32)   # around the clamp edge
    xb = torch.from_numpy(x).to(torch.bfloat16)
    # finite inputs only (a precondition of both sides): stay below 3.3e38
    xtv = np.clip(x.astype(np.float64) * rng.uniform(0.9, 1.1, x.shape), -3.3e38,
                  3.3e38).astype(np.float32)
    xtv[8, :] *= 1e20                                           # far past the rollout's range
    xt = torch.from_numpy(xtv).to(torch.bfloat16)
    assert torch.isfinite(xt.float()).all()
    check(oracle_mod, "special", xb, xt)
    check(oracle_mod, "special_same", xb, xb)


def _all_finite_bf16():
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    return np.concatenate([p, np.zeros((-p.size) % 256, np.uint16)]).reshape(-1, 256)


def test_mx_exhaustive_forwards(oracle_mod):
    """Every finite bf16 pattern under every E8M0 scale byte the forwards
    accept (0..252: capture's range), with both cached bits and cycled
    rollout codes."""
    pats = _all_finite_bf16()
    slab, C = pats.shape
    sbytes = np.arange(253, dtype=np.uint8)
    x = np.tile(pats, (len(sbytes), 1))
    R = x.shape[0]
    scales = np.repeat(np.repeat(sbytes, slab), C // 32).reshape(R, C // 32)
    idx = np.arange(R * C, dtype=np.int64)
    mbits = ((idx // 32 * 2654435761) & 0xFFFFFFFF).astype(np.uint32)[: R * C // 32]
    nib = ((idx + idx // (slab * C)) % 16).astype(np.uint8)
    rcodes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    xd = inputs.from_bits(x, DEV)
    cache = ops.MxCapture(codes=torch.from_numpy(rcodes).to(DEV),
                          mbits=torch.from_numpy(mbits.view(np.int32)).to(DEV),
                          scales=torch.from_numpy(scales).to(DEV))
    out, mask = ops.mx_guided_fq_fwd(xd, cache)
    out_r, mask_r = ops.mx_rtn_fq_fwd(xd, cache.scales)
    out_f, mask_f = ops.mx_full_guided_fq_fwd(xd, cache)
    torch.cuda.synchronize()
    ro, rm = oracle_mod.mx_guided_fwd(x, mbits, scales)
    _eq("guided_out", _u(out), ro)
    _eq("guided_mask", _u(mask), rm)
    rr, rrm = oracle_mod.mx_rtn_fwd(x, scales)
    _eq("rtn_out", _u(out_r), rr)
    _eq("rtn_mask", _u(mask_r), rrm)
    rf, rfm = oracle_mod.mx_full_guided_fwd(x, rcodes, scales)
    _eq("full_out", _u(out_f), rf)
    _eq("full_mask", _u(mask_f), rfm)


def test_mx_exhaustive_capture(oracle_mod):
    """All finite bf16 patterns through capture, and each positive pattern as
    the maximum of its own 32-element block next to smaller values."""
    pats = _all_finite_bf16()
    p = np.arange(1, 0x7F80, dtype=np.uint16)
    blocks = np.zeros((p.size, 32), np.uint16)
    blocks[:, 0] = p
    blocks[:, 1:17] = (p[:, None] >> 1) & 0x7FFF
    blocks[:, 17:] = ((p[:, None] - 1) | 0x8000)
    blocks = np.concatenate([blocks, np.zeros((((-blocks.size) % 256) // 32, 32), np.uint16)])
    x = np.concatenate([pats, blocks.reshape(-1, 256)])
    xb = inputs.from_bits(x)
    check(oracle_mod, "capture_sweep", xb, xb)


def test_mx_cfg2_full(oracle_mod):
    s = inputs.attention_input(device=DEV)
    check(oracle_mod, "attn_in", s.x_roll, s.x_train, s.grad)


@pytest.mark.parametrize("layer,site", [(20, 1), (39, 2)])
def test_mx_cfg5_sampled_rows(oracle_mod, layer, site):
    """MX scales are per block, so sampled rows are checked on their own."""
    s = inputs.layer_sweep_site(layer, site, device=DEV)
    got = run_gpu(s.x_roll, s.x_train)
    R, C = s.x_roll.shape
    rng = np.random.default_rng(layer)
    rows = np.unique(np.concatenate([[0, R - 1], rng.integers(0, R, 64)]))
    xr, xt = inputs.bits(s.x_roll)[rows], inputs.bits(s.x_train)[rows]
    codes, mbits, scales = oracle_mod.mx_capture(xr)
    out, mask = oracle_mod.mx_guided_fwd(xt, mbits, scales)
    out_r, _ = oracle_mod.mx_rtn_fwd(xt, scales)
    out_f, _ = oracle_mod.mx_full_guided_fwd(xt, codes, scales)
    _eq("codes", got["codes"].reshape(R, C // 2)[rows], codes)
    _eq("mbits", got["mbits"].reshape(R, C // 32)[rows], mbits)
    _eq("scales", got["scales"].reshape(R, C // 32)[rows], scales)
    _eq("out", got["out"].reshape(R, C)[rows], out)
    _eq("mask", got["mask"].reshape(R, C // 32)[rows], mask)
    _eq("out_rtn", got["out_rtn"].reshape(R, C)[rows], out_r)
    _eq("out_full", got["out_full"].reshape(R, C)[rows], out_f)


def test_mx_argument_errors():
    lib = ops.library()
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    cap = ops.mx_capture(x)
    out = torch.empty_like(x)
    mask = torch.zeros(8, dtype=torch.int32, device=DEV)
    P = lambda t: t.data_ptr()
    assert lib.trace_mx_capture(P(x), 4, 48, P(cap.codes), P(cap.mbits), P(cap.scales), None) == 2
    assert lib.trace_mx_capture(P(x) + 2, 4, 64, P(cap.codes), P(cap.mbits), P(cap.scales), None) == 3
    assert lib.trace_mx_guided_fq_fwd(P(x), 4, 64, None, P(cap.scales), P(out), P(mask), None) == 1
    assert lib.trace_mx_rtn_fq_fwd(P(x), 4, 64, P(cap.scales), P(out) + 16, P(mask), None) == 3
    assert lib.trace_mx_full_guided_fq_fwd(P(x), -1, 64, P(cap.codes), P(cap.scales), P(out),
                                           P(mask), None) == 2
    torch.cuda.synchronize()
    assert int(mask.abs().sum()) == 0
