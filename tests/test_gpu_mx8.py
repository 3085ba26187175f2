"""Bit-exact parity of the W4A8 kernels (E4M3 activations with MX scales)
with the oracle: capture (E8M0 scales, one-byte codes, mantissa bits) and the
1-bit guided, round-to-nearest and full-information guided forwards with
their STE masks.  The oracle's E4M3 bracket scans all 127 codes per element,
so the large workloads are checked on sampled rows (MX scales are per block:
rows are independent)."""
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


def run_gpu(xr, xt):
    cap = ops.mx8_capture(xr.to(DEV).contiguous())
    xtd = xt.to(DEV).contiguous()
    out, mask = ops.mx8_guided_fq_fwd(xtd, cap)
    out_r, mask_r = ops.mx8_rtn_fq_fwd(xtd, cap.scales)
    out_f, mask_f = ops.mx8_full_guided_fq_fwd(xtd, cap)
    torch.cuda.synchronize()
    return dict(codes=_u(cap.codes), mbits=_u(cap.mbits), scales=_u(cap.scales), out=_u(out),
                mask=_u(mask), out_rtn=_u(out_r), mask_rtn=_u(mask_r), out_full=_u(out_f),
                mask_full=_u(mask_f))


def run_oracle(oracle_mod, xr_b, xt_b):
    codes, mbits, scales = oracle_mod.mx8_capture(xr_b)
    out, mask = oracle_mod.mx8_guided_fwd(xt_b, mbits, scales)
    out_r, mask_r = oracle_mod.mx8_rtn_fwd(xt_b, scales)
    out_f, mask_f = oracle_mod.mx8_full_guided_fwd(xt_b, codes, scales)
    return dict(codes=codes, mbits=mbits, scales=scales, out=out, mask=mask, out_rtn=out_r,
                mask_rtn=mask_r, out_full=out_f, mask_full=mask_f)


def check(oracle_mod, name, xr, xt):
    got = run_gpu(xr, xt)
    ref = run_oracle(oracle_mod, inputs.bits(xr), inputs.bits(xt))
    for k in ref:
        _eq(f"{name}.{k}", got[k], ref[k])
    return got


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 32), (37, 96), (129, 160), (300, 2048)])
def test_mx8_small_shapes(oracle_mod, rows, cols):
    s = inputs.tiny_site(rows * 17 + cols, rows, cols, eps=0.02)
    check(oracle_mod, f"mx8_{rows}x{cols}", s.x_roll, s.x_train)


def test_mx8_special_values(oracle_mod):
    rng = np.random.default_rng(23)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x[0, :32] = 0.0
    x[0, 3] = -0.0
    x[1, :32] = 1e-39 * rng.standard_normal(32)
    x[2, :] *= 1e30
    x[3, 5] = 3.3e38
    x[4, :32] = 2.0 ** -133
    x[5, :] = np.tile([2.0 ** -9, 3 * 2.0 ** -10, 2.0 ** -6, 1.0625, 240.0, 448.0, 464.0, 500.0], 32)
    x[6, :] *= 1e-30
    x[7, :32] = 2.0 ** -119 * rng.uniform(0.5, 1.99, 32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xtv = np.clip(x.astype(np.float64) * rng.uniform(0.9, 1.1, x.shape), -3.3e38,
                  3.3e38).astype(np.float32)
    xtv[8, :] *= 1e20
    xtv[9, :] = -xtv[9, :]
    xt = torch.from_numpy(xtv).to(torch.bfloat16)
    assert torch.isfinite(xt.float()).all()
    check(oracle_mod, "special", xb, xt)
    got = check(oracle_mod, "special_same", xb, xb)
    assert np.array_equal(got["out"], got["out_rtn"])


def _all_finite_bf16():
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    return np.concatenate([p, np.zeros((-p.size) % 256, np.uint16)]).reshape(-1, 256)


def test_mx8_exhaustive_forwards(oracle_mod):
    """Every finite bf16 pattern under scale bytes across the whole accepted
    range (0..246), both cached bits and cycled rollout codes."""
    pats = _all_finite_bf16()
    slab, C = pats.shape
    sbytes = np.array([0, 1, 2, 40, 100, 118, 119, 126, 127, 128, 136, 160, 200, 245, 246], np.uint8)
    x = np.tile(pats, (len(sbytes), 1))
    R = x.shape[0]
    scales = np.repeat(np.repeat(sbytes, slab), C // 32).reshape(R, C // 32)
    idx = np.arange(R * C, dtype=np.int64)
    mbits = ((idx[: R * C // 32] * 2654435761) & 0xFFFFFFFF).astype(np.uint32)
    rcodes = ((idx * 37 + idx // (slab * C)) % 255).astype(np.uint8)
    rcodes[(rcodes & 0x7F) == 0x7F] = 0x00               # no NaN encodings
    xd = inputs.from_bits(x, DEV)
    cache = ops.MxCapture(codes=torch.from_numpy(rcodes).to(DEV),
                          mbits=torch.from_numpy(mbits.view(np.int32)).to(DEV),
                          scales=torch.from_numpy(scales).to(DEV))
    out, mask = ops.mx8_guided_fq_fwd(xd, cache)
    out_r, mask_r = ops.mx8_rtn_fq_fwd(xd, cache.scales)
    out_f, mask_f = ops.mx8_full_guided_fq_fwd(xd, cache)
    torch.cuda.synchronize()
    ro, rm = oracle_mod.mx8_guided_fwd(x, mbits, scales)
    _eq("guided_out", _u(out), ro)
    _eq("guided_mask", _u(mask), rm)
    rr, rrm = oracle_mod.mx8_rtn_fwd(x, scales)
    _eq("rtn_out", _u(out_r), rr)
    _eq("rtn_mask", _u(mask_r), rrm)
    rf, rfm = oracle_mod.mx8_full_guided_fwd(x, rcodes, scales)
    _eq("full_out", _u(out_f), rf)
    _eq("full_mask", _u(mask_f), rfm)


def test_mx8_exhaustive_capture(oracle_mod):
    pats = _all_finite_bf16()
    p = np.arange(1, 0x7F80, dtype=np.uint16)
    blocks = np.zeros((p.size, 32), np.uint16)
    blocks[:, 0] = p
    blocks[:, 1:17] = (p[:, None] >> 1) & 0x7FFF
    blocks[:, 17:] = ((p[:, None] - 1) | 0x8000)
    blocks = np.concatenate([blocks, np.zeros((((-blocks.size) % 256) // 32, 32), np.uint16)])
    x = np.concatenate([pats, blocks.reshape(-1, 256)])
    xb = inputs.from_bits(x)
    got = run_gpu(xb, xb)
    codes, mbits, scales = oracle_mod.mx8_capture(x)
    _eq("codes", got["codes"], codes)
    _eq("mbits", got["mbits"], mbits)
    _eq("scales", got["scales"], scales)


@pytest.mark.parametrize("which", ["attn_in", "layer_sweep"])
def test_mx8_workloads_sampled_rows(oracle_mod, which):
    s = (inputs.attention_input(device=DEV) if which == "attn_in"
         else inputs.layer_sweep_site(20, 3, device=DEV))
    got = run_gpu(s.x_roll, s.x_train)
    R, C = s.x_roll.shape
    rows = np.unique(np.concatenate([[0, R - 1], np.random.default_rng(5).integers(0, R, 48)]))
    ref = run_oracle(oracle_mod, inputs.bits(s.x_roll)[rows], inputs.bits(s.x_train)[rows])
    per_row = dict(codes=C, mbits=C // 32, scales=C // 32, out=C, mask=C // 32, out_rtn=C,
                   mask_rtn=C // 32, out_full=C, mask_full=C // 32)
    for k, w in per_row.items():
        _eq(f"{which}.{k}", got[k].reshape(R, w)[rows], ref[k])


def test_mx8_argument_errors():
    lib = ops.library()
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    cap = ops.mx8_capture(x)
    out = torch.empty_like(x)
    mask = torch.zeros(8, dtype=torch.int32, device=DEV)
    P = lambda t: t.data_ptr()
    assert lib.trace_mx8_capture(P(x), 4, 48, P(cap.codes), P(cap.mbits), P(cap.scales), None) == 2
    assert lib.trace_mx8_capture(P(x), 4, 64, P(cap.codes) + 16, P(cap.mbits), P(cap.scales),
                                 None) == 3
    assert lib.trace_mx8_guided_fq_fwd(P(x), 4, 64, None, P(cap.scales), P(out), P(mask), None) == 1
    assert lib.trace_mx8_full_guided_fq_fwd(P(x), 4, 64, P(cap.codes) + 8, P(cap.scales), P(out),
                                            P(mask), None) == 3
    torch.cuda.synchronize()
    assert int(mask.abs().sum()) == 0
