"""Parity of the mismatch-distance histogram kernel with the oracle.

The histogram counts, per rule (round to nearest, 1-bit guided, full-
information guided), how many ladder steps the training side's code lies from
the rollout's code (the compact-cache paragraph of the TRACE post: nearly all
disagreements are one adjacent codeword).  Counts are integers, so the bar is
exact equality.  Because a histogram is an aggregate, the exhaustive sweep
and the small cases are launched slice by slice and each slice's counts are
compared on their own, so one wrong site cannot hide behind another.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _offs_np(site):
    return None if site.offsets is None else site.offsets.cpu().numpy()


def _gpu_hist(xt, cap, hist=None):
    h = ops.mismatch_histogram(xt, cap, hist)
    torch.cuda.synchronize()
    return h.cpu().numpy().view(np.uint64)


def _site_on_gpu(site):
    xr = site.x_roll.to(DEV).contiguous()
    xt = site.x_train.to(DEV).contiguous()
    offs = None if site.offsets is None else site.offsets.to(DEV)
    return xt, ops.capture(xr, offs)


def _oracle_site(oracle_mod, site):
    xr, xt = inputs.bits(site.x_roll), inputs.bits(site.x_train)
    G, offs = site.num_groups, _offs_np(site)
    codes, _, scales, gscale = oracle_mod.capture(xr, G, offs)
    return oracle_mod.mismatch_histogram(xt, codes, scales, gscale, G, offs)


def check_site(oracle_mod, site):
    xt, cap = _site_on_gpu(site)
    got = _gpu_hist(xt, cap)
    ref = _oracle_site(oracle_mod, site)
    assert np.array_equal(got, ref), f"{site.name}:\n{got}\nvs\n{ref}"
    n = site.x_roll.numel()
    assert np.all(got.sum(axis=1) == n)
    return got


def _row_slices(xt, cap, r0, r1, g):
    """A Capture view of rows [r0, r1) that lie in group g."""
    C = xt.shape[1]
    return xt[r0:r1], ops.Capture(codes=cap.codes[r0 * C // 2:r1 * C // 2], mbits=None,
                                  scales=cap.scales[r0:r1], gscale=cap.gscale[g:g + 1])


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 32), (37, 96), (129, 160), (513, 2048),
                                       (4099, 128)])
def test_hist_small_shapes(oracle_mod, rows, cols):
    check_site(oracle_mod, inputs.tiny_site(rows * 7 + cols, rows, cols, eps=0.05))


def test_hist_per_row_slices(oracle_mod):
    """Each row launched alone and compared with the oracle on that row."""
    s = inputs.tiny_site(77, 48, 256, eps=0.3)
    xt, cap = _site_on_gpu(s)
    xr_b, xt_b = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    codes, _, scales, gscale = oracle_mod.capture(xr_b)
    C = xt.shape[1]
    for r in range(xt.shape[0]):
        x1, c1 = _row_slices(xt, cap, r, r + 1, 0)
        got = _gpu_hist(x1, c1)
        ref = oracle_mod.mismatch_histogram(xt_b[r:r + 1], codes[r * C // 2:(r + 1) * C // 2],
                                            scales[r:r + 1], gscale)
        assert np.array_equal(got, ref), f"row {r}"


def test_hist_cfg1_and_ragged_groups(oracle_mod):
    check_site(oracle_mod, inputs.single_activation(0))
    s = inputs.tiny_site(5, 777, 96, eps=0.01)
    x = s.x_roll.float()
    x[100:300] *= 1e4
    x[500:520] *= 1e-6
    s.x_roll = x.to(torch.bfloat16)
    s.x_train = (s.x_roll.float() * 1.003).to(torch.bfloat16)
    s.offsets = torch.tensor([0, 0, 1, 100, 300, 300, 301, 520, 777, 777], dtype=torch.int64)
    check_site(oracle_mod, s)


def test_hist_empty_zero_and_special(oracle_mod):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    cap = ops.capture(x)
    h = _gpu_hist(x, cap)
    assert np.all(h == 0)
    z = torch.zeros(64, 64)
    z[::2, 1::3] = -0.0
    zt = z.clone()
    zt[1::2, ::5] = -0.0
    got = check_site(oracle_mod, inputs.Site("zeros", z.to(torch.bfloat16), zt.to(torch.bfloat16),
                                             torch.ones(64, 64).to(torch.bfloat16)))
    assert np.all(got[:, 0] == 64 * 64)
    rng = np.random.default_rng(9)
    xv = rng.standard_normal((64, 256)).astype(np.float32)
    xv[0, :16] = 0.0
    xv[1, :16] = 1e-39 * rng.standard_normal(16)
    xv[2, :] *= 1e30
    xv[3, 5] = 3.3e38
    xv[4, :32] = 2.0 ** -133
    xv[5, :] = np.tile([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], 32)
    xv[6, :] *= 1e-30
    xb = torch.from_numpy(xv).to(torch.bfloat16)
    xt = torch.from_numpy(-xv * rng.uniform(0.5, 1.0, xv.shape).astype(np.float32)).to(torch.bfloat16)
    check_site(oracle_mod, inputs.Site("special", xb, xt, xb))
    check_site(oracle_mod, inputs.Site("special_tiny", (xb.float() * 1e-30).to(torch.bfloat16),
                                       xt, xb))


def test_hist_same_input_is_all_zero_distance(oracle_mod):
    s = inputs.attention_input(seed=4, rows=512)
    s.x_train = s.x_roll.clone()
    got = check_site(oracle_mod, s)
    assert np.all(got[:, 1:] == 0)


def test_hist_exhaustive_sweep(oracle_mod):
    """Every finite bf16 pattern x every signed rollout code x every E4M3 block
    scale x global scales inside and outside the fast range, one launch per
    slab of 255 x 256 elements (one scale byte, one global scale)."""
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    pats = np.concatenate([p, np.zeros((-p.size) % 256, np.uint16)]).reshape(-1, 256)
    gs_vals = np.array([1.0, 0.3712345, 2.0 ** -140, 1.9e30, 2.0 ** 9, 911.0, 3.1e10], np.float32)
    slab, C = pats.shape
    sbytes = np.arange(0x7F, dtype=np.uint8)
    xd = inputs.from_bits(pats, DEV)
    idx = np.arange(slab * C, dtype=np.int64)
    for gi, gv in enumerate(gs_vals):
        hs_gpu, hs_ref = [], []
        for sb in sbytes:
            nib = ((idx + int(sb) + 5 * gi) % 16).astype(np.uint8)
            rcodes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
            scales = np.full((slab, C // 16), sb, np.uint8)
            cache = ops.Capture(codes=torch.from_numpy(rcodes).to(DEV), mbits=None,
                                scales=torch.from_numpy(scales).to(DEV),
                                gscale=torch.tensor([gv], dtype=torch.float32, device=DEV))
            hs_gpu.append(ops.mismatch_histogram(xd, cache))
            hs_ref.append(oracle_mod.mismatch_histogram(pats, rcodes, scales,
                                                        np.array([gv], np.float32)))
        torch.cuda.synchronize()
        for sb, hg, hr in zip(sbytes, hs_gpu, hs_ref):
            assert np.array_equal(hg.cpu().numpy().view(np.uint64), hr), f"gs {gv} scale 0x{sb:02x}"


def test_hist_cfg2_full(oracle_mod):
    got = check_site(oracle_mod, inputs.attention_input(device=DEV))
    # the drifted pairs disagree rarely and by one codeword; the rules that
    # use the rollout agree with it more often than round to nearest
    assert got[0, 1] > 0 and got[0, 2:].sum() < got[0, 1] // 100
    assert got[1, 0] > got[0, 0] and got[2, 0] >= got[1, 0]
    # at 0.5% drift q_roll always lies in the bracket of z_train: leaving it
    # takes a relative move of at least 1/7 (from just under the midpoint
    # 1.75 up to the codeword 2, or 3.5 up to 4), about 29 standard
    # deviations here; full guidance then reproduces every rollout code, and
    # so does the 1-bit cache
    assert got[2, 0] == got[2].sum() and got[1, 0] == got[1].sum()


def test_hist_cfg3_and_cfg4(oracle_mod):
    check_site(oracle_mod, inputs.moe_experts(seed=12, cols=768, device=DEV, name="expert_down_in"))
    for which in ("k", "v"):
        check_site(oracle_mod, inputs.kv_cache(device=DEV, which=which))


@pytest.mark.parametrize("layer,site", [(20, 0), (39, 3)])
def test_hist_cfg5_sampled_and_additive(oracle_mod, layer, site):
    """Full size: the whole-tensor counts sum to N per rule and equal the sum
    of launches over row chunks; sampled rows match the oracle, with the
    global scale the oracle computes over the whole tensor."""
    s = inputs.layer_sweep_site(layer, site, device=DEV)
    xt, cap = _site_on_gpu(s)
    R, C = xt.shape
    whole = _gpu_hist(xt, cap)
    assert np.all(whole.sum(axis=1) == R * C)
    acc = torch.zeros(3, 15, dtype=torch.int64, device=DEV)
    step = 4096
    for r0 in range(0, R, step):
        x1, c1 = _row_slices(xt, cap, r0, min(R, r0 + step), 0)
        ops.mismatch_histogram(x1, c1, acc)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().view(np.uint64), whole)
    xr_b, xt_b = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    amax = oracle_mod.group_amax(xr_b, 1, None)
    gs = np.array([oracle_mod.global_scale(float(amax[0]))], np.float32)
    assert cap.gscale.cpu().numpy().view(np.uint32)[0] == gs.view(np.uint32)[0]
    rng = np.random.default_rng(layer * 4 + site)
    rows_idx = np.unique(np.concatenate([[0, R - 1], rng.integers(0, R, 64)]))
    rg = np.full(rows_idx.size, gs[0], np.float32)
    codes, _, scales = oracle_mod.capture_rows(xr_b[rows_idx], rg)
    ref = oracle_mod.mismatch_histogram(np.ascontiguousarray(xt_b[rows_idx]), codes, scales, gs)
    assert whole[2, 0] == R * C          # no q_roll outside its bracket at 0.5% drift
    acc.zero_()
    for r in rows_idx:
        x1, c1 = _row_slices(xt, cap, int(r), int(r) + 1, 0)
        ops.mismatch_histogram(x1, c1, acc)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().view(np.uint64), ref)


def test_hist_argument_errors():
    lib = ops.library()
    x = torch.zeros(4, 32, dtype=torch.bfloat16, device=DEV)
    cap = ops.capture(x)
    h = torch.zeros(3, 15, dtype=torch.int64, device=DEV)
    P = lambda t: t.data_ptr()
    assert lib.trace_mismatch_histogram(P(x), 4, 32, 1, None, P(cap.codes), P(cap.scales),
                                        P(cap.gscale), None, None) == 1
    assert lib.trace_mismatch_histogram(P(x), 4, 33, 1, None, P(cap.codes), P(cap.scales),
                                        P(cap.gscale), P(h), None) == 2
    assert lib.trace_mismatch_histogram(P(x) + 2, 4, 32, 1, None, P(cap.codes), P(cap.scales),
                                        P(cap.gscale), P(h), None) == 3
    assert lib.trace_mismatch_histogram(P(x), 4, 32, 1, None, P(cap.codes), P(cap.scales),
                                        P(cap.gscale), P(h) + 4, None) == 3
    torch.cuda.synchronize()
    assert int(h.abs().sum()) == 0


# --------------------------------------------------------------------------
# The MXFP4 variant of the diagnostic
# --------------------------------------------------------------------------

def _mx_check(oracle_mod, xr, xt):
    cap = ops.mx_capture(xr.to(DEV).contiguous())
    got = ops.mx_mismatch_histogram(xt.to(DEV).contiguous(), cap)
    torch.cuda.synchronize()
    got = got.cpu().numpy().view(np.uint64)
    xrb, xtb = inputs.bits(xr), inputs.bits(xt)
    codes, _, scales = oracle_mod.mx_capture(xrb)
    ref = oracle_mod.mx_mismatch_histogram(xtb, codes, scales)
    assert np.array_equal(got, ref), f"\n{got}\nvs\n{ref}"
    return got


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 96), (513, 2048)])
def test_mx_hist_small_and_special(oracle_mod, rows, cols):
    s = inputs.tiny_site(rows * 11 + cols, rows, cols, eps=0.05)
    _mx_check(oracle_mod, s.x_roll, s.x_train)
    rng = np.random.default_rng(rows)
    xt = torch.from_numpy((rng.standard_normal((rows, cols)) * 4).astype(np.float32)).to(torch.bfloat16)
    _mx_check(oracle_mod, s.x_roll, xt)              # independent: sign flips, long distances


def test_mx_hist_exhaustive_sweep(oracle_mod):
    """Every finite bf16 pattern x cycled rollout codes, one launch per E8M0
    scale byte across capture's range."""
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    pats = np.concatenate([p, np.zeros((-p.size) % 256, np.uint16)]).reshape(-1, 256)
    slab, C = pats.shape
    xd = inputs.from_bits(pats, DEV)
    idx = np.arange(slab * C, dtype=np.int64)
    hs = []
    for sb in range(0, 253, 4):
        nib = ((idx + sb) % 16).astype(np.uint8)
        rcodes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
        scales = np.full((slab, C // 32), sb, np.uint8)
        cache = ops.MxCapture(codes=torch.from_numpy(rcodes).to(DEV), mbits=None,
                              scales=torch.from_numpy(scales).to(DEV))
        hs.append((sb, ops.mx_mismatch_histogram(xd, cache),
                   oracle_mod.mx_mismatch_histogram(pats, rcodes, scales)))
    torch.cuda.synchronize()
    for sb, hg, hr in hs:
        assert np.array_equal(hg.cpu().numpy().view(np.uint64), hr), f"scale byte {sb}"


def test_mx_hist_cfg2(oracle_mod):
    s = inputs.attention_input(device=DEV)
    got = _mx_check(oracle_mod, s.x_roll, s.x_train)
    assert np.all(got.sum(axis=1) == s.x_roll.numel())
