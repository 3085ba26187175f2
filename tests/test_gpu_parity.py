"""Bit-exact parity of the CUDA path (through the C ABI) with the CPU oracle.

Every output -- FP4 codes, mantissa bits, E4M3 block scales, global scales,
dequantised bf16 outputs, STE masks and STE gradients -- must match the
oracle bit for bit (tolerance 0 ULP): the format fixes every rounding.

Workloads are the seeded synthetic sites of
``fp4_quantization_aware_trace_b200.inputs``; full tensors go through the
oracle where it finishes in seconds, and the largest ones are checked on
sampled rows, with the global scales computed by the oracle over the whole
tensor.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _u(t: torch.Tensor) -> np.ndarray:
    """device tensor -> host numpy array of its raw bits"""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    if t.dtype == torch.float32:
        return t.numpy()
    return t.numpy()


def _eq(name, got, ref):
    got = np.asarray(got).reshape(-1)
    ref = np.asarray(ref).reshape(-1)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    if got.dtype == np.float32:
        got, ref = got.view(np.uint32), ref.view(np.uint32)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, (f"{name}: {bad.size} mismatches, first at {bad[:8].tolist()}: "
                           f"got {got[bad[:8]].tolist()} ref {ref[bad[:8]].tolist()}")


def _offs_np(site):
    return None if site.offsets is None else site.offsets.cpu().numpy()


def run_gpu(site: inputs.Site):
    """capture(x_roll) -> guided(x_train) -> bwd(grad), plus RTN(x_train)."""
    xr = site.x_roll.to(DEV).contiguous()
    xt = site.x_train.to(DEV).contiguous()
    g = site.grad.to(DEV).contiguous()
    offs = None if site.offsets is None else site.offsets.to(DEV)
    cap = ops.capture(xr, offs)
    out, mask = ops.guided_fq_fwd(xt, cap)
    gin = ops.fq_bwd(g, mask)
    out_r, mask_r = ops.rtn_fq_fwd(xt, cap.scales, cap.gscale, offs)
    out_f, mask_f = ops.full_guided_fq_fwd(xt, cap)
    torch.cuda.synchronize()
    return dict(codes=_u(cap.codes), mbits=_u(cap.mbits), scales=_u(cap.scales),
                gscale=_u(cap.gscale), out=_u(out), mask=_u(mask), grad_in=_u(gin),
                out_rtn=_u(out_r), mask_rtn=_u(mask_r), out_full=_u(out_f), mask_full=_u(mask_f))


def run_oracle(oracle_mod, site: inputs.Site):
    xr, xt, g = inputs.bits(site.x_roll), inputs.bits(site.x_train), inputs.bits(site.grad)
    G, offs = site.num_groups, _offs_np(site)
    codes, mbits, scales, gscale = oracle_mod.capture(xr, G, offs)
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale, G, offs)
    out_r, mask_r = oracle_mod.rtn_fwd(xt, scales, gscale, G, offs)
    out_f, mask_f = oracle_mod.full_guided_fwd(xt, codes, scales, gscale, G, offs)
    gin = oracle_mod.fq_bwd(g, mask)
    return dict(codes=codes, mbits=mbits, scales=scales, gscale=gscale, out=out, mask=mask,
                grad_in=gin, out_rtn=out_r, mask_rtn=mask_r, out_full=out_f, mask_full=mask_f)


def run_oracle_mt(site: inputs.Site):
    """run_oracle through the threaded driver (row chunks on every core):
    the same results, for the largest tensors."""
    import oracle.threaded as ot
    xr, xt, g = inputs.bits(site.x_roll), inputs.bits(site.x_train), inputs.bits(site.grad)
    G, offs = site.num_groups, _offs_np(site)
    codes, mbits, scales, gscale = ot.capture_mt(xr, G, offs)
    out, mask = ot.guided_fwd_mt(xt, mbits, scales, gscale, G, offs)
    out_r, mask_r = ot.rtn_fwd_mt(xt, scales, gscale, G, offs)
    out_f, mask_f = ot.full_guided_fwd_mt(xt, codes, scales, gscale, G, offs)
    gin = ot.fq_bwd_mt(g, mask)
    return dict(codes=codes, mbits=mbits, scales=scales, gscale=gscale, out=out, mask=mask,
                grad_in=gin, out_rtn=out_r, mask_rtn=mask_r, out_full=out_f, mask_full=mask_f)


def check_full(oracle_mod, site, threaded: bool = False):
    got = run_gpu(site)
    ref = run_oracle_mt(site) if threaded else run_oracle(oracle_mod, site)
    for k in ref:
        _eq(f"{site.name}.{k}", got[k], ref[k])
    return got, ref


def check_sampled_rows(oracle_mod, site, rows_idx):
    """Parity on sampled rows of a tensor too large for the whole-tensor
    oracle: the oracle computes the per-group amax over the full tensor,
    then captures and fake-quantises the sampled rows on its own."""
    got = run_gpu(site)
    xr, xt, g = inputs.bits(site.x_roll), inputs.bits(site.x_train), inputs.bits(site.grad)
    R, C = xr.shape
    G, offs = site.num_groups, _offs_np(site)
    amax = oracle_mod.group_amax(xr, G, offs)
    gs = np.array([oracle_mod.global_scale(float(a)) for a in amax], np.float32)
    _eq(f"{site.name}.gscale", got["gscale"], gs)
    row_g = np.full(R, gs[0], np.float32) if G == 1 else np.repeat(gs, np.diff(offs))
    rows_idx = np.asarray(sorted(set(int(r) for r in rows_idx)))
    rg = np.ascontiguousarray(row_g[rows_idx], np.float32)
    codes, mbits, scales = oracle_mod.capture_rows(xr[rows_idx], rg)
    out, mask = oracle_mod.fake_quant_rows(xt[rows_idx], rg, scales, mbits)
    out_r, mask_r = oracle_mod.fake_quant_rows(xt[rows_idx], rg, scales, None)
    out_f, mask_f = oracle_mod.full_guided_rows(xt[rows_idx], rg, scales, codes)
    gin = oracle_mod.fq_bwd(np.ascontiguousarray(g[rows_idx]), mask)
    _eq(f"{site.name}.codes", got["codes"].reshape(R, C // 2)[rows_idx], codes)
    _eq(f"{site.name}.mbits", got["mbits"].reshape(R, C // 32)[rows_idx], mbits)
    _eq(f"{site.name}.scales", got["scales"].reshape(R, C // 16)[rows_idx], scales)
    _eq(f"{site.name}.out", got["out"].reshape(R, C)[rows_idx], out)
    _eq(f"{site.name}.mask", got["mask"].reshape(R, C // 32)[rows_idx], mask)
    _eq(f"{site.name}.out_rtn", got["out_rtn"].reshape(R, C)[rows_idx], out_r)
    _eq(f"{site.name}.mask_rtn", got["mask_rtn"].reshape(R, C // 32)[rows_idx], mask_r)
    _eq(f"{site.name}.grad_in", got["grad_in"].reshape(R, C)[rows_idx], gin)
    _eq(f"{site.name}.out_full", got["out_full"].reshape(R, C)[rows_idx], out_f)
    _eq(f"{site.name}.mask_full", got["mask_full"].reshape(R, C // 32)[rows_idx], mask_f)


def _sample_rows(R, k=96, seed=0):
    rng = np.random.default_rng(seed)
    return np.concatenate([[0, 1, R // 2, R - 2, R - 1], rng.integers(0, R, k)])


# ---------------------------------------------------------------------------
# Small cases: several tiles, ragged tails, groups, edge cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 32), (37, 96), (129, 160), (1000, 64),
                                       (513, 2048), (4099, 128)])
def test_parity_small_shapes(oracle_mod, rows, cols):
    check_full(oracle_mod, inputs.tiny_site(rows * 7 + cols, rows, cols, eps=0.02))


def test_parity_cfg1_single_activation(oracle_mod):
    check_full(oracle_mod, inputs.single_activation(0))


def test_parity_ragged_groups(oracle_mod):
    s = inputs.tiny_site(5, 777, 96, eps=0.01)
    x = s.x_roll.float()
    x[100:300] *= 1e4
    x[500:520] *= 1e-6
    s.x_roll = x.to(torch.bfloat16)
    s.x_train = (s.x_roll.float() * 1.003).to(torch.bfloat16)
    s.offsets = torch.tensor([0, 0, 1, 100, 300, 300, 301, 520, 777, 777], dtype=torch.int64)
    got, ref = check_full(oracle_mod, s)
    assert got["gscale"][0] == 1.0 and got["gscale"][4] == 1.0


def test_parity_many_small_groups(oracle_mod):
    s = inputs.tiny_site(6, 2000, 64)
    x = s.x_roll.float() * torch.exp(torch.linspace(-20, 20, 2000))[:, None]
    s.x_roll = x.to(torch.bfloat16)
    s.x_train = inputs._perturb(s.x_roll, 0.005, inputs._gen(1, "cpu"))
    s.offsets = torch.cat([torch.arange(0, 2000, 3, dtype=torch.int64), torch.tensor([2000])])
    check_full(oracle_mod, s)


def test_parity_empty_and_zero(oracle_mod):
    # rows == 0: only the global scales are written (amax 0 -> 1.0)
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    offs = torch.tensor([0, 0, 0], dtype=torch.int64, device=DEV)
    cap = ops.capture(x, offs)
    out, mask = ops.guided_fq_fwd(x, cap)
    torch.cuda.synchronize()
    assert cap.gscale.cpu().tolist() == [1.0, 1.0] and out.numel() == 0
    # all-zero tensor with negative zeros: zero blocks everywhere
    z = torch.zeros(64, 64)
    z[::2, 1::3] = -0.0
    s = inputs.Site("zeros", z.to(torch.bfloat16), z.to(torch.bfloat16),
                    torch.ones(64, 64).to(torch.bfloat16))
    got, _ = check_full(oracle_mod, s)
    assert np.all(got["mask"] == 0xFFFFFFFF)


def test_parity_special_values(oracle_mod):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x[0, :16] = 0.0                              # zero block
    x[1, :16] = 1e-39 * rng.standard_normal(16)  # subnormal block
    x[2, :] *= 1e30                              # large rows
    x[3, 5] = 3.3e38                             # near the bf16 maximum
    x[4, :32] = 2.0 ** -133                      # smallest subnormal
    x[5, :] = np.tile([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], 32)
    x[6, :] *= 1e-30
    xb = torch.from_numpy(x).to(torch.bfloat16)
    s = inputs.Site("special", xb, (xb.float() * 1.01).to(torch.bfloat16),
                    torch.from_numpy(rng.standard_normal((64, 256)).astype(np.float32)).to(torch.bfloat16))
    check_full(oracle_mod, s)
    s2 = inputs.Site("special_tiny", (xb.float() * 1e-30).to(torch.bfloat16), s.x_train, s.grad)
    check_full(oracle_mod, s2)


def test_parity_signed_zero_quotients(oracle_mod):
    """Zeros of both signs, and values whose quotient underflows to zero, in
    blocks whose scale keeps them on the kernels' fast path (block maxima
    from 1 to 1e30): every such element's code is the zero with the sign of
    x, and everything else matches the oracle."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((96, 256)).astype(np.float32)
    x[32:64] *= 1e30                  # d near 2^97: tiny values underflow
    x[:, 0::4] = np.float32(0.0)
    x[:, 1::4] = np.float32(-0.0)
    tiny = np.float32(2.0 ** -133)    # smallest bf16 subnormal
    x[:, 2::8] = tiny
    x[:, 6::8] = -tiny
    x[64:, 3::16] = np.float32(-1e-39)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    # one group per band of 32 rows, so each band gets its own global scale
    s = inputs.Site("signed_zeros", xb, (xb.float() * 1.003).to(torch.bfloat16),
                    torch.from_numpy(rng.standard_normal((96, 256)).astype(np.float32)).to(torch.bfloat16),
                    torch.tensor([0, 32, 64, 96], dtype=torch.int64))
    got, _ = check_full(oracle_mod, s)
    # every block is scaled (no zero-block shortcut)
    assert np.all(got["scales"] > 0)
    codes = got["codes"].reshape(-1)
    nib = np.stack([codes & 0xF, codes >> 4], axis=1).reshape(96, 256)
    assert np.all(nib[:, 0::4] == 0x0) and np.all(nib[:, 1::4] == 0x8)
    # the quotient of +-2^-133 by d >= 2^90 underflows: zero code, sign of x
    assert np.all(nib[32:64, 2::8] == 0x0) and np.all(nib[32:64, 6::8] == 0x8)


def test_guided_equals_rollout_rtn_when_same_input(oracle_mod):
    s = inputs.attention_input(seed=4, rows=512)
    s.x_train = s.x_roll.clone()
    got, _ = check_full(oracle_mod, s)
    assert np.array_equal(got["out"], got["out_rtn"])


# ---------------------------------------------------------------------------
# Exhaustive sweeps over bf16 inputs and scale choices
# ---------------------------------------------------------------------------

def _all_finite_bf16():
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    pad = (-p.size) % 256
    return np.concatenate([p, np.zeros(pad, np.uint16)]).reshape(-1, 256)


@pytest.mark.parametrize("bit", [0, 1])
def test_exhaustive_bf16_fake_quant(oracle_mod, bit):
    """All finite bf16 patterns x every E4M3 block scale x several global
    scales (power of two, full-mantissa, subnormal, huge, and around the
    edges of the kernels' fast range) through the guided and round-to-nearest
    forwards."""
    pats = _all_finite_bf16()                     # [255, 256]
    # includes scales at the edges of the kernels' fast ranges (d from 2^-90
    # to 2^16 for the guided forward, to 2^100 otherwise) and beyond them,
    # with every bf16 input, subnormals included
    gs_vals = np.array([1.0, 0.3712345, 2.0 ** -10, 7.1e-3, 2.0 ** -140, 1.9e30,
                        2.0 ** 30, 1.37 * 2.0 ** -80, 3.1e10, 2.0 ** 9, 911.0],
                       np.float32)
    sbytes = np.arange(0x7F, dtype=np.uint8)
    slab = pats.shape[0]
    x = np.tile(pats, (len(sbytes) * len(gs_vals), 1))
    R, C = x.shape
    scales = np.repeat(np.tile(np.repeat(sbytes, slab), len(gs_vals)), C // 16).reshape(R, C // 16)
    offs = np.arange(0, R + 1, slab * len(sbytes), dtype=np.int64)
    G = len(gs_vals)
    mbits = np.full(R * C // 32, 0xFFFFFFFF if bit else 0, np.uint32)

    xd = inputs.from_bits(x, DEV)
    sc = torch.from_numpy(scales).to(DEV)
    gs = torch.from_numpy(gs_vals).to(DEV)
    od = torch.from_numpy(offs).to(DEV)
    mb = torch.from_numpy(mbits.view(np.int32)).to(DEV)
    cache = ops.Capture(codes=None, mbits=mb, scales=sc, gscale=gs, offsets=od)
    out, mask = ops.guided_fq_fwd(xd, cache)
    out_r, mask_r = ops.rtn_fq_fwd(xd, sc, gs, od)
    torch.cuda.synchronize()
    ref, ref_m = oracle_mod.guided_fwd(x, mbits, scales, gs_vals, G, offs)
    _eq("guided_out", _u(out), ref)
    _eq("guided_mask", _u(mask), ref_m)
    ref_r, ref_rm = oracle_mod.rtn_fwd(x, scales, gs_vals, G, offs)
    _eq("rtn_out", _u(out_r), ref_r)
    _eq("rtn_mask", _u(mask_r), ref_rm)


def test_exhaustive_bf16_full_guided(oracle_mod):
    """Full-information guidance: every finite bf16 pattern against every
    signed rollout code (cycled across the slabs), every E4M3 block scale and
    the same global scales as the bit-guided sweep."""
    pats = _all_finite_bf16()
    gs_vals = np.array([1.0, 0.3712345, 2.0 ** -140, 1.9e30, 2.0 ** 9, 911.0], np.float32)
    sbytes = np.arange(0x7F, dtype=np.uint8)
    slab = pats.shape[0]
    x = np.tile(pats, (len(sbytes) * len(gs_vals), 1))
    R, C = x.shape
    scales = np.repeat(np.tile(np.repeat(sbytes, slab), len(gs_vals)), C // 16).reshape(R, C // 16)
    offs = np.arange(0, R + 1, slab * len(sbytes), dtype=np.int64)
    G = len(gs_vals)
    idx = np.arange(R * C, dtype=np.int64)
    nib = ((idx + idx // (slab * C)) % 16).astype(np.uint8)
    rcodes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    xd = inputs.from_bits(x, DEV)
    cache = ops.Capture(codes=torch.from_numpy(rcodes).to(DEV), mbits=None,
                        scales=torch.from_numpy(scales).to(DEV),
                        gscale=torch.from_numpy(gs_vals).to(DEV),
                        offsets=torch.from_numpy(offs).to(DEV))
    out, mask = ops.full_guided_fq_fwd(xd, cache)
    torch.cuda.synchronize()
    ref, ref_m = oracle_mod.full_guided_fwd(x, rcodes, scales, gs_vals, G, offs)
    _eq("full_out", _u(out), ref)
    _eq("full_mask", _u(mask), ref_m)


def test_exhaustive_bf16_capture(oracle_mod):
    """All finite bf16 patterns through capture, in groups whose amax puts
    them in different parts of the scale range, and with every block holding
    one pattern next to a fixed maximum (every E4M3 rounding case of t)."""
    pats = _all_finite_bf16()
    R = pats.shape[0]
    rows = [pats]
    # each pattern p as the max of its own block, next to small values
    p = np.arange(1, 0x7F80, dtype=np.uint16)
    blocks = np.zeros((p.size, 16), np.uint16)
    blocks[:, 0] = p
    blocks[:, 1:] = (p[:, None] >> 1) & 0x7FFF
    blocks = np.concatenate([blocks, np.zeros(((-blocks.size) % (256 * 16) // 16, 16), np.uint16)])
    rows.append(blocks.reshape(-1, 256))
    x = np.concatenate(rows + [pats & 0x3FFF, pats & 0x1FFF])
    offs = np.array([0, R, R + rows[1].shape[0], R + rows[1].shape[0] + R, x.shape[0]], np.int64)
    s = inputs.Site("sweep", inputs.from_bits(x), inputs.from_bits(x), inputs.from_bits(x),
                    torch.from_numpy(offs))
    check_full(oracle_mod, s)


# ---------------------------------------------------------------------------
# The workloads at their full sizes
# ---------------------------------------------------------------------------

def test_parity_cfg2_attention_input_full(oracle_mod):
    check_full(oracle_mod, inputs.attention_input(device=DEV))


@pytest.mark.parametrize("which", ["k", "v"])
def test_parity_cfg4_kv_cache_full(oracle_mod, which):
    check_full(oracle_mod, inputs.kv_cache(device=DEV, which=which))


@pytest.mark.parametrize("cols,name", [(2048, "expert_up_in"), (768, "expert_down_in")])
def test_parity_cfg3_moe_experts_full(oracle_mod, cols, name):
    s = inputs.moe_experts(seed=2 if cols == 2048 else 12, cols=cols, device=DEV, name=name)
    check_full(oracle_mod, s, threaded=True)


@pytest.mark.parametrize("layer,site", [(20, 0), (39, 3)])
def test_parity_cfg5_layer_sweep_full(oracle_mod, layer, site):
    """Two whole sites of the sweep ([65536, 4096], 268 M elements each),
    every output compared element by element."""
    check_full(oracle_mod, inputs.layer_sweep_site(layer, site, device=DEV), threaded=True)


@pytest.mark.parametrize("layer,site", [(31, 2), (27, 1)])
def test_parity_cfg5_layer_sweep_sampled(oracle_mod, layer, site):
    s = inputs.layer_sweep_site(layer, site, device=DEV)
    check_sampled_rows(oracle_mod, s, _sample_rows(s.x_roll.shape[0], 64, layer))


# ---------------------------------------------------------------------------
# Buffer discipline: aliasing, canaries, argument errors
# ---------------------------------------------------------------------------

def test_inplace_aliasing(oracle_mod):
    s = inputs.tiny_site(3, 300, 128)
    xr, xt = s.x_roll.to(DEV), s.x_train.to(DEV)
    cap = ops.capture(xr)
    ref, _ = ops.guided_fq_fwd(xt, cap)
    buf = xt.clone()
    ops.guided_fq_fwd(buf, cap, out=buf)
    g = s.grad.to(DEV)
    _, mask = ops.guided_fq_fwd(xt, cap)
    gref = ops.fq_bwd(g, mask)
    gbuf = g.clone()
    ops.fq_bwd(gbuf, mask, out=gbuf)
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(gbuf.view(torch.int16), gref.view(torch.int16))


def test_canaries_untouched():
    """Outputs padded with 4 KiB sentinels on both sides: no call writes
    outside its buffers (odd row counts, several group counts)."""
    PAD = 4096
    for rows, cols, offs in [(37, 96, None), (257, 64, [0, 100, 100, 257]),
                             (1001, 32, list(range(0, 1001, 7)) + [1001])]:
        s = inputs.tiny_site(rows, rows, cols)
        n = rows * cols
        o = None if offs is None else torch.tensor(offs, dtype=torch.int64, device=DEV)
        G = 1 if offs is None else len(offs) - 1

        def padded(nbytes):
            b = torch.full((nbytes + 2 * PAD,), 0xA5, dtype=torch.uint8, device=DEV)
            return b, b[PAD:PAD + nbytes]

        bufs = {k: padded(v) for k, v in dict(codes=n // 2, mbits=n // 8, scales=n // 16,
                                                 gscale=4 * G, out=2 * n, mask=n // 8,
                                                 gin=2 * n).items()}
        v = {k: b[1] for k, b in bufs.items()}
        ws = torch.zeros(ops.trace_capture_workspace_bytes(rows, cols, G), dtype=torch.uint8, device=DEV)
        xr, xt, g = s.x_roll.to(DEV), s.x_train.to(DEV), s.grad.to(DEV)
        ops.trace_capture(xr, rows, cols, G, o, v["codes"], v["mbits"], v["scales"], v["gscale"],
                          ws, ws.numel())
        ops.trace_guided_fq_fwd(xt, rows, cols, G, o, v["mbits"], v["scales"], v["gscale"],
                                v["out"], v["mask"])
        ops.trace_rtn_fq_fwd(xt, rows, cols, G, o, v["scales"], v["gscale"], v["out"], v["mask"])
        ops.trace_fq_bwd(g, v["mask"], n, v["gin"])
        torch.cuda.synchronize()
        for k, (b, _) in bufs.items():
            assert torch.all(b[:PAD] == 0xA5) and torch.all(b[-PAD:] == 0xA5), k


def test_argument_errors_enqueue_nothing():
    lib = ops.library()
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    cap, ws = ops.alloc_capture(64, 64)
    P = lambda t, off=0: __import__("ctypes").c_void_p(t.data_ptr() + off)
    assert lib.trace_capture(P(x), 64, 48, 1, None, P(cap.codes), P(cap.mbits), P(cap.scales),
                             P(cap.gscale), P(ws), ws.numel(), None) == 2
    assert lib.trace_capture(P(x, 2), 64, 64, 1, None, P(cap.codes), P(cap.mbits), P(cap.scales),
                             P(cap.gscale), P(ws), ws.numel(), None) == 3
    assert lib.trace_capture(P(x), 64, 64, 1, None, P(cap.codes), P(cap.mbits), P(cap.scales),
                             P(cap.gscale), P(ws), 0, None) == 4
    assert lib.trace_capture(P(x), 64, 64, 2, None, P(cap.codes), P(cap.mbits), P(cap.scales),
                             P(cap.gscale), P(ws), ws.numel(), None) == 1
    assert lib.trace_fq_bwd(P(x), P(cap.mbits), 48, P(x), None) == 2
    torch.cuda.synchronize()


def test_two_sites_on_two_lanes_in_a_cuda_graph(oracle_mod):
    """Two independent sites captured into one graph on two stream lanes
    (each lane: capture -> guided -> bwd, with the RTN comparator on the
    lane's side stream), forked from and joined to the capture stream, as
    the benchmark runs multi-site workloads: every output matches the
    oracle."""
    sites = [inputs.tiny_site(71, 384, 256, eps=0.01), inputs.tiny_site(72, 512, 128, eps=0.02)]
    bufs = []
    for st in sites:
        R, C = st.x_roll.shape
        cap, ws = ops.alloc_capture(R, C)
        bufs.append(dict(xr=st.x_roll.to(DEV), xt=st.x_train.to(DEV), g=st.grad.to(DEV),
                         cap=cap, ws=ws, out=torch.empty(R, C, dtype=torch.bfloat16, device=DEV),
                         mask=torch.empty(R * C // 32, dtype=torch.int32, device=DEV),
                         gin=torch.empty(R, C, dtype=torch.bfloat16, device=DEV),
                         out_r=torch.empty(R, C, dtype=torch.bfloat16, device=DEV),
                         mask_r=torch.empty(R * C // 32, dtype=torch.int32, device=DEV)))
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    lanes = [(torch.cuda.Stream(), torch.cuda.Stream()) for _ in sites]
    gph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gph, stream=cs, capture_error_mode="thread_local"):
        for (m, sd), b in zip(lanes, bufs):
            m.wait_stream(cs)
            ops.capture(b["xr"], None, b["cap"], b["ws"], m)
            sd.wait_stream(m)
            ops.rtn_fq_fwd(b["xt"], b["cap"].scales, b["cap"].gscale, None, b["out_r"], b["mask_r"], sd)
            ops.guided_fq_fwd(b["xt"], b["cap"], b["out"], b["mask"], m)
            ops.fq_bwd(b["g"], b["mask"], b["gin"], m)
        for m, sd in lanes:
            cs.wait_stream(m)
            cs.wait_stream(sd)
    gph.replay()
    torch.cuda.synchronize()
    for k, (st, b) in enumerate(zip(sites, bufs)):
        ref = run_oracle(oracle_mod, st)
        got = dict(codes=_u(b["cap"].codes), mbits=_u(b["cap"].mbits), scales=_u(b["cap"].scales),
                   gscale=_u(b["cap"].gscale), out=_u(b["out"]), mask=_u(b["mask"]),
                   grad_in=_u(b["gin"]), out_rtn=_u(b["out_r"]), mask_rtn=_u(b["mask_r"]))
        for key in got:
            _eq(f"lanes.{k}.{key}", got[key], ref[key])
    del gph


@pytest.mark.parametrize("forked", [False, True])
def test_step_in_a_cuda_graph(oracle_mod, forked):
    """The library's launches (with programmatic stream serialization) can be
    captured into a CUDA graph: a captured capture -> guided -> bwd -> RTN step
    replays to the oracle's outputs, also on new inputs copied into the same
    buffers.  Forked: the RTN comparator on a second stream after the
    capture, beside the guided forward and the backward (the benchmark's
    graph)."""
    s = inputs.tiny_site(61, 640, 512, eps=0.01)
    xr, xt, g = (t.to(DEV) for t in (s.x_roll, s.x_train, s.grad))
    cap, ws = ops.alloc_capture(640, 512)
    out = torch.empty_like(xt)
    mask = torch.empty(640 * 512 // 32, dtype=torch.int32, device=DEV)
    gin = torch.empty_like(g)
    out_r = torch.empty_like(xt)
    mask_r = torch.empty_like(mask)
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    gph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(gph, stream=cs, capture_error_mode="thread_local"):
        ops.capture(xr, None, cap, ws, cs)
        if forked:
            side.wait_stream(cs)
            ops.rtn_fq_fwd(xt, cap.scales, cap.gscale, None, out_r, mask_r, side)
        ops.guided_fq_fwd(xt, cap, out, mask, cs)
        ops.fq_bwd(g, mask, gin, cs)
        if forked:
            cs.wait_stream(side)
        else:
            ops.rtn_fq_fwd(xt, cap.scales, cap.gscale, None, out_r, mask_r, cs)
    for seed in (61, 62):
        if seed == 62:
            s = inputs.tiny_site(seed, 640, 512, eps=0.03)
            xr.copy_(s.x_roll.to(DEV))
            xt.copy_(s.x_train.to(DEV))
            g.copy_(s.grad.to(DEV))
        gph.replay()
        torch.cuda.synchronize()
        ref = run_oracle(oracle_mod, s)
        got = dict(codes=_u(cap.codes), mbits=_u(cap.mbits), scales=_u(cap.scales),
                   gscale=_u(cap.gscale), out=_u(out), mask=_u(mask), grad_in=_u(gin),
                   out_rtn=_u(out_r), mask_rtn=_u(mask_r))
        for k in got:
            _eq(f"graph.{seed}.{k}", got[k], ref[k])
    del gph


def test_workspace_left_zeroed_and_reused(oracle_mod):
    """Capture leaves its workspace ready for the next call -- the arrival
    count and the accumulators zero (the grid barrier's last CTA resets
    them), the error flag clear, the call count advanced by one -- so one
    workspace serves calls one after another: a tensor with a huge maximum,
    then ragged groups of small values, then an empty tensor -- each matches
    the oracle."""
    cases = []
    a = inputs.tiny_site(501, 700, 256).x_roll.float()
    a[13, 7] = 3.0e5
    cases.append((a.to(torch.bfloat16), None))
    b = (inputs.tiny_site(502, 300, 128).x_roll.float() * 1e-4).to(torch.bfloat16)
    cases.append((b, np.array([0, 50, 50, 300], np.int64)))
    cases.append((torch.zeros(0, 64, dtype=torch.bfloat16), None))
    G_max = 3
    ws = torch.zeros(ops.trace_capture_workspace_bytes(1, 32, G_max), dtype=torch.uint8, device=DEV)
    for k, (x, offs) in enumerate(cases):
        R, C = x.shape
        G = 1 if offs is None else len(offs) - 1
        o = None if offs is None else torch.from_numpy(offs).to(DEV)
        cap, _ = ops.alloc_capture(R, C, G, DEV, o)
        ops.capture(x.to(DEV), o, cap, ws)
        torch.cuda.synchronize()
        w = ws.view(torch.int32).cpu()
        assert int(w[0]) == 0 and int(w[2]) == 0 and int(w[1]) == k + 1
        assert int(w[3:].count_nonzero()) == 0
        ref = oracle_mod.capture(inputs.bits(x), G, offs)
        for name, got, want in zip(("codes", "mbits", "scales", "gscale"),
                                   (cap.codes, cap.mbits, cap.scales, cap.gscale), ref):
            _eq(name, _u(got), want)


@pytest.mark.parametrize("numel", [16, 8192 * 16 - 16, 8192 * 16 * 37 + 48])
def test_copy_yardsticks_copy_every_byte(numel):
    """The two bandwidth yardsticks (plain, and reads staged through shared
    memory by the bulk-copy engine) copy every element, ragged last tile
    included, and the staged one reports no timed-out wait."""
    src = torch.randn(numel, device=DEV).to(torch.bfloat16)
    for staged in (False, True):
        dst = torch.full_like(src, 7.0)
        if staged:
            err = torch.zeros(1, dtype=torch.int32, device=DEV)
            ops.trace_copy_bf16_staged(src, dst, numel, err)
        else:
            ops.trace_copy_bf16(src, dst, numel)
        torch.cuda.synchronize()
        assert torch.equal(dst.view(torch.int16), src.view(torch.int16)), staged
        if staged:
            assert int(err.item()) == 0


@pytest.mark.parametrize("drift", ["drifted", "independent"])
def test_guided_rules_in_place_and_separate_vs_oracle(oracle_mod, drift):
    """Every guided rule of every format, written to a separate buffer (the
    forwards then recompute disagreeing pairs after storing round to
    nearest) and in place over x_train (they patch each block in registers),
    against the oracle.  Independent training values make most sites
    disagree with the rollout, so the recompute paths carry most of the
    work; drifted ones exercise the common sparse case."""
    s = inputs.tiny_site(611, 640, 256, eps=0.02)
    xr = s.x_roll
    xt = s.x_train if drift == "drifted" else inputs.tiny_site(612, 640, 256).x_roll
    hr, ht = inputs.bits(xr), inputs.bits(xt)
    xr_d, xt_d = xr.to(DEV), xt.to(DEV)
    codes, mbits, scales, gscale = oracle_mod.capture(hr)
    c4, b4, s4 = oracle_mod.mx_capture(hr)
    c8, b8, s8 = oracle_mod.mx8_capture(hr)
    cases = {
        "nvfp4 guided": (lambda x, o: ops.guided_fq_fwd(x, ops.capture(xr_d), out=o),
                         oracle_mod.guided_fwd(ht, mbits, scales, gscale)),
        "nvfp4 full": (lambda x, o: ops.full_guided_fq_fwd(x, ops.capture(xr_d), out=o),
                       oracle_mod.full_guided_fwd(ht, codes, scales, gscale)),
        "mxfp4 guided": (lambda x, o: ops.mx_guided_fq_fwd(x, ops.mx_capture(xr_d), out=o),
                         oracle_mod.mx_guided_fwd(ht, b4, s4)),
        "mxfp4 full": (lambda x, o: ops.mx_full_guided_fq_fwd(x, ops.mx_capture(xr_d), out=o),
                       oracle_mod.mx_full_guided_fwd(ht, c4, s4)),
        "w4a8 guided": (lambda x, o: ops.mx8_guided_fq_fwd(x, ops.mx8_capture(xr_d), out=o),
                        oracle_mod.mx8_guided_fwd(ht, b8, s8)),
        "w4a8 full": (lambda x, o: ops.mx8_full_guided_fq_fwd(x, ops.mx8_capture(xr_d), out=o),
                      oracle_mod.mx8_full_guided_fwd(ht, c8, s8)),
    }
    for name, (fn, (ref_out, ref_mask)) in cases.items():
        sep_out, sep_mask = fn(xt_d, torch.empty_like(xt_d))
        buf = xt_d.clone()
        inp_out, inp_mask = fn(buf, buf)
        torch.cuda.synchronize()
        _eq(f"{name} separate out", _u(sep_out), ref_out)
        _eq(f"{name} separate mask", _u(sep_mask), ref_mask)
        _eq(f"{name} in-place out", _u(buf), ref_out)
        _eq(f"{name} in-place mask", _u(inp_mask), ref_mask)


def test_guided_separate_outputs_many_tiles_per_cta(oracle_mod):
    """The guided forwards with separate outputs store round to nearest and
    then recompute the pairs where the rule disagrees.  A [40960, 8192]
    tensor gives every CTA eight or nine tiles; its rows 1024-3071 carry
    training values drawn independently of the rollout's, so that most
    pairs there are recomputed, while the other rows drift slightly.  The
    whole tensor of both guided rules against the threaded oracle."""
    import oracle.threaded as ot
    R, C = 40960, 8192
    s = inputs.lognormal_site(7301, R, C, device=DEV, name="sep_many_tiles")
    other = inputs.lognormal_site(7302, 2048, C, device=DEV, name="other")
    xt = s.x_train.clone()
    xt[1024:3072] = other.x_roll
    cap = ops.capture(s.x_roll)
    out, mask = ops.guided_fq_fwd(xt, cap)
    out_f, mask_f = ops.full_guided_fq_fwd(xt, cap)
    torch.cuda.synchronize()
    hr, ht = inputs.bits(s.x_roll), inputs.bits(xt)
    del s, other, xt
    codes, mbits, scales, gscale = ot.capture_mt(hr)
    _eq("sep_many_tiles.codes", _u(cap.codes), codes)
    _eq("sep_many_tiles.mbits", _u(cap.mbits), mbits)
    ref_out, ref_mask = ot.guided_fwd_mt(ht, mbits, scales, gscale)
    _eq("sep_many_tiles.out", _u(out), ref_out)
    _eq("sep_many_tiles.mask", _u(mask), ref_mask)
    del ref_out, ref_mask
    ref_out, ref_mask = ot.full_guided_fwd_mt(ht, codes, scales, gscale)
    _eq("sep_many_tiles.out_full", _u(out_f), ref_out)
    _eq("sep_many_tiles.mask_full", _u(mask_f), ref_mask)


def test_capture_grid_barrier_gives_up_and_flags(oracle_mod):
    """The one-launch capture's grid barrier waits a bounded time.  A
    workspace whose arrival count starts far from zero never lets any CTA
    see itself arrive last, so nobody releases the barrier: every CTA gives
    up after its polls (about two seconds on B200), sets the workspace's error flag and
    returns.  The call itself succeeds, the GPU stays usable, and a capture
    with a clean workspace right after matches the oracle."""
    x = inputs.tiny_site(901, 512, 256).x_roll
    R, C = x.shape
    ws = torch.zeros(ops.trace_capture_workspace_bytes(R, C, 1), dtype=torch.uint8, device=DEV)
    w = ws.view(torch.int32)
    w[0] = 1 << 30  # the arrival count: no CTA draws gridDim.x - 1
    cap, _ = ops.alloc_capture(R, C, 1, DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ops.capture(x.to(DEV), None, cap, ws)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    print(f"grid barrier gave up after {waited:.2f} s")
    assert int(w[2].item()) == 1, "the barrier did not report giving up"
    assert waited < 30.0
    assert ops.capture_status(ws) is False  # TRACE_ERR_TIMEOUT, and the word is cleared
    assert int(w[2].item()) == 0
    ws.zero_()
    cap, _ = ops.alloc_capture(R, C, 1, DEV)
    ops.capture(x.to(DEV), None, cap, ws)
    torch.cuda.synchronize()
    assert int(w[2].item()) == 0 and ops.capture_status(ws) is True
    ref = oracle_mod.capture(inputs.bits(x), 1, None)
    for name, got, want in zip(("codes", "mbits", "scales", "gscale"),
                               (cap.codes, cap.mbits, cap.scales, cap.gscale), ref):
        _eq(name, _u(got), want)
