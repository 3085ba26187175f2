"""Capture and forwards with the block scales in the 128 x 4 tiled layout of
a block-scaled FP4 GEMM: the tiled scale bytes equal the oracle's row-major
scales put through the oracle's layout transform (itself pinned against
vllm's), the other outputs equal the row-major path's oracle outputs, and
the padding is never written."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"
RULES = (ops.TRACE_RULE_RTN, ops.TRACE_RULE_GUIDED, ops.TRACE_RULE_FULL)


def _u(t):
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def _eq(name, got, ref):
    got, ref = np.asarray(got).reshape(-1), np.asarray(ref).reshape(-1)
    assert got.shape == ref.shape, f"{name}: {got.shape} vs {ref.shape}"
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"{name}: {bad.size} mismatches at {bad[:8].tolist()}"


def _nv_oracle(oracle_mod, xr, xt, G, offs):
    codes, mbits, scales, gscale = oracle_mod.capture(xr, G, offs)
    outs = {ops.TRACE_RULE_GUIDED: oracle_mod.guided_fwd(xt, mbits, scales, gscale, G, offs),
            ops.TRACE_RULE_RTN: oracle_mod.rtn_fwd(xt, scales, gscale, G, offs),
            ops.TRACE_RULE_FULL: oracle_mod.full_guided_fwd(xt, codes, scales, gscale, G, offs)}
    return codes, mbits, scales, gscale, outs


def check_nv(oracle_mod, site):
    xr, xt = site.x_roll.to(DEV), site.x_train.to(DEV)
    offs = None if site.offsets is None else site.offsets.to(DEV)
    cap = ops.capture_tiled(xr, offs)
    got = {r: ops.fq_fwd_tiled(r, xt, cap) for r in RULES}
    torch.cuda.synchronize()
    G = site.num_groups
    o = None if site.offsets is None else site.offsets.numpy()
    codes, mbits, scales, gscale, outs = _nv_oracle(oracle_mod, inputs.bits(site.x_roll),
                                                    inputs.bits(site.x_train), G, o)
    _eq("codes", _u(cap.codes), codes)
    _eq("mbits", _u(cap.mbits), mbits)
    _eq("gscale", _u(cap.gscale).view(np.uint32), gscale.view(np.uint32))
    _eq("tiled scales", _u(cap.scales), oracle_mod.swizzle_scales(scales))
    for r in RULES:
        _eq(f"out rule {r}", _u(got[r][0]), outs[r][0])
        _eq(f"mask rule {r}", _u(got[r][1]), outs[r][1])


def check_mx(oracle_mod, xr_cpu, xt_cpu):
    xr, xt = xr_cpu.to(DEV), xt_cpu.to(DEV)
    cap = ops.mx_capture_tiled(xr)
    got = {r: ops.mx_fq_fwd_tiled(r, xt, cap) for r in RULES}
    torch.cuda.synchronize()
    xrb, xtb = inputs.bits(xr_cpu), inputs.bits(xt_cpu)
    codes, mbits, scales = oracle_mod.mx_capture(xrb)
    outs = {ops.TRACE_RULE_GUIDED: oracle_mod.mx_guided_fwd(xtb, mbits, scales),
            ops.TRACE_RULE_RTN: oracle_mod.mx_rtn_fwd(xtb, scales),
            ops.TRACE_RULE_FULL: oracle_mod.mx_full_guided_fwd(xtb, codes, scales)}
    _eq("mx codes", _u(cap.codes), codes)
    _eq("mx mbits", _u(cap.mbits), mbits)
    _eq("mx tiled scales", _u(cap.scales), oracle_mod.swizzle_scales(scales))
    for r in RULES:
        _eq(f"mx out rule {r}", _u(got[r][0]), outs[r][0])
        _eq(f"mx mask rule {r}", _u(got[r][1]), outs[r][1])


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (37, 64), (129, 160), (300, 2048),
                                       (513, 128)])
def test_tiled_small_shapes(oracle_mod, rows, cols):
    s = inputs.tiny_site(rows * 3 + cols, rows, cols, eps=0.02)
    check_nv(oracle_mod, s)
    check_mx(oracle_mod, s.x_roll, s.x_train)


def test_tiled_grouped(oracle_mod):
    s = inputs.tiny_site(5, 777, 96, eps=0.01)
    x = s.x_roll.float()
    x[100:300] *= 1e4
    s.x_roll = x.to(torch.bfloat16)
    s.x_train = (s.x_roll.float() * 1.003).to(torch.bfloat16)
    s.offsets = torch.tensor([0, 0, 1, 100, 300, 300, 301, 520, 777, 777], dtype=torch.int64)
    check_nv(oracle_mod, s)


def test_tiled_cfg2_full(oracle_mod):
    s = inputs.attention_input(device=DEV)
    check_nv(oracle_mod, s)
    check_mx(oracle_mod, s.x_roll, s.x_train)


def test_tiled_scales_match_library_swizzle():
    """The tiled E4M3 scales of capture equal vllm's swizzle of the row-major
    scales of capture (both on the GPU)."""
    nv = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_utils")
    s = inputs.tiny_site(11, 300, 512, eps=0.01)
    xr = s.x_roll.to(DEV)
    lin = ops.capture(xr)
    tiled = ops.capture_tiled(xr)
    ref = nv.swizzle_blockscale(lin.scales.view(torch.float8_e4m3fn))
    torch.cuda.synchronize()
    _eq("library swizzle", _u(tiled.scales), ref.reshape(-1).view(torch.uint8).cpu().numpy())


def test_tiled_padding_untouched():
    x = torch.randn(130, 96, device=DEV).to(torch.bfloat16)
    nb = ops.trace_scale_bytes(130, 96, 16, ops.TRACE_SCALES_TILED_128x4)
    assert nb == 2 * 2 * 512
    cap, ws = ops.alloc_capture(130, 96)
    sc = torch.full((nb,), 0xA5, dtype=torch.uint8, device=DEV)
    ops.trace_capture_ex(x, 130, 96, 1, None, cap.codes, cap.mbits, sc, cap.gscale, ws,
                         ws.numel(), ops.TRACE_SCALES_TILED_128x4)
    torch.cuda.synchronize()
    h = sc.cpu().numpy()
    r = np.arange(256)[:, None]
    c = np.arange(8)[None, :]
    off = ((r // 128) * 2 + c // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + c % 4
    data = (r < 130) & (c < 6)
    assert np.all(h[off[~data]] == 0xA5)          # padding never written


def test_ex_argument_errors():
    lib = ops.library()
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    cap, ws = ops.alloc_capture(4, 64)
    out = torch.empty_like(x)
    mask = torch.zeros(8, dtype=torch.int32, device=DEV)
    P = lambda t: t.data_ptr()
    assert lib.trace_capture_ex(P(x), 4, 64, 1, None, P(cap.codes), P(cap.mbits), P(cap.scales),
                                P(cap.gscale), P(ws), ws.numel(), 2, None) == 2
    assert lib.trace_fq_fwd_ex(3, P(x), 4, 64, 1, None, P(cap.mbits), P(cap.codes), P(cap.scales),
                               P(cap.gscale), P(out), P(mask), 0, None) == 2
    assert lib.trace_mx_fq_fwd_ex(-1, P(x), 4, 64, P(cap.mbits), P(cap.codes), P(cap.scales),
                                  P(out), P(mask), 1, None) == 2
    assert lib.trace_scale_bytes(4, 64, 8, 0) == 0 and lib.trace_scale_bytes(4, 64, 16, 5) == 0
    torch.cuda.synchronize()
    assert int(mask.abs().sum()) == 0


def test_row_sharded_capture_matches_whole(oracle_mod):
    """Three row shards of one grouped tensor, captured with the two-pass
    entry points around a MAX reduction of the per-group amax (done here
    with torch.maximum on one GPU, as the all-reduce would across GPUs):
    every shard's outputs equal the oracle's capture of the whole tensor."""
    s = inputs.tiny_site(21, 600, 256, eps=0.01)
    x = s.x_roll.float()
    x[100:250] *= 1e3
    s.x_roll = x.to(torch.bfloat16)
    offs = np.array([0, 150, 150, 420, 600], np.int64)
    G = 4
    cuts = [0, 200, 333, 600]
    xd = s.x_roll.to(DEV)
    amaxes, shards = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        lo = np.clip(offs - a, 0, b - a)
        o = torch.from_numpy(lo).to(DEV)
        am = torch.empty(G, dtype=torch.int32, device=DEV)
        ops.trace_capture_amax(xd[a:b], b - a, 256, G, o, am)
        amaxes.append(am)
        shards.append((a, b, o))
    red = torch.stack(amaxes).max(dim=0).values
    codes, mbits, scales, gscale = oracle_mod.capture(inputs.bits(s.x_roll), G, offs)
    for a, b, o in shards:
        cap, _ = ops.alloc_capture(b - a, 256, G, DEV, o)
        ops.trace_capture_with_amax(xd[a:b], b - a, 256, G, o, red, cap.codes, cap.mbits,
                                    cap.scales, cap.gscale)
        torch.cuda.synchronize()
        _eq("gscale", _u(cap.gscale).view(np.uint32), gscale.view(np.uint32))
        _eq("codes", _u(cap.codes), codes[a * 128:b * 128])
        _eq("mbits", _u(cap.mbits), mbits[a * 8:b * 8])
        _eq("scales", _u(cap.scales), scales[a:b])
    # one GPU, no process group: the sharded helper is a whole capture
    one = ops.capture_sharded(xd, torch.from_numpy(offs).to(DEV))
    torch.cuda.synchronize()
    _eq("sharded helper codes", _u(one.codes), codes)
    _eq("sharded helper scales", _u(one.scales), scales)
    _eq("sharded helper gscale", _u(one.gscale).view(np.uint32), gscale.view(np.uint32))


@pytest.mark.parametrize("rows,cols,chunks,grouped", [(600, 256, 4, True), (1000, 96, 3, False),
                                                       (16384, 2048, 4, False)])
def test_host_step_matches_oracle(oracle_mod, rows, cols, chunks, grouped):
    """The host-to-host step (row chunks, amax accumulated across chunks,
    copies overlapped on three streams) returns the oracle's outputs."""
    from fp4_quantization_aware_trace_b200 import host_step
    if rows == 16384:
        s = inputs.attention_input()
    else:
        s = inputs.tiny_site(rows + cols, rows, cols, eps=0.01)
    offs = np.array([0, rows // 5, rows // 5, rows * 3 // 4, rows], np.int64) if grouped else None
    G = 4 if grouped else 1
    h = host_step.HostStep(rows, cols, offs, chunks=chunks)
    assert len(h.cuts) >= 2
    xr_h, xt_h, g_h = (t.contiguous().pin_memory() for t in (s.x_roll, s.x_train, s.grad))
    out_h = h.alloc_host()
    for _ in range(2):                       # twice: buffers are reused
        h.run(xr_h, xt_h, g_h, out_h)
        torch.cuda.synchronize()
    xr, xt, g = inputs.bits(s.x_roll), inputs.bits(s.x_train), inputs.bits(s.grad)
    codes, mbits, scales, gscale = oracle_mod.capture(xr, G, offs)
    out, mask = oracle_mod.guided_fwd(xt, mbits, scales, gscale, G, offs)
    out_r, mask_r = oracle_mod.rtn_fwd(xt, scales, gscale, G, offs)
    gin = oracle_mod.fq_bwd(g, mask)
    ref = dict(codes=codes, mbits=mbits, scales=scales, gscale=gscale, out=out, mask=mask,
               grad_in=gin, out_rtn=out_r, mask_rtn=mask_r)
    for k, v in ref.items():
        got = _u(out_h[k])
        if k == "gscale":
            got, v = got.view(np.uint32), v.view(np.uint32)
        _eq(f"host step {k}", got, v)


@pytest.mark.parametrize("rows,cols", [(3, 64), (129, 160), (300, 2048)])
def test_w4a8_tiled(oracle_mod, rows, cols):
    s = inputs.tiny_site(rows * 5 + cols, rows, cols, eps=0.02)
    xr, xt = s.x_roll.to(DEV), s.x_train.to(DEV)
    cap = ops.mx8_capture_tiled(xr)
    got = {r: ops.mx8_fq_fwd_tiled(r, xt, cap) for r in RULES}
    torch.cuda.synchronize()
    xrb, xtb = inputs.bits(s.x_roll), inputs.bits(s.x_train)
    codes, mbits, scales = oracle_mod.mx8_capture(xrb)
    outs = {ops.TRACE_RULE_GUIDED: oracle_mod.mx8_guided_fwd(xtb, mbits, scales),
            ops.TRACE_RULE_RTN: oracle_mod.mx8_rtn_fwd(xtb, scales),
            ops.TRACE_RULE_FULL: oracle_mod.mx8_full_guided_fwd(xtb, codes, scales)}
    _eq("w4a8 codes", _u(cap.codes), codes)
    _eq("w4a8 mbits", _u(cap.mbits), mbits)
    _eq("w4a8 tiled scales", _u(cap.scales), oracle_mod.swizzle_scales(scales))
    for r in RULES:
        _eq(f"w4a8 out rule {r}", _u(got[r][0]), outs[r][0])
        _eq(f"w4a8 mask rule {r}", _u(got[r][1]), outs[r][1])


def test_validate_offsets():
    ok = torch.tensor([0, 0, 5, 5, 9], dtype=torch.int64, device=DEV)
    assert ops.validate_offsets(ok, 9) == 0
    assert ops.validate_offsets(torch.tensor([1, 5, 9], dtype=torch.int64, device=DEV), 9) == 1
    assert ops.validate_offsets(torch.tensor([0, 6, 5, 9], dtype=torch.int64, device=DEV), 9) == 3
    assert ops.validate_offsets(torch.tensor([0, 5, 8], dtype=torch.int64, device=DEV), 9) == 3
    assert ops.validate_offsets(torch.tensor([0, 12, 9], dtype=torch.int64, device=DEV), 9) == 2
    big = torch.arange(0, 100001, dtype=torch.int64, device=DEV)
    assert ops.validate_offsets(big, 100000) == 0
    big[77777] = big[77776] - 1
    assert ops.validate_offsets(big, 100000) == 77778


def test_debug_mode_rejects_bad_offsets(monkeypatch):
    monkeypatch.setattr(ops, "DEBUG", True)
    x = torch.zeros(9, 32, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ops.TraceError):
        ops.capture(x, torch.tensor([0, 6, 5, 9], dtype=torch.int64, device=DEV))
    cap = ops.capture(x, torch.tensor([0, 5, 9], dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
    assert cap.gscale.cpu().tolist() == [1.0, 1.0]
