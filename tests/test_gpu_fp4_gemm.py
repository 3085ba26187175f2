"""What capture writes is what a block-scaled FP4 GEMM consumes.

An activation A [M, K] and a weight W [N, K] are captured with the scales in
the 128 x 4 tiled layout (trace_capture_ex); their packed E2M1 codes, tiled
E4M3 block scales and the product of their global scales (as the GEMM's
alpha) go, unchanged, into vLLM's CUTLASS NVFP4 GEMM (a library kernel,
used here only as the consumer to check against, on this GPU's own memory).
Its bf16 output must equal the product of the dequantised operands
A_q W_q^T, computed in float64 from the oracle's capture of the same
inputs, within the error of the GEMM's arithmetic:

  * every product of two dequantised elements is exact in fp32 (2 x 4
    significant bits per factor), so the only roundings are the fp32
    accumulation over K (at most K * 2^-24 * sum |a_k w_k|), alpha = s_gA
    s_gW rounded to fp32 (2^-24 relative) and the final bf16 rounding (2^-9
    relative);
  * bound used: |out - ref| <= 2^-8 |ref| + K 2^-24 sum_k |a_k w_k|.

A negative control feeds the same GEMM the row-major scales instead of the
tiled ones and must fail the bound (the layout is what is being shown)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

M, N, K = 256, 384, 1024


def _vllm_fp4_mm():
    try:
        import vllm._custom_ops as vops
    except Exception as exc:  # the checker itself is missing: say so loudly
        pytest.fail(f"vLLM's custom ops are not importable: {exc!r}")
    cap = torch.cuda.get_device_capability()
    if not vops.cutlass_scaled_mm_supports_fp4(cap[0] * 10 + cap[1]):
        pytest.fail(f"vLLM's NVFP4 GEMM does not support sm_{cap[0]}{cap[1]}")
    return vops.cutlass_scaled_fp4_mm


def _dequant(oracle_mod, codes, scales, gscale, rows, cols):
    """float64 [rows, cols] = E2M1 value * E4M3 block scale * global scale,
    every factor decoded by the oracle (its bf16 dequant of a code at unit
    scales is the exact codeword; E4M3 bytes decode exactly)."""
    e2m1 = np.array([float(np.array([oracle_mod.dequant_bf16(c & 7, bool(c & 8), 1.0, 1.0) << 16],
                                    np.uint32).view(np.float32)[0]) for c in range(16)])
    e4m3 = np.array([oracle_mod.e4m3_to_f32(b) for b in range(256)], np.float64)
    c = np.asarray(codes, np.uint8).reshape(rows, cols // 2)
    nib = np.empty((rows, cols), np.uint8)
    nib[:, 0::2] = c & 0xF
    nib[:, 1::2] = c >> 4
    sb = e4m3[np.asarray(scales, np.uint8).reshape(rows, cols // 16)]
    return e2m1[nib] * np.repeat(sb, 16, axis=1) * float(gscale[0])


def _operands():
    a = inputs.tiny_site(9001, M, K).x_roll.cuda()
    g = torch.Generator(device="cpu")
    g.manual_seed(9002)
    w = torch.randn(N, K, generator=g) * 0.05
    w[:, torch.randperm(K, generator=g)[:16]] *= 20.0
    return a, w.to(torch.bfloat16).cuda()


def _tiled_fp8(cap, rows, cols):
    return cap.scales.view(torch.float8_e4m3fn).view((rows + 127) // 128 * 128,
                                                     (cols // 16 + 3) // 4 * 4)


def test_capture_output_feeds_block_scaled_fp4_gemm(oracle_mod):
    fp4_mm = _vllm_fp4_mm()
    a, w = _operands()
    ca, cw = ops.capture_tiled(a), ops.capture_tiled(w)
    alpha = (ca.gscale * cw.gscale).to(torch.float32).reshape(1)
    out = fp4_mm(ca.codes.view(M, K // 2), cw.codes.view(N, K // 2), _tiled_fp8(ca, M, K),
                 _tiled_fp8(cw, N, K), alpha, torch.bfloat16)
    torch.cuda.synchronize()
    # the reference operands come from the oracle's capture of the same inputs
    # (the library's codes and tiled scales equal it: checked here too)
    ra = oracle_mod.capture(inputs.bits(a.cpu()))
    rw = oracle_mod.capture(inputs.bits(w.cpu()))
    assert np.array_equal(ca.codes.cpu().numpy(), ra[0])
    assert np.array_equal(cw.codes.cpu().numpy(), rw[0])
    assert np.array_equal(ca.scales.cpu().numpy(), oracle_mod.swizzle_scales(ra[2]).reshape(-1))
    assert np.array_equal(cw.scales.cpu().numpy(), oracle_mod.swizzle_scales(rw[2]).reshape(-1))
    da = _dequant(oracle_mod, ra[0], ra[2], ra[3], M, K)
    dw = _dequant(oracle_mod, rw[0], rw[2], rw[3], N, K)
    ref = da @ dw.T
    mag = np.abs(da) @ np.abs(dw).T
    got = out.float().cpu().numpy().astype(np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -24 * mag
    err = np.abs(got - ref)
    assert np.all(err <= bound), (f"{int(np.sum(err > bound))} of {err.size} outputs outside "
                                  f"the bound; worst excess {float(np.max(err - bound))}")
    assert np.count_nonzero(ref) > 0.99 * ref.size  # a real product, not zeros


def test_row_major_scales_do_not_fit_the_gemm(oracle_mod):
    """Negative control: the same codes with the scales left row-major (the
    layout trace_capture writes) give a different product."""
    fp4_mm = _vllm_fp4_mm()
    a, w = _operands()
    ca, cw = ops.capture(a), ops.capture(w)
    ta, tw = ops.capture_tiled(a), ops.capture_tiled(w)
    # the row-major bytes, padded to the tiled buffer's size
    sa = torch.zeros_like(ta.scales)
    sw = torch.zeros_like(tw.scales)
    sa[:ca.scales.numel()] = ca.scales.reshape(-1)
    sw[:cw.scales.numel()] = cw.scales.reshape(-1)
    alpha = (ca.gscale * cw.gscale).to(torch.float32).reshape(1)
    ta.scales, tw.scales = sa, sw
    bad = fp4_mm(ca.codes.view(M, K // 2), cw.codes.view(N, K // 2), _tiled_fp8(ta, M, K),
                 _tiled_fp8(tw, N, K), alpha, torch.bfloat16)
    torch.cuda.synchronize()
    ra = oracle_mod.capture(inputs.bits(a.cpu()))
    rw = oracle_mod.capture(inputs.bits(w.cpu()))
    ref = _dequant(oracle_mod, ra[0], ra[2], ra[3], M, K) @ \
        _dequant(oracle_mod, rw[0], rw[2], rw[3], N, K).T
    err = np.abs(bad.float().cpu().numpy() - ref)
    assert np.mean(err > 2.0 ** -6 * np.abs(ref)) > 0.5
