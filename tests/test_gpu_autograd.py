"""The autograd wrapper: forward outputs and the masked straight-through
gradient, through torch.autograd, against the oracle for every format and
rule."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from fp4_quantization_aware_trace_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "w4a8"])
@pytest.mark.parametrize("rule", ["guided", "full", "rtn"])
def test_autograd_matches_oracle(oracle_mod, fmt, rule):
    s = inputs.tiny_site(91, 96, 256, eps=0.05)
    xr = s.x_roll.to(DEV)
    cache = {"nvfp4": ops.capture, "mxfp4": ops.mx_capture, "w4a8": ops.mx8_capture}[fmt](xr)
    x = s.x_train.to(DEV).requires_grad_(True)
    y = ops.trace_fake_quant(x, cache, fmt, rule)
    w = s.grad.to(DEV)
    (y.float() * w.float()).sum().backward()
    torch.cuda.synchronize()
    xrb, xtb, gb = inputs.bits(s.x_roll), inputs.bits(s.x_train), inputs.bits(s.grad)
    if fmt == "nvfp4":
        codes, mbits, scales, gscale = oracle_mod.capture(xrb)
        ref = {"guided": lambda: oracle_mod.guided_fwd(xtb, mbits, scales, gscale),
               "full": lambda: oracle_mod.full_guided_fwd(xtb, codes, scales, gscale),
               "rtn": lambda: oracle_mod.rtn_fwd(xtb, scales, gscale)}[rule]()
    else:
        cap = oracle_mod.mx_capture if fmt == "mxfp4" else oracle_mod.mx8_capture
        codes, mbits, scales = cap(xrb)
        pre = "mx" if fmt == "mxfp4" else "mx8"
        ref = {"guided": lambda: getattr(oracle_mod, f"{pre}_guided_fwd")(xtb, mbits, scales),
               "full": lambda: getattr(oracle_mod, f"{pre}_full_guided_fwd")(xtb, codes, scales),
               "rtn": lambda: getattr(oracle_mod, f"{pre}_rtn_fwd")(xtb, scales)}[rule]()
    out, mask = ref
    assert np.array_equal(_bits(y).reshape(-1), out.reshape(-1))
    # d(sum(y * w))/dy = w in bf16; the backward keeps it where |z| is in range
    gin = oracle_mod.fq_bwd(gb, mask)
    assert np.array_equal(_bits(x.grad).reshape(-1), gin.reshape(-1))
