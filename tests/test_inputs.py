"""The seeded synthetic workloads follow their stated recipes (shapes,
determinism, relative drift of the training side, outlier channels, group
offsets); small sizes on the CPU."""
from __future__ import annotations

import numpy as np
import torch

from fp4_quantization_aware_trace_b200 import inputs


def _rel_drift(s):
    xr, xt = s.x_roll.float(), s.x_train.float()
    nz = xr != 0
    return ((xt - xr)[nz] / xr[nz].abs()).std().item()


def test_same_seed_same_tensors():
    a = inputs.attention_input(seed=7, rows=64, cols=256)
    b = inputs.attention_input(seed=7, rows=64, cols=256)
    c = inputs.attention_input(seed=8, rows=64, cols=256)
    for k in ("x_roll", "x_train", "grad"):
        assert torch.equal(getattr(a, k).view(torch.int16), getattr(b, k).view(torch.int16))
    assert not torch.equal(a.x_roll.view(torch.int16), c.x_roll.view(torch.int16))


def test_shapes_and_dtypes():
    s = inputs.single_activation(0)
    assert s.x_roll.shape == (256, 2048) and s.x_roll.dtype == torch.bfloat16
    s = inputs.attention_input(rows=128)
    assert s.x_roll.shape == (128, 2048) and s.grad.shape == (128, 2048)
    s = inputs.kv_cache(tokens=64, which="v")
    assert s.x_roll.shape == (64 * 4, 128)
    s = inputs.layer_sweep_site(20, 1, rows=32)
    assert s.x_roll.shape == (32, 4096)


def test_training_side_drift():
    """x_train = bf16(x_roll + eps |x_roll| n): the relative drift has the
    stated standard deviation (bf16 rounding adds a little), and a share of
    the sites stay bit-equal."""
    for s, eps in ((inputs.attention_input(rows=256), 0.005), (inputs.single_activation(0), 0.01)):
        d = _rel_drift(s)
        assert 0.8 * eps < d < 1.4 * eps, (s.name, d)
        same = (s.x_roll.view(torch.int16) == s.x_train.view(torch.int16)).float().mean().item()
        assert 0.05 < same < 0.95


def test_outlier_channels():
    """single activation: 8 channels x50; attention input: 1% of the channels
    x100 on top of lognormal channel scales."""
    s = inputs.single_activation(0)
    ch_rms = s.x_roll.float().pow(2).mean(0).sqrt()
    assert int((ch_rms > 20).sum()) == 8
    s = inputs.attention_input(rows=512)
    ch_rms = s.x_roll.float().pow(2).mean(0).sqrt().numpy()
    top = np.sort(ch_rms)[::-1]
    n_out = round(0.01 * 2048)
    assert top[n_out - 1] > 8 * np.median(ch_rms) and top[n_out + 5] < top[n_out - 1]


def test_moe_groups():
    s = inputs.moe_experts(experts=6, tokens=10, cols=256)
    assert s.num_groups == 6 and s.offsets.tolist() == list(range(0, 61, 10))
    # experts differ in scale (per-expert factor)
    rms = [s.x_roll[a:a + 10].float().pow(2).mean().sqrt().item() for a in range(0, 60, 10)]
    assert max(rms) / min(rms) > 1.5
