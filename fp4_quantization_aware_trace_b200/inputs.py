"""Seeded synthetic activations for the capture / guided fake-quant path.

This module only draws random numbers: it holds none of the quantisation
arithmetic, and both the CUDA path and the CPU oracle take their inputs from
it.  Every generator returns bf16 tensors (x_roll, x_train, grad) on the
requested device; the recipe of each workload is in its docstring.

The noise model follows the TRACE post's rounding-boundary discussion: the
training-side activation is the rollout activation plus a small relative
perturbation, x_train = bf16(x_roll + eps * |x_roll| * n), n ~ N(0,1), so a
share of the sites straddle codeword midpoints while most are bit-equal.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass
class Site:
    """One capture site: the rollout activation, its paired training-side
    activation, an upstream gradient, and the row offsets of its groups
    (None for a single group)."""
    name: str
    x_roll: torch.Tensor
    x_train: torch.Tensor
    grad: torch.Tensor
    offsets: torch.Tensor | None = None

    @property
    def num_groups(self) -> int:
        return 1 if self.offsets is None else int(self.offsets.numel()) - 1


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _perturb(x: torch.Tensor, eps: float, g: torch.Generator) -> torch.Tensor:
    xf = x.float()
    n = torch.randn(xf.shape, generator=g, device=xf.device, dtype=torch.float32)
    return (xf + eps * xf.abs() * n).to(torch.bfloat16)


def _grad(shape, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def single_activation(seed: int = 0, rows: int = 256, cols: int = 2048,
                      n_outlier: int = 8, outlier_scale: float = 50.0,
                      eps: float = 0.01, device="cpu") -> Site:
    """Single activation [256, 2048]: N(0,1) with 8 random outlier channels
    scaled x50; x_train = x_roll + N(0, (0.01|x_roll|)^2); grad N(0,1)."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    ch = torch.randperm(cols, generator=g, device=device)[:n_outlier]
    x[:, ch] *= outlier_scale
    xr = x.to(torch.bfloat16)
    return Site("single", xr, _perturb(xr, eps, g), _grad((rows, cols), g, device))


def lognormal_site(seed: int, rows: int, cols: int, outlier_frac: float = 0.01,
                   outlier_scale: float = 100.0, sigma: float = 1.0, eps: float = 0.005,
                   device="cpu", name: str = "site") -> Site:
    """Attention-input-like site: N(0,1) x per-channel lognormal scale
    exp(N(0, sigma^2)), with round(outlier_frac * cols) outlier channels
    scaled x outlier_scale; relative training noise eps."""
    g = _gen(seed, device)
    ch_scale = torch.exp(sigma * torch.randn(cols, generator=g, device=device))
    n_out = max(1, int(round(outlier_frac * cols)))
    ch = torch.randperm(cols, generator=g, device=device)[:n_out]
    ch_scale[ch] *= outlier_scale
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    x *= ch_scale
    xr = x.to(torch.bfloat16)
    return Site(name, xr, _perturb(xr, eps, g), _grad((rows, cols), g, device))


def attention_input(seed: int = 1, rows: int = 16384, cols: int = 2048, device="cpu") -> Site:
    """Qwen3-30B-A3B-shaped attention-input site [16384 tokens, 2048]:
    lognormal per-channel scales (sigma 1) x N(0,1), 1% outlier channels
    x100, relative noise 0.5%."""
    return lognormal_site(seed, rows, cols, device=device, name="attn_in")


def moe_experts(seed: int = 2, experts: int = 128, tokens: int = 512, cols: int = 2048,
                eps: float = 0.005, device="cpu", name: str = "expert_up_in") -> Site:
    """Routed-expert input for `experts` experts x `tokens` tokens each, as
    one [experts*tokens, cols] tensor with uniform group offsets: per-expert
    lognormal channel scales, a per-expert factor exp(N(0,1)), 1% outlier
    channels x100 per expert, relative noise eps."""
    g = _gen(seed, device)
    rows = experts * tokens
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    x = x.view(experts, tokens, cols)
    ch_scale = torch.exp(torch.randn(experts, 1, cols, generator=g, device=device))
    factor = torch.exp(torch.randn(experts, 1, 1, generator=g, device=device))
    n_out = max(1, int(round(0.01 * cols)))
    for e in range(experts):
        ch = torch.randperm(cols, generator=g, device=device)[:n_out]
        ch_scale[e, 0, ch] *= 100.0
    x = (x * ch_scale * factor).view(rows, cols)
    xr = x.to(torch.bfloat16)
    offs = torch.arange(0, rows + 1, tokens, dtype=torch.int64, device=device)
    return Site(name, xr, _perturb(xr, eps, g), _grad((rows, cols), g, device), offs)


def kv_cache(seed: int = 3, tokens: int = 32768, heads: int = 4, head_dim: int = 128,
             eps: float = 0.005, device="cpu", which: str = "k") -> Site:
    """FP4 KV-cache site: [tokens, heads, head_dim] viewed as
    [tokens*heads, head_dim] (16-element blocks run along head_dim).  Pairs
    (2i, 2i+1) of N(0,1) x per-(head, dim) lognormal scale, rotated by the
    angle t * 10000^(-2i/head_dim) (RoPE-like); 2 outlier dims per head x20."""
    g = _gen(seed + (0 if which == "k" else 7919), device)
    x = torch.randn(tokens, heads, head_dim, generator=g, device=device)
    scale = torch.exp(torch.randn(heads, head_dim, generator=g, device=device))
    for h in range(heads):
        dims = torch.randperm(head_dim, generator=g, device=device)[:2]
        scale[h, dims] *= 20.0
    x = x * scale
    i = torch.arange(head_dim // 2, device=device, dtype=torch.float32)
    inv = torch.pow(torch.tensor(10000.0, device=device), -2.0 * i / head_dim)
    t = torch.arange(tokens, device=device, dtype=torch.float32)
    ang = t[:, None] * inv[None, :]                      # [tokens, head_dim/2]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    y = torch.empty_like(x)
    y[..., 0::2] = a * c - b * s
    y[..., 1::2] = a * s + b * c
    xr = y.reshape(tokens * heads, head_dim).to(torch.bfloat16)
    return Site(f"kv_{which}", xr, _perturb(xr, eps, g),
                _grad((tokens * heads, head_dim), g, device))


LAYER_SWEEP_SITES = ("qkv_in", "o_in", "up_in", "down_in")


def layer_sweep_site(layer: int, site: int, rows: int = 65536, cols: int = 4096,
                     device="cpu", seed_offset: int = 0) -> Site:
    """One site of the later-half-layer sweep (layers 20..39 of 40, four
    sites per layer, each [65536, 4096]): as the attention-input recipe,
    seeded per (layer, site); seed_offset gives another draw of the same
    recipe (one per rank of a multi-GPU run)."""
    assert 0 <= site < len(LAYER_SWEEP_SITES)
    return lognormal_site(1000 + 4 * layer + site + seed_offset, rows, cols, device=device,
                          name=f"L{layer}_{LAYER_SWEEP_SITES[site]}")


def tiny_site(seed: int, rows: int, cols: int, device="cpu", eps: float = 0.01,
              outliers: bool = True) -> Site:
    """Small mixed-scale site for oracle / brute-force cases."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device)
    x *= torch.exp(torch.randn(1, cols, generator=g, device=device))
    if outliers:
        ch = torch.randperm(cols, generator=g, device=device)[: max(1, cols // 32)]
        x[:, ch] *= 30.0
    xr = x.to(torch.bfloat16)
    return Site("tiny", xr, _perturb(xr, eps, g), _grad((rows, cols), g, device))


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit array (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bit array -> bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def numel_gb(n: int) -> float:
    return n * 2 / 1e9


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("math", "torch", "dataclasses")]
