"""Seeded synthetic inputs for tests and the benchmark.

This module holds no quantization arithmetic: it only draws random bf16
tensors with the shapes, value distributions and structure of the five
workloads below, and converts between torch bf16 tensors and their raw
16-bit patterns.  Both the CUDA parity tests and the CPU oracle consume
what it produces.

Workloads (the pages' own experiments use trained models and datasets that
are not available; these synthetic tensors stand in for them):

  activation_outliers  4096x2048, N(0,1), 0.1% of entries x50 (seed 0);
                       train-side copy x' = bf16(x + N(0, (1e-3|x|)^2)) (seed 1)
  layer_stack          40 layers of 65536x4096, 0.5 * Student-t(4) times a
                       per-channel LogNormal(0,1) scale (seed 100 + layer)
  moe_dispatch         32768 tokens, top-8 of 128 experts with Zipf(1.1)
                       expert popularity, hidden 2048, N(0,1) rows gathered
                       and grouped by expert (ragged, possibly empty groups)
  weights              8192x28672, N(0, 0.02^2) (seed 4)
  kv_cache             K and V of [131072 tokens, 8 heads, 128], N(0,1) with
                       4 outlier head_dim channels x20 (seed 5)

Every generator draws in fp32 on ``device`` with a seeded torch.Generator
and rounds once to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import math

import numpy as np
import torch

LAYER_STACK_LAYERS = 40
LAYER_STACK_DEEP = 20  # guidance kept for the deepest 20 of 40 layers


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 patterns of a bf16 tensor (copied to host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(bits: np.ndarray, device="cpu") -> torch.Tensor:
    """bf16 tensor with the given raw uint16 patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(device)


def perturb(x: torch.Tensor, seed: int, rel: float = 1e-3) -> torch.Tensor:
    """Train-side copy x' = bf16(x + eps * rel * |x|), eps ~ N(0, 1)."""
    g = _gen(seed, x.device)
    xf = x.float()
    eps = torch.randn(xf.shape, generator=g, device=x.device, dtype=torch.float32)
    return (xf + eps * rel * xf.abs()).to(torch.bfloat16)


def activation_outliers(device="cuda", rows=4096, cols=2048, seed=0, train_seed=1):
    g = _gen(seed, device)
    x = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    n = rows * cols
    k = int(math.floor(0.001 * n))
    idx = torch.randperm(n, generator=g, device=device)[:k]
    x.view(-1)[idx] *= 50.0
    xb = x.to(torch.bfloat16)
    return dict(x=xb, x_train=perturb(xb, train_seed))


def layer_stack_layer(layer: int, device="cuda", rows=65536, cols=4096, base_seed=100):
    """One layer of the activation stack: 0.5 * t_4 * c_j, c_j ~ LogNormal(0,1).

    Student-t(4) = z / sqrt(chi2_4 / 4) with chi2_4 = -2 ln(u1 u2)."""
    g = _gen(base_seed + layer, device)
    c = torch.exp(torch.randn((cols,), generator=g, device=device, dtype=torch.float32))
    z = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    u1 = torch.rand((rows, cols), generator=g, device=device, dtype=torch.float32)
    u2 = torch.rand((rows, cols), generator=g, device=device, dtype=torch.float32)
    chi2 = -2.0 * (torch.log1p(-u1) + torch.log1p(-u2))  # u in [0,1): 1-u in (0,1]
    t4 = z * torch.rsqrt(chi2 / 4.0)
    del u1, u2, chi2, z
    return (0.5 * t4 * c).to(torch.bfloat16)


def moe_dispatch(device="cuda", tokens=32768, experts=128, topk=8, hidden=2048, seed=3,
                 zipf_s=1.1, train_seed=1):
    """Expert inputs grouped by expert: returns x [tokens*topk, hidden] bf16,
    seg_off (np.int64, experts+1 row offsets) and the train-side copy."""
    g = _gen(seed, device)
    p = torch.arange(1, experts + 1, device=device, dtype=torch.float64).pow(-zipf_s)
    p = (p / p.sum()).float()
    choice = torch.multinomial(p.expand(tokens, experts), topk, replacement=False, generator=g)
    h = torch.randn((tokens, hidden), generator=g, device=device, dtype=torch.float32)
    expert = choice.reshape(-1)
    token = torch.arange(tokens, device=device).repeat_interleave(topk)
    order = torch.sort(expert, stable=True).indices
    x = h[token[order]].to(torch.bfloat16)
    counts = torch.bincount(expert, minlength=experts).cpu().numpy().astype(np.int64)
    seg_off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return dict(x=x, seg_off=seg_off, x_train=perturb(x, train_seed))


def weights(device="cuda", rows=8192, cols=28672, seed=4, std=0.02):
    g = _gen(seed, device)
    return (std * torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)).to(
        torch.bfloat16)


def kv_cache(device="cuda", tokens=131072, heads=8, head_dim=128, seed=5, n_outlier=4,
             outlier_scale=20.0, train_seed=1):
    """K and V [tokens, heads, head_dim] viewed as [tokens*heads, head_dim]."""
    g = _gen(seed, device)
    ch = torch.randperm(head_dim, generator=g, device=device)[:n_outlier]
    out = {}
    for name in ("k", "v"):
        t = torch.randn((tokens, heads, head_dim), generator=g, device=device, dtype=torch.float32)
        t[:, :, ch] *= outlier_scale
        out[name] = t.to(torch.bfloat16).reshape(tokens * heads, head_dim)
    out["k_train"] = perturb(out["k"], train_seed)
    out["v_train"] = perturb(out["v"], train_seed + 1)
    out["outlier_channels"] = ch.cpu().numpy()
    return out


def random_bf16(shape, seed=0, device="cpu", scale=1.0, outlier_frac=0.0, outlier_mult=50.0):
    """Small generic case for tests: N(0, scale^2) with optional outliers."""
    g = _gen(seed, device)
    x = scale * torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if outlier_frac > 0:
        n = x.numel()
        k = max(1, int(outlier_frac * n))
        idx = torch.randperm(n, generator=g, device=device)[:k]
        x.view(-1)[idx] *= outlier_mult
    return x.to(torch.bfloat16)
