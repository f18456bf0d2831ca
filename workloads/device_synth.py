"""Seeded synthetic tensors drawn directly on the GPU (torch Philox), for the
full-size benchmark where drawing billions of values with numpy would take
minutes.  Same recipes as :mod:`workloads.synth` (N(0, 0.02) weights, bf16
N(0, 1) activations with a fixed set of outlier channels, N(0, 1) K/V with
outlier key channels, bf16 N(0, 1) queries); different random streams, so
these are not bit-identical to the numpy draws.  No method arithmetic.
"""

from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weight(seed: int, n_out: int, n_in: int, device="cuda", std: float = 0.02) -> torch.Tensor:
    return torch.randn((n_out, n_in), generator=_gen(seed, device), device=device, dtype=torch.float32) * std


def outlier_channels(seed: int, n: int, count: int, device="cuda") -> torch.Tensor:
    return torch.randperm(n, generator=_gen(seed, device), device=device)[:count].sort().values


def activations(seed: int, batch: int, n_in: int, outliers: torch.Tensor | None, scale: float,
                device="cuda") -> torch.Tensor:
    x = torch.randn((batch, n_in), generator=_gen(seed, device), device=device, dtype=torch.float32)
    if outliers is not None and outliers.numel():
        x[:, outliers] *= scale
    return x.to(torch.bfloat16)


def kv(seed: int, n_kv_heads: int, n_tokens: int, head_dim: int, n_outlier_ch: int = 4,
       outlier_scale: float = 10.0, device="cuda") -> tuple[torch.Tensor, torch.Tensor]:
    """K, V as [n_kv_heads * n_tokens][head_dim] fp32 (rows = token-heads)."""
    g = _gen(seed, device)
    k = torch.randn((n_kv_heads, n_tokens, head_dim), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((n_kv_heads, n_tokens, head_dim), generator=g, device=device, dtype=torch.float32)
    for h in range(n_kv_heads):
        ch = torch.randperm(head_dim, generator=g, device=device)[:n_outlier_ch]
        k[h][:, ch] *= outlier_scale
    return k.reshape(-1, head_dim), v.reshape(-1, head_dim)


def query(seed: int, n_q_heads: int, head_dim: int, device="cuda") -> torch.Tensor:
    return torch.randn((n_q_heads, head_dim), generator=_gen(seed, device), device=device,
                       dtype=torch.float32).to(torch.bfloat16)
