"""Workload shapes for the StrataFlux hot path, named by what they are.

Sizes follow the models and settings the StrataFlux abstract evaluates
(Llama-3.1-8B-Instruct and Qwen3-8B decode, 2-4-bit weights, 2-3-bit KV,
128K context).  Counts given as a percentage ("top 3% of channels", "a 10%
cache") are turned into integers by :func:`count_fraction`.
"""

from __future__ import annotations

from fractions import Fraction


def count_fraction(percent: Fraction | int | str, n: int) -> int:
    """floor(p * n + 1/2) for a percentage p, in exact rational arithmetic.

    5% of 512 -> 26, 3% of 4096 -> 123, 1% of 32768 -> 328, 10% of 14336 -> 1434.
    """
    p = Fraction(percent) / 100
    v = p * n + Fraction(1, 2)
    return v.numerator // v.denominator


# One decode linear layer at CPU-seconds scale: 512x512, group 64,
# 2-bit resident + 2-bit refinement, batch 1, 1% outlier channels x20,
# top-26 channels, refinement cache holding every column (preloaded).
LINEAR_512 = dict(
    name="linear_512",
    matrices={"w": (512, 512)},
    group=64, b_r=2, b_f=2, batch=1,
    outlier_percent=1, outlier_scale=20.0, outliers_fixed=True,
    topk_percent=5, cache_percent=100, preload_all=True,
)

# Llama-3.1-8B-shaped decode linear layers, 2-bit resident + 2-bit
# refinement, group 128, batch 1, 0.5% outlier channels x30 (a fixed set, so
# selections recur across steps), top 3% channels, LRU cache of 10% of the
# columns of each matrix, misses fetched from pinned host RAM one layer ahead.
LLAMA31_8B_LINEAR = dict(
    name="llama31_8b_linear",
    matrices={"q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
              "gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336)},
    layers=32, group=128, b_r=2, b_f=2, batch=1,
    outlier_percent=Fraction(1, 2), outlier_scale=30.0, outliers_fixed=True,
    topk_percent=3, cache_percent=10, preload_all=False,
)

# Qwen3-8B-shaped decode linear layers: 3-bit resident + 1-bit refinement,
# group 128, batch 1/4/16, top 5% channels per row (union over the batch),
# LRU cache of 25% of the columns.  Activations are plain N(0, 1).
QWEN3_8B_LINEAR = dict(
    name="qwen3_8b_linear",
    matrices={"q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
              "gate": (12288, 4096), "up": (12288, 4096), "down": (4096, 12288)},
    layers=36, group=128, b_r=3, b_f=1, batches=(1, 4, 16),
    outlier_percent=0, outlier_scale=1.0, outliers_fixed=True,
    topk_percent=5, cache_percent=25, preload_all=False,
)

# Decode attention at 32K context: 32 query heads, 8 KV heads, head_dim 128,
# batch 1; K/V N(0,1) with 4 outlier key channels per KV head x10, quantized
# per token-head (group 128) to 2-bit resident + 2-bit refinement; top 1% of
# tokens per query head refined in both K and V.
ATTN_32K = dict(
    name="attn_32k",
    n_tokens=32768, n_q_heads=32, n_kv_heads=8, head_dim=128,
    b_r=2, b_f=2, group=128, n_outlier_ch=4, outlier_scale=10.0,
    topk_percent=1, layers=32,
)

# Full decode step of a 32-layer Llama-3.1-8B-shaped model at 131072 tokens
# of context: 3-bit resident + 1-bit refinement weights, 2-bit + 2-bit KV.
LLAMA31_8B_DECODE_128K = dict(
    name="llama31_8b_decode_128k",
    layers=32, hidden=4096, mlp=14336, n_q_heads=32, n_kv_heads=8, head_dim=128,
    n_tokens=131072, w_bits=(3, 1), kv_bits=(2, 2), group=128,
)

WORKLOADS = {w["name"]: w for w in
             (LINEAR_512, LLAMA31_8B_LINEAR, QWEN3_8B_LINEAR, ATTN_32K, LLAMA31_8B_DECODE_128K)}
