"""Seeded draws for every synthetic tensor the hot path consumes.

All draws use numpy's PCG64 (``numpy.random.default_rng``).  The recipes
follow the workloads described for StrataFlux ("StrataFlux:
Memory-Hierarchy-Native Low-Bit LLM Inference", abstract): random-init
weights N(0, 0.02), bf16 N(0, 1) activations with a small fixed set of
outlier channels, N(0, 1) keys/values with a few outlier key channels per
head, and bf16 N(0, 1) queries.  Real checkpoints and datasets are not used.
"""

from __future__ import annotations

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the
    16-bit patterns as uint16.  Inputs must be finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(seed: int, n_channels: int, count: int) -> np.ndarray:
    """A fixed, seeded set of ``count`` distinct channel indices in
    ``[0, n_channels)``, ascending."""
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n_channels, size=count, replace=False)).astype(np.int64)


def gen_weight(seed: int, n_out: int, n_in: int, std: float = 0.02) -> np.ndarray:
    """Random-init weight matrix W[n_out][n_in], fp32 N(0, std)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n_out, n_in), dtype=np.float32) * np.float32(std)).astype(np.float32)


def gen_activations(seed: int, batch: int, n_in: int, outliers: np.ndarray | None = None,
                    outlier_scale: float = 1.0) -> np.ndarray:
    """Decode activations x[batch][n_in] as bf16 bit patterns.

    Each value is drawn fp32 N(0, 1); channels listed in ``outliers`` are
    multiplied by ``outlier_scale`` in fp32; the result is rounded once to
    bf16.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, n_in), dtype=np.float32)
    if outliers is not None and len(outliers):
        x[:, outliers] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def gen_kv(seed: int, n_kv_heads: int, n_tokens: int, head_dim: int, n_outlier_ch: int = 4,
           outlier_scale: float = 10.0) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Keys and values [n_kv_heads][n_tokens][head_dim], fp32 N(0, 1).

    Per KV head, ``n_outlier_ch`` key channels (the same for every token of
    that head) are multiplied by ``outlier_scale``.  Returns (K, V, channels)
    with channels[h] the outlier channels of head h.
    """
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n_kv_heads, n_tokens, head_dim), dtype=np.float32)
    v = rng.standard_normal((n_kv_heads, n_tokens, head_dim), dtype=np.float32)
    ch = np.stack([np.sort(rng.choice(head_dim, size=n_outlier_ch, replace=False))
                   for _ in range(n_kv_heads)]) if n_outlier_ch else np.zeros((n_kv_heads, 0), np.int64)
    for h in range(n_kv_heads):
        k[h][:, ch[h]] *= np.float32(outlier_scale)
    return k, v, ch


def gen_query(seed: int, n_q_heads: int, head_dim: int) -> np.ndarray:
    """Decode query q[n_q_heads][head_dim] as bf16 bit patterns of N(0, 1)."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((n_q_heads, head_dim), dtype=np.float32))
