"""Comparator modes of the refined decode GEMV (oracle; test infrastructure).

The rag-lover.com explainer of StrataFlux (既存手法との違い, differences from
existing methods) sets the method against fetching FP16 residual columns
inside the projection (DecDEC-like) and against choosing what to refine at
random (an ablation).  Both are run here as switches on the same GEMV; the
pages give no formula, so the plainest readings are taken:

R1  random selection: per step, the k channels with the largest keys
    key_j = (splitmix64(seed + K * step + j) >> 49) mod 32640, ties to the
    lower channel, listed ascending -- a uniform random k-subset up to key
    collisions, drawn from a counter-based generator so any step of any
    channel is reproducible on its own.  splitmix64 is the finalizer of
    Steele, Lea and Flood ("Fast splittable pseudorandom number
    generators", 2014): z += 0x9E3779B97F4A7C15; z = (z ^ z >> 30) *
    0xBF58476D1CE4E5B9; z = (z ^ z >> 27) * 0x94D049BB133111EB; z ^ z >> 31.
    The key is below 0x7F80, so it reads as a finite positive bf16 and the
    selection is the top-k selection of :mod:`oracle.select` on those keys.
F1  FP16 fetch: a selected column j uses w_res + r_j with the residual
    r = fp16_RNE(w - w_res) of the fp32 weight against its resident value
    (the difference is exact in fp64, so one rounding), instead of the
    refinement bits; other columns keep w_res.  y = x w_eff in fp64.
"""

from __future__ import annotations

import numpy as np

from .gemv import bf16_to_f64
from .quant import dequant_resident
from .select import select_topk

_M64 = (1 << 64) - 1


def splitmix64(z: int) -> int:
    """The splitmix64 output for state z (before the state's own increment
    is applied: the function adds the golden-ratio constant first)."""
    z = (z + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def random_keys(K: int, seed: int, step: int) -> np.ndarray:
    """R1: the 15-bit keys of channels 0..K-1 (as uint16, below 0x7F80)."""
    base = (seed + K * step) & _M64
    return np.array([(splitmix64((base + j) & _M64) >> 49) % 0x7F80 for j in range(K)], dtype=np.uint16)


def select_random(K: int, k: int, seed: int, step: int) -> np.ndarray:
    """R1: the ascending random selection of k channels."""
    return select_topk(random_keys(K, seed, step)[None, :], k)


def residual_fp16(W: np.ndarray, qz: dict) -> np.ndarray:
    """F1: fp16 residual of the fp32 weights against their resident values."""
    d = np.asarray(W, dtype=np.float32).astype(np.float64) - dequant_resident(qz)
    return d.astype(np.float16)


def gemv_fp16_fetch(qz: dict, W: np.ndarray, x_bits: np.ndarray, S) -> tuple[np.ndarray, np.ndarray]:
    """F1: (y fp64 [B][N], sum_j |w_eff x| fp64 [B][N])."""
    x = bf16_to_f64(np.atleast_2d(x_bits))
    w = dequant_resident(qz)
    S = np.asarray(S, dtype=np.int64)
    if S.size:
        w[:, S] += residual_fp16(W, qz)[:, S].astype(np.float64)
    return x @ w.T, np.abs(x) @ np.abs(w).T
