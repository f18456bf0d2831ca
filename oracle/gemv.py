"""Refined decode GEMV (oracle; test infrastructure).

StrataFlux refines the weight columns whose input activations are largest
(rag-lover.com explainer, 解説 section): a selected column uses the full
(resident + refinement) code, every other column its resident code.

G1  y[b][i] = sum_j x[b][j] * w_eff[i][j], w_eff = full value (Q5) for j in S
    and resident value otherwise; fp64 throughout, reported as fp32.
G2  this oracle does not factor scale and zero out of the sum.
G3  the GPU result is accepted when |y_gpu - y| <= 2e-3 * sum_j |w_eff x| per
    output; ``abs_sum`` returns that right-hand sum (without the factor).
"""

from __future__ import annotations

import numpy as np

from .quant import dequant_full, dequant_resident


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def effective_weights(qz: dict, S) -> np.ndarray:
    w = dequant_resident(qz)
    S = np.asarray(S, dtype=np.int64)
    if S.size:
        w[:, S] = dequant_full(qz)[:, S]
    return w


def gemv_refine(qz: dict, x_bits: np.ndarray, S) -> tuple[np.ndarray, np.ndarray]:
    """G1: returns (y fp64 [B][N], sum_j |w_eff[i][j] x[b][j]| fp64 [B][N])."""
    x = bf16_to_f64(np.atleast_2d(x_bits))
    w = effective_weights(qz, S)
    y = x @ w.T
    abs_sum = np.abs(x) @ np.abs(w).T
    return y, abs_sum
