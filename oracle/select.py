"""Top-k input-channel selection by |x| (oracle; test infrastructure).

StrataFlux chooses which weight refinements to fetch by the magnitude of the
input activations (rag-lover.com explainer, 解説 section).  Reading taken:

T1  the key of channel j in batch row b is |x[b][j]|, compared as exact bf16
    magnitudes (so +0 and -0 tie); NaN or Inf activations are rejected.
T2  order by key descending, then channel index ascending (ties go to the
    lower index); keep the first k.
T3  the selected set is the union over batch rows, listed in ascending
    order; every selected column is refined for every row of the batch.
"""

from __future__ import annotations

import numpy as np


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def topk_row(x_bits_row: np.ndarray, k: int) -> list[int]:
    """T1-T2 for one row of bf16 bit patterns: the k chosen channel indices,
    in rank order."""
    vals = _bf16_to_f64(x_bits_row)
    if not np.all(np.isfinite(vals)):
        raise ValueError("non-finite activation")
    K = len(vals)
    if not 0 <= k <= K:
        raise ValueError("k out of range")
    mag = [abs(float(v)) for v in vals]
    order = sorted(range(K), key=lambda j: (-mag[j], j))
    return order[:k]


def select_topk(x_bits: np.ndarray, k: int) -> np.ndarray:
    """T1-T3: x_bits [B][K] bf16 bit patterns -> ascending int32 union."""
    x_bits = np.atleast_2d(x_bits)
    chosen: set[int] = set()
    for b in range(x_bits.shape[0]):
        chosen.update(topk_row(x_bits[b], k))
    return np.array(sorted(chosen), dtype=np.int32)
