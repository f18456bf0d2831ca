"""Refined decode attention over low-bit K/V (oracle; test infrastructure).

StrataFlux keeps a 2-3-bit KV cache resident (arXiv 2611.08363 abstract) and
refines the tokens that the low-bit keys say carry the most attention weight
(rag-lover.com explainer, 解説 section).  Reading taken:

A1  grouped-query attention: query head h reads KV head h // (Hq / Hkv).
A2  resident score s[h][t] = q_h . k_res_t / sqrt(d), fp64.
A3  selection key kappa[h][t] = fp64(scale_t * E[h][t]) with
    E[h][t] = sum_d q[h][d] * (c[t][d] 2^b_f + m_f - zero_t), c the resident
    key code.  Every product carries few significant bits, so E is exact in
    fp64 whatever the summation order, provided the exponents of the nonzero
    query entries of a head span at most 53 - 9 - b - ceil(log2 d) binades;
    :func:`check_exact_span` enforces that.  kappa orders tokens exactly as
    the resident scores do, and so as the softmax weights.
A4  per query head keep the k tokens of largest kappa (ties: lower token
    index); U_g = union over the query heads of KV group g.  A refined token
    is refined for every head that reads it.
A5  k'_t, v'_t are full-code values (Q5) for t in U_g and resident values
    otherwise; s'[h][t] = q_h . k'_t / sqrt(d); o_h = sum_t softmax(s'_h)_t v'_t
    in fp64, reported as fp32.
A6  the GPU output is accepted within 2e-3 max-abs.
A7  refinement bits held in a cache (the deadline reading of a KV
    refinement cache): only the union tokens whose bits are on the device
    when the step starts are refined, E_g = U_g ∩ available_g; the others
    keep resident K and V this step (a miss keeps resident precision:
    rag-lover.com explainer, 限界と未検証の範囲) and are fetched for later
    steps.  The selection and the reported union do not change.
"""

from __future__ import annotations

import math

import numpy as np

from .quant import dequant_full, dequant_resident


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def check_exact_span(q: np.ndarray, b: int, d: int) -> None:
    """Raise if some head's nonzero query entries span too many binades for
    E to be exact in fp64 (see A3)."""
    limit = 53 - 9 - b - math.ceil(math.log2(d))
    for h in range(q.shape[0]):
        nz = q[h][q[h] != 0]
        if nz.size == 0:
            continue
        _, e = np.frexp(nz)
        if int(e.max()) - int(e.min()) > limit:
            raise ValueError(f"query head {h}: exponent span exceeds {limit}")


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Plain softmax attention of one query vector over k[T][d], v[T][d], fp64."""
    s = (k @ q) / math.sqrt(q.shape[0])
    m = s.max()
    p = np.exp(s - m)
    return (p @ v) / p.sum()


def selection_keys(qh: np.ndarray, qzk: dict, rows: slice) -> np.ndarray:
    """A3 keys of one query head (fp64 vector qh) against the token-heads in
    ``rows`` of the quantized key matrix."""
    b_f = qzk["b_f"]
    m_f = (2 ** b_f - 1) / 2.0
    c = qzk["q_r"][rows].astype(np.float64)
    z = qzk["zero"][0, rows].astype(np.float64)
    s = qzk["scale"][0, rows].astype(np.float64)
    A = c * 2 ** b_f + m_f - z[:, None]
    E = A @ qh
    return s * E


def topk_tokens(kappa: np.ndarray, k: int) -> np.ndarray:
    """A4 per head: the k token indices of largest kappa, ties to the lower
    index, returned ascending."""
    T = kappa.shape[0]
    order = np.lexsort((np.arange(T), -kappa))
    return np.sort(order[:k]).astype(np.int32)


def attn_decode_refine(q_bits: np.ndarray, qzk: dict, qzv: dict, Hkv: int, T: int, k_tokens: int,
                       refine: bool = True, available: np.ndarray | None = None) -> dict:
    """A1-A5 (A7 when ``available``, bool [Hkv][T], is given).  q_bits
    [Hq][d] bf16 patterns; qzk / qzv quantized K and V with rows =
    token-heads ordered [Hkv][T] and groups of the full head dim.

    Returns dict(out fp64 [Hq][d], sel list of per-head ascending token
    arrays, union list of per-KV-head ascending token arrays, refined list
    of per-KV-head ascending arrays of the tokens actually refined)."""
    q = bf16_to_f64(q_bits)
    Hq, d = q.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    grp = Hq // Hkv
    check_exact_span(q, qzk["b_r"] + qzk["b_f"], d)
    k_res = dequant_resident(qzk)
    v_res = dequant_resident(qzv)
    k_full = dequant_full(qzk) if refine else None
    v_full = dequant_full(qzv) if refine else None
    out = np.zeros((Hq, d))
    sel, union, refined = [], [], []
    for g in range(Hkv):
        rows = slice(g * T, (g + 1) * T)
        heads = range(g * grp, (g + 1) * grp)
        picked: set[int] = set()
        for h in heads:
            if refine and k_tokens > 0:
                st = topk_tokens(selection_keys(q[h], qzk, rows), k_tokens)
            else:
                st = np.zeros(0, np.int32)
            sel.append(st)
            picked.update(int(t) for t in st)
        U = np.array(sorted(picked), dtype=np.int64)
        union.append(U.astype(np.int32))
        E = U if available is None else U[np.asarray(available[g], dtype=bool)[U]]   # A7
        refined.append(E.astype(np.int32))
        kk = k_res[rows].copy()
        vv = v_res[rows].copy()
        if E.size:
            kk[E] = k_full[rows][E]
            vv[E] = v_full[rows][E]
        for h in heads:
            out[h] = attend(q[h], kk, vv)
    return dict(out=out, sel=sel, union=union, refined=refined)
