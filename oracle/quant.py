"""Nested quantization, packing and dequantization (oracle; test infrastructure).

StrataFlux keeps a low-bit code resident on the GPU and fetches extra
low-order bits that subdivide between resident levels ("nested
refinement"; rag-lover.com explainer, 解説 section; arXiv 2611.08363
abstract: 2-4-bit weights, 2-3-bit KV).  The pages give no quantizer
formula, so this module takes the plainest reading and states it:

Q1  per row r and group g of G consecutive inputs: lo = min, hi = max (fp32).
Q2  s = fp16_RNE(fp32((hi - lo) / (2^b - 1))) with IEEE fp32 subtraction and
    division; a quotient above 65504 is first clamped to 65504 (the largest
    finite fp16); if s rounds to 0, s = 1.  s_f = float(s).
Q3  z = clamp(rint(-lo / s_f), 0, 2^b - 1) with fp32 division and
    round-half-to-even; z is an integer, stored as fp16 (zero as +0).
Q4  q = clamp(rint(w / s_f) + z, 0, 2^b - 1); resident code q_r = q >> b_f,
    refinement code q_f = q & (2^b_f - 1).
Q5  full value s_f (q - z); resident value s_f (q_r 2^b_f + m_f - z) with
    m_f = (2^b_f - 1) / 2, the midpoint of the refinement interval; their
    difference is s_f (q_f - m_f).
Q6  packing: little-endian bitstreams in uint32 words.  Resident codes are
    row-major: row r holds code j at stream bits [b_r j, b_r j + b_r).
    Weight refinement codes are column-major ([K][N b_f / 32]); KV refinement
    codes are row-major like the resident codes.  Scale and zero are
    [K / G][N] fp16.
"""

from __future__ import annotations

import numpy as np

FP16_MAX = np.float32(65504.0)


def quantize_nested(W: np.ndarray, G: int, b_r: int, b_f: int) -> dict:
    """Quantize W[N][K] (fp32) per Q1-Q4.  Returns full codes ``q`` [N][K]
    (uint8), ``q_r``, ``q_f`` and fp16 ``scale``/``zero`` [K/G][N]."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if K % G:
        raise ValueError("K must be a multiple of G")
    b = b_r + b_f
    qmax = np.float32(2 ** b - 1)
    q = np.empty((N, K), dtype=np.uint8)
    scale = np.empty((K // G, N), dtype=np.float16)
    zero = np.empty((K // G, N), dtype=np.float16)
    for g in range(K // G):
        Wg = W[:, g * G:(g + 1) * G]
        lo = Wg.min(axis=1)                                   # Q1
        hi = Wg.max(axis=1)
        span = (hi - lo).astype(np.float32)                   # fp32 subtraction
        s32 = (span / qmax).astype(np.float32)                # Q2: fp32 division
        s32 = np.minimum(s32, FP16_MAX)
        s16 = s32.astype(np.float16)                          # RNE to fp16
        s16[s16 == 0] = np.float16(1.0)
        sf = s16.astype(np.float32)
        z = np.clip(np.rint((-lo / sf).astype(np.float32)), 0, qmax)          # Q3
        z = z + np.float32(0.0)          # an integer: store 0 as +0, never -0
        qg = np.clip(np.rint((Wg / sf[:, None]).astype(np.float32)) + z[:, None], 0, qmax)  # Q4
        q[:, g * G:(g + 1) * G] = qg.astype(np.uint8)
        scale[g] = s16
        zero[g] = z.astype(np.float16)
    return dict(q=q, q_r=(q >> b_f).astype(np.uint8), q_f=(q & ((1 << b_f) - 1)).astype(np.uint8),
                scale=scale, zero=zero, G=G, b_r=b_r, b_f=b_f)


def pack_bits(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes[R][C] (each < 2^bits) into little-endian bitstreams, one per
    row: code j occupies stream bits [bits*j, bits*j + bits); stream bit t is
    bit (t mod 32) of word t // 32.  Returns uint32 [R][C*bits/32]."""
    codes = np.ascontiguousarray(codes).astype(np.uint32)
    R, C = codes.shape
    if (C * bits) % 32:
        raise ValueError("row length in bits must be a multiple of 32")
    stream = np.zeros((R, C * bits), dtype=np.uint32)
    for b in range(bits):
        stream[:, b::bits] = (codes >> np.uint32(b)) & np.uint32(1)
    W = C * bits // 32
    stream = stream.reshape(R, W, 32)
    words = np.zeros((R, W), dtype=np.uint32)
    for t in range(32):
        words |= stream[:, :, t] << np.uint32(t)
    return words


def unpack_bits(words: np.ndarray, C: int, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_bits`: uint32 [R][C*bits/32] -> codes [R][C]."""
    words = np.ascontiguousarray(words, dtype=np.uint32)
    R, W = words.shape
    if W * 32 != C * bits:
        raise ValueError("word count does not match C*bits/32")
    stream = np.zeros((R, W, 32), dtype=np.uint32)
    for t in range(32):
        stream[:, :, t] = (words >> np.uint32(t)) & np.uint32(1)
    stream = stream.reshape(R, C * bits)
    codes = np.zeros((R, C), dtype=np.uint32)
    for b in range(bits):
        codes |= stream[:, b::bits] << np.uint32(b)
    return codes.astype(np.uint8)


def pack_nested(qz: dict, layout: str) -> dict:
    """Canonical packed form (Q6).  ``layout`` is "by_column" (weights:
    refinement [K][N b_f/32]) or "by_row" (KV: refinement [N][K b_f/32])."""
    res = pack_bits(qz["q_r"], qz["b_r"])
    if layout == "by_column":
        ref = pack_bits(qz["q_f"].T, qz["b_f"])
    elif layout == "by_row":
        ref = pack_bits(qz["q_f"], qz["b_f"])
    else:
        raise ValueError(layout)
    return dict(res=res, ref=ref, scale=qz["scale"], zero=qz["zero"])


def _expand_groups(a: np.ndarray, G: int) -> np.ndarray:
    """[K/G][N] per-group parameter -> [N][K] fp64, one value per weight."""
    return np.repeat(a.astype(np.float64).T, G, axis=1)


def dequant_full(qz: dict) -> np.ndarray:
    """Q5 full-code value s (q - z), fp64 [N][K]."""
    s = _expand_groups(qz["scale"], qz["G"])
    z = _expand_groups(qz["zero"], qz["G"])
    return s * (qz["q"].astype(np.float64) - z)


def dequant_resident(qz: dict) -> np.ndarray:
    """Q5 resident value s (q_r 2^b_f + m_f - z), fp64 [N][K]."""
    s = _expand_groups(qz["scale"], qz["G"])
    z = _expand_groups(qz["zero"], qz["G"])
    m_f = (2 ** qz["b_f"] - 1) / 2.0
    return s * (qz["q_r"].astype(np.float64) * 2 ** qz["b_f"] + m_f - z)
