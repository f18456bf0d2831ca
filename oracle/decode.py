"""One full decode step of a Llama-shaped model with nested-refined weights
and KV cache (oracle; test infrastructure).

The pages measure the method end to end on a decode step of a Llama-3.1-8B
sized model at 128K context (arXiv 2611.08363 abstract: tokens/s and GPU
memory at 128K).  The benchmark configuration names the shape: hidden 4096,
MLP 14336, 32 query / 8 KV heads, head dim 128, RMSNorm, RoPE, 3-bit
resident + 1-bit refinement weights, 2+2-bit KV, random-init weights.  The
pages give no formula for the model itself; the plainest reading of
"Llama-3.1-8B-shaped" is taken:

D1  RMSNorm: y = x / sqrt(mean(x^2) + eps) * w, eps = 1e-5, fp64.
D2  RoPE with base theta = 500000 over head dim d: for i < d/2, dims i and
    i + d/2 of a head rotate by the angle pos * theta^(-2i/d) (rotate-half
    pairing); no frequency rescaling.
D3  a layer: n1 = RMSNorm(x); q, k, v = refined GEMVs of n1 (G1); q and k
    rotated (D2) at the new token's position T; the rotated k and v of the
    new token are quantized per token-head (Q1-Q6 with G = d) and appended to
    the layer's cache as token T; a = refined attention of q over the T + 1
    tokens (A1-A6); h = x + o(a); n2 = RMSNorm(h);
    out = h + down(silu(gate(n2)) * up(n2)), silu(z) = z / (1 + e^-z).
D4  every GEMV input, and q as it enters the attention, is the bf16 rounding
    (to nearest, ties to even) of its fp64 value: the refined GEMV and the
    attention take bf16 operands (G1, A2).  Everything else stays fp64.
D5  each GEMV refines the top-k channels of its own input row (T1-T3) with
    k = round_half_up(p K) for one fraction p; the attention refines the top
    round_half_up(p_t (T + 1)) tokens per query head.  Counts are taken in
    exact integer arithmetic: floor(p n + 1/2).
D6  after the last layer, RMSNorm and the refined LM head give the logits.
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

from .attn import attn_decode_refine
from .gemv import gemv_refine
from .quant import quantize_nested
from .select import select_topk


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """D4: round finite fp64 values to bf16 (8 significant bits, to nearest,
    ties to even) and return the 16-bit patterns."""
    a = np.asarray(a, dtype=np.float64)
    if not np.all(np.isfinite(a)):
        raise ValueError("non-finite activation")
    m, e = np.frexp(a)                      # a = m 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # rint: ties to even
    r32 = r.astype(np.float32)              # exact: r has <= 8 significant bits
    if np.any(np.isinf(r32)) or np.any((r32 != 0) & (np.abs(r32) < np.finfo(np.float32).tiny)):
        raise ValueError("activation outside the normal bf16 range")
    return (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def count_half_up(p: Fraction, n: int) -> int:
    """D5: floor(p n + 1/2) in exact arithmetic."""
    p = Fraction(p)
    return int((2 * p.numerator * n + p.denominator) // (2 * p.denominator))


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """D1 over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, dtype=np.float64)


def rope(x: np.ndarray, pos: int, theta: float = 500000.0) -> np.ndarray:
    """D2: rotate every head of x [H][d] to position pos, fp64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    ang = pos * theta ** (-2.0 * np.arange(half) / d)
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[..., :half], x[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    """D3: z / (1 + e^-z), fp64."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def refined_linear(qz: dict, x: np.ndarray, p: Fraction) -> np.ndarray:
    """D4-D5 for one matrix: x (fp64 [K]) rounded to bf16, its top-k
    channels refined, y fp64 [N]."""
    xb = f64_to_bf16_bits(x)[None, :]
    K = qz["q"].shape[1]
    S = select_topk(xb, count_half_up(p, K))
    y, _ = gemv_refine(qz, xb, S)
    return y[0]


def kv_append(qz: dict, new_rows: np.ndarray, Hkv: int, T: int, b_r: int, b_f: int) -> dict:
    """D3: quantize the new token's rows [Hkv][d] (one group per row) and
    insert them as token T of every KV head: rows [Hkv][T] -> [Hkv][T + 1]."""
    d = new_rows.shape[1]
    new = quantize_nested(np.asarray(new_rows, dtype=np.float32), d, b_r, b_f)

    def grow(old: np.ndarray, add: np.ndarray) -> np.ndarray:
        o = old.reshape(Hkv, T, *old.shape[1:])
        a = add.reshape(Hkv, 1, *add.shape[1:])
        return np.concatenate([o, a], axis=1).reshape(Hkv * (T + 1), *old.shape[1:])

    out = {k: v for k, v in qz.items()}
    for key in ("q", "q_r", "q_f"):
        out[key] = grow(qz[key], new[key])
    for key in ("scale", "zero"):  # [1][Hkv T]
        out[key] = grow(qz[key][0], new[key][0])[None, :]
    return out


def decode_layer(x: np.ndarray, layer: dict, kv: dict, T: int, Hq: int, Hkv: int, p: Fraction,
                 p_tok: Fraction) -> tuple[np.ndarray, dict]:
    """D3 for one layer.  ``layer`` holds the quantized matrices q, k, v, o,
    gate, up, down (dicts of :func:`quantize_nested`) and the RMSNorm weights
    norm1, norm2; ``kv`` holds the quantized cache ``k``, ``v`` with rows
    [Hkv][T].  Returns (the layer output fp64 [hidden], the cache with the
    new token appended)."""
    d = layer["q"]["q"].shape[0] // Hq
    n1 = rms_norm(x, layer["norm1"])
    q = rope(refined_linear(layer["q"], n1, p).reshape(Hq, d), T)
    k = rope(refined_linear(layer["k"], n1, p).reshape(Hkv, d), T)
    v = refined_linear(layer["v"], n1, p).reshape(Hkv, d)
    b_r, b_f = kv["k"]["b_r"], kv["k"]["b_f"]
    kv2 = dict(k=kv_append(kv["k"], k, Hkv, T, b_r, b_f), v=kv_append(kv["v"], v, Hkv, T, b_r, b_f))
    att = attn_decode_refine(f64_to_bf16_bits(q), kv2["k"], kv2["v"], Hkv, T + 1, count_half_up(p_tok, T + 1))
    h = x + refined_linear(layer["o"], att["out"].reshape(-1), p)
    n2 = rms_norm(h, layer["norm2"])
    g = refined_linear(layer["gate"], n2, p)
    u = refined_linear(layer["up"], n2, p)
    out = h + refined_linear(layer["down"], silu(g) * u, p)
    return out, kv2


def decode_step(x: np.ndarray, layers: list, kvs: list, T: int, Hq: int, Hkv: int, final_norm: np.ndarray,
                lm_head: dict, p: Fraction, p_tok: Fraction) -> tuple[np.ndarray, list]:
    """D3 for every layer, then D6.  x: the new token's embedding, fp64
    [hidden].  Returns (logits fp64 [vocab], the caches with the token
    appended)."""
    out_kv = []
    for layer, kv in zip(layers, kvs):
        x, kv2 = decode_layer(x, layer, kv, T, Hq, Hkv, p, p_tok)
        out_kv.append(kv2)
    logits = refined_linear(lm_head, rms_norm(x, final_norm), p)
    return logits, out_kv
