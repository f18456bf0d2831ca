"""Property tests of the oracle over random seeds, sizes and odd shapes
(bounded example counts, so the CPU suite stays fast).  Each property is
checked against something other than the function itself: a library
primitive, a brute-force enumeration, an error bound fixed by the format, or
an identity of the mathematics."""

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st
from scipy.special import softmax

from oracle import attn as oattn
from oracle import decode as od
from oracle import gemv as ogemv
from oracle import quant as oquant
from oracle import select as oselect

SETTINGS = settings(max_examples=25, deadline=None)


def _bf16_bits(a):
    return od.f64_to_bf16_bits(np.asarray(a, dtype=np.float64))


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), rows=st.integers(1, 6), groups=st.integers(1, 3), G=st.sampled_from([32, 64]),
       bits=st.sampled_from([(2, 2), (3, 1), (2, 1)]), scale=st.floats(1e-3, 1e3))
def test_quant_bounds_and_round_trip(seed, rows, groups, G, bits, scale):
    b_r, b_f = bits
    W = (np.random.default_rng(seed).standard_normal((rows, groups * G)) * scale).astype(np.float32)
    qz = oquant.quantize_nested(W, G, b_r, b_f)
    b = b_r + b_f
    assert qz["q"].max() <= 2 ** b - 1
    # the full code is within half a step of every weight (the group's min and
    # max bound the range), except that s is rounded to fp16 (relative error
    # <= 2^-11), so the grid's span (2^b - 1) s may fall short of hi - lo by
    # (2^b - 1) 2^-11 s at the top end
    s = np.repeat(qz["scale"].astype(np.float64).T, G, axis=1)
    slack = (2 ** b - 1) * 2.0 ** -11 + 1e-6
    err = np.abs(oquant.dequant_full(qz) - W.astype(np.float64))
    assert np.all(err <= s * (0.5 + slack) + 1e-12)
    # the resident value (midpoint of the refinement interval) is within
    # s (2^b_f - 1) / 2 of the full code, so within s 2^b_f / 2 of the weight
    err_r = np.abs(oquant.dequant_resident(qz) - W.astype(np.float64))
    assert np.all(err_r <= s * (2 ** b_f / 2 + slack) + 1e-12)
    # packing round trip, and agreement with numpy's little-endian bit packing
    for codes, nb in ((qz["q_r"], b_r), (qz["q_f"], b_f)):
        words = oquant.pack_bits(codes, nb)
        np.testing.assert_array_equal(oquant.unpack_bits(words, codes.shape[1], nb), codes)
        bitsarr = ((codes[:, :, None].astype(np.uint32) >> np.arange(nb, dtype=np.uint32)) & 1).astype(np.uint8)
        lib = np.packbits(bitsarr.reshape(codes.shape[0], -1), axis=1, bitorder="little")
        np.testing.assert_array_equal(words.view(np.uint8).reshape(codes.shape[0], -1), lib)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), B=st.integers(1, 4), K=st.integers(1, 200), frac=st.floats(0, 1),
       levels=st.integers(1, 8))
def test_select_matches_brute_force(seed, B, K, frac, levels):
    rng = np.random.default_rng(seed)
    # few distinct magnitudes (many ties), both signs and zeros
    x = rng.integers(-levels, levels + 1, size=(B, K)).astype(np.float64) * 0.5
    bits = _bf16_bits(x)
    k = int(frac * K)
    got = oselect.select_topk(bits, k)
    want = set()
    for b in range(B):
        keyed = sorted(range(K), key=lambda j: (-abs(x[b, j]), j))   # library sort, stable rule
        want.update(keyed[:k])
    np.testing.assert_array_equal(got, np.array(sorted(want), dtype=np.int32))


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), N=st.integers(1, 16), groups=st.integers(1, 3), B=st.integers(1, 3))
def test_gemv_extremes_equal_dense_matmul(seed, N, groups, B):
    rng = np.random.default_rng(seed)
    K = 32 * groups
    qz = oquant.quantize_nested((rng.standard_normal((N, K)) * 0.05).astype(np.float32), 32, 2, 2)
    xb = _bf16_bits(rng.standard_normal((B, K)))
    x = ogemv.bf16_to_f64(xb)
    y_all, _ = ogemv.gemv_refine(qz, xb, np.arange(K))
    y_none, _ = ogemv.gemv_refine(qz, xb, np.zeros(0, np.int64))
    np.testing.assert_allclose(y_all, np.matmul(x, oquant.dequant_full(qz).T), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y_none, np.matmul(x, oquant.dequant_resident(qz).T), rtol=1e-12, atol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), Hkv=st.integers(1, 2), grp=st.sampled_from([1, 2, 4]), T=st.integers(1, 40))
def test_attention_extremes_equal_plain_softmax(seed, Hkv, grp, T):
    rng = np.random.default_rng(seed)
    d = 32
    Hq = Hkv * grp
    K = rng.standard_normal((Hkv * T, d)).astype(np.float32)
    V = rng.standard_normal((Hkv * T, d)).astype(np.float32)
    qzk, qzv = oquant.quantize_nested(K, d, 2, 2), oquant.quantize_nested(V, d, 2, 2)
    qb = _bf16_bits(rng.standard_normal((Hq, d)))
    q = oattn.bf16_to_f64(qb)
    for k_tok, deq in ((T, oquant.dequant_full), (0, oquant.dequant_resident)):
        got = oattn.attn_decode_refine(qb, qzk, qzv, Hkv, T, k_tok)["out"]
        Kd, Vd = deq(qzk).reshape(Hkv, T, d), deq(qzv).reshape(Hkv, T, d)
        for h in range(Hq):
            g = h // grp
            want = softmax(Kd[g] @ q[h] / math.sqrt(d)) @ Vd[g]
            np.testing.assert_allclose(got[h], want, rtol=1e-10, atol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), half=st.integers(1, 64), m=st.integers(0, 200000), n=st.integers(0, 200000))
def test_rope_relative_position_and_norms(seed, half, m, n):
    rng = np.random.default_rng(seed)
    d = 2 * half
    q, k = rng.standard_normal((2, d)), rng.standard_normal((2, d))
    a = np.sum(od.rope(q, m) * od.rope(k, n), axis=1)
    b = np.sum(od.rope(q, m - n) * k, axis=1) if m >= n else np.sum(q * od.rope(k, n - m), axis=1)
    np.testing.assert_allclose(a, b, rtol=1e-8, atol=1e-8)
    r = od.rope(q, m)
    np.testing.assert_allclose(np.hypot(r[:, :half], r[:, half:]), np.hypot(q[:, :half], q[:, half:]), rtol=1e-12)
