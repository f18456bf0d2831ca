"""Pins for the oracle's refined GEMV (CPU only).

* brute force: a pure-Python triple loop that decodes every weight straight
  from the packed bitstreams (read back with numpy.unpackbits) and the fp16
  scale/zero, with exact rational arithmetic;
* the two invariants of nested refinement: selecting every channel gives the
  full-code GEMV, selecting none gives the resident-only GEMV;
* the correction in closed form: y(S) - y(empty) = sum over S of
  x_j s (q_f - m_f), evaluated term by term;
* the quantization error bound against the unquantized fp32 weights.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import gemv, quant, select
from workloads import gen_weight, gen_activations, outlier_channels, count_fraction


def _bits_of(words_row):
    return np.unpackbits(np.ascontiguousarray(words_row, dtype="<u4").view(np.uint8), bitorder="little")


def _code(stream, j, bits):
    return sum(int(stream[j * bits + t]) << t for t in range(bits))


def _brute(W, x_bits, S, G, b_r, b_f):
    qz = quant.quantize_nested(W, G, b_r, b_f)
    pk = quant.pack_nested(qz, "by_column")
    N, K = W.shape
    xs = (x_bits.astype(np.uint32) << 16).view(np.float32)
    m_f = Fraction(2 ** b_f - 1, 2)
    S = set(int(j) for j in S)
    refcols = [_bits_of(pk["ref"][j]) for j in range(K)]
    y = np.zeros((x_bits.shape[0], N))
    for i in range(N):
        rs = _bits_of(pk["res"][i])
        for b in range(x_bits.shape[0]):
            acc = Fraction(0)
            for j in range(K):
                s = Fraction(float(pk["scale"][j // G, i]))
                z = Fraction(float(pk["zero"][j // G, i]))
                cr = _code(rs, j, b_r)
                if j in S:
                    cf = _code(refcols[j], i, b_f)
                    w = s * (cr * 2 ** b_f + cf - z)
                else:
                    w = s * (cr * 2 ** b_f + m_f - z)
                acc += Fraction(float(xs[b, j])) * w
            y[b, i] = float(acc)
    return y


@pytest.mark.parametrize("b_r,b_f,B", [(2, 2, 1), (3, 1, 2)])
def test_brute_force_small(b_r, b_f, B):
    N, K, G = 32, 64, 32
    W = gen_weight(31, N, K)
    x = gen_activations(32, B, K, outlier_channels(33, K, 2), 20.0)
    S = select.select_topk(x, 5)
    y, _ = gemv.gemv_refine(quant.quantize_nested(W, G, b_r, b_f), x, S)
    yb = _brute(W, x, S, G, b_r, b_f)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-15)


def test_invariants_and_closed_form_delta():
    N, K, G, b_r, b_f = 64, 512, 64, 2, 2
    W = gen_weight(41, N, K)
    x = gen_activations(42, 1, K, outlier_channels(43, K, 5), 20.0)
    qz = quant.quantize_nested(W, G, b_r, b_f)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y_all, _ = gemv.gemv_refine(qz, x, np.arange(K))
    y_none, _ = gemv.gemv_refine(qz, x, [])
    np.testing.assert_allclose(y_all, xf @ quant.dequant_full(qz).T, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(y_none, xf @ quant.dequant_resident(qz).T, rtol=1e-13, atol=1e-14)
    S = select.select_topk(x, count_fraction(5, K))
    y_S, _ = gemv.gemv_refine(qz, x, S)
    m_f = (2 ** b_f - 1) / 2
    delta = np.zeros(N)
    for i in range(N):
        for j in S:
            s = float(qz["scale"][j // G, i])
            delta[i] += xf[0, j] * s * (int(qz["q_f"][i, j]) - m_f)
    np.testing.assert_allclose(y_S[0] - y_none[0], delta, rtol=1e-9, atol=1e-12)


def test_quantization_error_bound():
    N, K, G = 32, 256, 64
    W = gen_weight(51, N, K)
    x = gen_activations(52, 1, K)
    qz = quant.quantize_nested(W, G, 2, 2)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y_all, _ = gemv.gemv_refine(qz, x, np.arange(K))
    s = np.repeat(qz["scale"].astype(np.float64).T, G, axis=1)
    bound = (np.abs(xf) @ (s / 2).T)[0]
    exact = (xf @ W.astype(np.float64).T)[0]
    assert np.all(np.abs(y_all[0] - exact) <= bound * (1 + 1e-9))
    # refinement strictly helps on average: full-code error below resident error
    y_none, _ = gemv.gemv_refine(qz, x, [])
    assert np.abs(y_all[0] - exact).mean() < np.abs(y_none[0] - exact).mean()


def test_abs_sum():
    W = gen_weight(61, 16, 128)
    x = gen_activations(62, 2, 128)
    qz = quant.quantize_nested(W, 64, 2, 2)
    S = [3, 17]
    y, a = gemv.gemv_refine(qz, x, S)
    w = gemv.effective_weights(qz, S)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for b in range(2):
        for i in range(16):
            assert a[b, i] == pytest.approx(sum(abs(w[i, j] * xf[b, j]) for j in range(128)), rel=1e-12)
            assert abs(y[b, i]) <= a[b, i] * (1 + 1e-12)
