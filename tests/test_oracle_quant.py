"""Pins for the oracle's nested quantizer and packing (CPU only).

Each check ties the oracle to something other than itself: hand-worked
examples (tests/golden/quant_worked.json), numpy.packbits, an fp64 route to
the fp32 quotient, Python's struct half-precision rounding, and the
quantization error bounds that hold by construction of round-to-nearest.
"""

import json
import os
import struct

import numpy as np
import pytest

from oracle import quant
from workloads import count_fraction, gen_weight

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_worked.json")


def test_count_rule():
    # floor(p*n + 1/2): 5% of 512 is 25.6 -> 26 (the top-k of the 512x512
    # layer); the other values are the counts of the Llama/Qwen/attention shapes.
    cases = {(5, 512): 26, (3, 4096): 123, (3, 14336): 430, (5, 4096): 205, (5, 12288): 614,
             (1, 32768): 328, (10, 4096): 410, (10, 14336): 1434, (25, 4096): 1024,
             (25, 12288): 3072, ("1/2", 4096): 20, ("1/2", 14336): 72, (1, 512): 5}
    for (p, n), want in cases.items():
        assert count_fraction(p, n) == want, (p, n)
    # exact half rounds up
    assert count_fraction(50, 1) == 1 and count_fraction(25, 2) == 1


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_worked_examples(case):
    W = np.array([case["w"]], dtype=np.float32)
    qz = quant.quantize_nested(W, 4, case["b_r"], case["b_f"])
    assert qz["q"][0].tolist() == case["q"]
    assert qz["q_r"][0].tolist() == case["q_r"]
    assert qz["q_f"][0].tolist() == case["q_f"]
    s = float(qz["scale"][0, 0])
    assert s == pytest.approx(case["scale"], rel=0, abs=1e-12)
    assert float(qz["zero"][0, 0]) == case["zero"]
    assert np.signbit(qz["zero"]).sum() == 0          # zero point stored as +0
    np.testing.assert_array_equal(quant.dequant_full(qz)[0], s * np.array(case["full_over_s"], float))
    np.testing.assert_array_equal(quant.dequant_resident(qz)[0], s * np.array(case["resident_over_s"], float))


def _half_rne_struct(v: float) -> float:
    # Python's struct 'e' format rounds to nearest, ties to even
    return struct.unpack("<e", struct.pack("<e", v))[0]


def test_scale_and_zero_against_independent_rounding():
    """Q2/Q3 recomputed through fp64 arithmetic (double rounding of +,-,/ from
    binary64 to binary32 is innocuous) and struct's fp16 rounding."""
    W = gen_weight(11, 64, 256)
    G, b_r, b_f = 64, 2, 2
    qz = quant.quantize_nested(W, G, b_r, b_f)
    for r in range(W.shape[0]):
        for g in range(W.shape[1] // G):
            grp = W[r, g * G:(g + 1) * G].astype(np.float64)
            lo, hi = float(grp.min()), float(grp.max())
            span = float(np.float32(hi - lo))
            s32 = float(np.float32(span / 15.0))
            s = _half_rne_struct(min(s32, 65504.0)) or 1.0
            assert float(qz["scale"][g, r]) == s
            z = min(max(float(np.rint(np.float32(-lo / s))), 0.0), 15.0)
            assert float(qz["zero"][g, r]) == z
            q = np.clip(np.rint((grp / s).astype(np.float32)) + z, 0, 15)
            np.testing.assert_array_equal(qz["q"][r, g * G:(g + 1) * G], q.astype(np.uint8))


@pytest.mark.parametrize("b_r,b_f", [(2, 2), (3, 1), (2, 1), (3, 0)])
def test_error_bounds(b_r, b_f):
    """Round-to-nearest bounds: |w - full| <= s/2 for every in-range w, and the
    resident value is within s/2 + s*m_f of w; delta full - resident equals
    s (q_f - m_f) exactly."""
    W = gen_weight(5, 48, 512)
    G = 128
    qz = quant.quantize_nested(W, G, b_r, b_f)
    s = np.repeat(qz["scale"].astype(np.float64).T, G, axis=1)
    z = np.repeat(qz["zero"].astype(np.float64).T, G, axis=1)
    full = quant.dequant_full(qz)
    res = quant.dequant_resident(qz)
    w = W.astype(np.float64)
    qmax = 2 ** (b_r + b_f) - 1
    in_range = (w >= s * (0 - z) - s / 2) & (w <= s * (qmax - z) + s / 2)
    assert in_range.mean() > 0.99
    assert np.all(np.abs(w - full)[in_range] <= s[in_range] / 2 * (1 + 1e-6))
    m_f = (2 ** b_f - 1) / 2
    assert np.all(np.abs(w - res)[in_range] <= (s / 2 + s * m_f)[in_range] * (1 + 1e-6))
    np.testing.assert_array_equal(full - res, s * (qz["q_f"].astype(np.float64) - m_f))
    # codes cover the range: min and max of every group map to 0 and qmax or near
    assert qz["q"].max() == qmax and qz["q"].min() == 0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_matches_numpy_packbits(bits):
    rng = np.random.default_rng(bits)
    R, C = 5, 96
    codes = rng.integers(0, 2 ** bits, size=(R, C)).astype(np.uint8)
    words = quant.pack_bits(codes, bits)
    # stream of bits: code j contributes bits j*bits .. j*bits+bits-1, LSB first
    stream = np.unpackbits(codes[:, :, None], axis=2, bitorder="little")[:, :, :bits].reshape(R, C * bits)
    ref = np.packbits(stream, axis=1, bitorder="little").view("<u4")
    np.testing.assert_array_equal(words, ref)
    np.testing.assert_array_equal(quant.unpack_bits(words, C, bits), codes)


def test_three_bit_straddle_by_hand():
    # codes 0..7 repeated: code 10 (value 2) sits at stream bits 30..32, i.e.
    # bits 30-31 of word 0 and bit 0 of word 1.
    codes = (np.arange(32) % 8).astype(np.uint8)[None, :]
    w = quant.pack_bits(codes, 3)
    assert w.shape == (1, 3)
    assert (int(w[0, 0]) >> 30) & 3 == 2 & 3 and int(w[0, 1]) & 1 == (2 >> 2) & 1
    # code 21 (value 5 = 0b101) at bits 63..65: bit 31 of word 1, bits 0-1 of word 2
    assert (int(w[0, 1]) >> 31) & 1 == 1 and int(w[0, 2]) & 3 == 0b10


def test_layouts():
    W = gen_weight(3, 128, 256)
    qz = quant.quantize_nested(W, 128, 2, 2)
    col = quant.pack_nested(qz, "by_column")
    row = quant.pack_nested(qz, "by_row")
    assert col["res"].shape == (128, 256 * 2 // 32)
    assert col["ref"].shape == (256, 128 * 2 // 32)
    assert row["ref"].shape == (128, 256 * 2 // 32)
    np.testing.assert_array_equal(quant.unpack_bits(col["ref"], 128, 2).T, qz["q_f"])
    np.testing.assert_array_equal(quant.unpack_bits(row["ref"], 256, 2), qz["q_f"])
