"""Pins for the oracle's top-k channel selection (CPU only): numpy's stable
argsort on -|x| (a library sort), adversarial ties, signed zeros, the union
over batch rows, and rejection of non-finite activations."""

import numpy as np
import pytest

from oracle import select
from workloads import f32_to_bf16_bits, gen_activations, outlier_channels, count_fraction


def _library_topk(bits_row, k):
    mag = np.abs((bits_row.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.argsort(-mag, kind="stable")[:k]


@pytest.mark.parametrize("K,k", [(512, 26), (4096, 123), (1024, 1), (256, 256), (64, 0)])
def test_matches_stable_argsort(K, k):
    out = outlier_channels(7, K, max(1, K // 200))
    x = gen_activations(9, 1, K, out, 30.0)
    got = select.select_topk(x, k)
    want = np.sort(_library_topk(x[0], k))
    np.testing.assert_array_equal(got, want)


def test_ties_go_to_lower_index():
    # many equal magnitudes with both signs: only the index decides
    vals = np.array([1.0, -2.0, 2.0, -1.0, 2.0, 0.5, -2.0, 1.0], np.float32)
    x = f32_to_bf16_bits(vals)[None, :]
    assert select.select_topk(x, 3).tolist() == [1, 2, 4]
    assert select.select_topk(x, 4).tolist() == [1, 2, 4, 6]
    assert select.select_topk(x, 5).tolist() == [0, 1, 2, 4, 6]


def test_signed_zero_ties():
    vals = np.array([0.0, -0.0, 0.0, -0.0], np.float32)
    x = f32_to_bf16_bits(vals)[None, :]
    assert select.select_topk(x, 2).tolist() == [0, 1]


def test_bf16_resolution_ties():
    # distinct fp32 values that round to the same bf16 magnitude tie exactly
    vals = np.array([1.0, 1.001, 1.002, 0.5], np.float32)
    x = f32_to_bf16_bits(vals)[None, :]
    assert select.select_topk(x, 2).tolist() == [0, 1]


def test_union_over_batch():
    K, k, B = 1024, count_fraction(5, 1024), 4
    x = gen_activations(21, B, K)
    got = select.select_topk(x, k)
    want = set()
    for b in range(B):
        want |= set(_library_topk(x[b], k).tolist())
    assert got.tolist() == sorted(want)
    assert len(got) <= B * k


def test_rejects_non_finite():
    x = f32_to_bf16_bits(np.array([1.0, np.inf, 0.0, 2.0], np.float32))[None, :]
    with pytest.raises(ValueError):
        select.select_topk(x, 1)
    nan = np.array([[0x7FC0, 0x3F80]], np.uint16)
    with pytest.raises(ValueError):
        select.select_topk(nan, 1)
