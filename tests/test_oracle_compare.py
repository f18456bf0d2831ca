"""Pins of the comparator-mode oracle (oracle.compare): the published
splitmix64 value, the random selection's invariants and uniformity, and the
FP16-fetch GEMV's extremes against a dense matmul."""

import numpy as np
import pytest

from oracle import compare as oc
from oracle.quant import dequant_resident, quantize_nested
from workloads import gen_activations, gen_weight, outlier_channels


def test_splitmix64_published_values():
    # the first three outputs of a splitmix64 generator whose state starts at
    # 0 (its published reference sequence); output i is the finalizer of
    # state (i - 1) * 0x9E3779B97F4A7C15
    g = 0x9E3779B97F4A7C15
    assert [oc.splitmix64((i * g) & (2 ** 64 - 1)) for i in range(3)] == \
        [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_random_selection_invariants():
    K, k = 1024, 31
    S = oc.select_random(K, k, seed=7, step=3)
    assert len(S) == k and np.all(np.diff(S) > 0) and S.min() >= 0 and S.max() < K
    np.testing.assert_array_equal(S, oc.select_random(K, k, seed=7, step=3))   # reproducible
    assert not np.array_equal(S, oc.select_random(K, k, seed=7, step=4))       # another step, another draw
    keys = oc.random_keys(K, 7, 3)
    assert keys.max() < 0x7F80
    # the chosen keys are the k largest (ties to the lower channel)
    order = sorted(range(K), key=lambda j: (-int(keys[j]), j))
    assert sorted(order[:k]) == S.tolist()


def test_random_selection_is_close_to_uniform():
    """Over many steps every channel is chosen with frequency ~ k / K
    (chi-square well inside its 1e-6 tail)."""
    K, k, steps = 256, 16, 400
    counts = np.zeros(K)
    for t in range(steps):
        counts[oc.select_random(K, k, seed=99, step=t)] += 1
    expect = steps * k / K
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 400.0, chi2                 # K - 1 = 255 degrees of freedom
    assert counts.min() > 0


@pytest.mark.parametrize("b_r,b_f", [(3, 1), (2, 2)])
def test_fp16_fetch_extremes(b_r, b_f):
    N, K = 48, 256
    W = gen_weight(61, N, K)
    qz = quantize_nested(W, 128, b_r, b_f)
    x = gen_activations(62, 2, K, outlier_channels(63, K, 3), 30.0)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # nothing fetched: the resident GEMV
    y0, _ = oc.gemv_fp16_fetch(qz, W, x, [])
    np.testing.assert_allclose(y0, xf @ dequant_resident(qz).T, rtol=1e-12, atol=1e-12)
    # everything fetched: the fp32 weights up to the fp16 rounding of the residual
    y1, _ = oc.gemv_fp16_fetch(qz, W, x, np.arange(K))
    r = W.astype(np.float64) - dequant_resident(qz)
    bound = np.abs(xf) @ (np.abs(r) * 2.0 ** -11).T + 1e-12
    assert np.all(np.abs(y1 - xf @ W.astype(np.float64).T) <= bound)
    # the residual is exactly the fp16 rounding of an exact fp64 difference
    np.testing.assert_array_equal(oc.residual_fp16(W, qz), r.astype(np.float16))
