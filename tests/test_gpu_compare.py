"""Comparator modes on the GPU against the oracle (rag-lover.com explainer of
StrataFlux, 既存手法との違い): random channel selection from a counter-based
splitmix64 (bit-exact selection), the FP16-fetch residual store (bit-exact
fp16) and the FP16-fetch GEMV (store and cache; within the GEMV bound)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import cache as ocache
from oracle import compare as ocmp
from oracle import quant as oquant
from oracle import select as oselect
from workloads import count_fraction, gen_activations, gen_weight, outlier_channels

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3


@pytest.fixture(scope="module")
def sf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    return sf


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def _check_gemv(y_gpu, y_ref, abs_sum):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bound = GEMV_TOL * abs_sum
    assert np.all(err <= bound), f"worst err/bound = {(err / np.maximum(bound, 1e-300)).max():.3g}"


@pytest.mark.parametrize("K,k,seed,step", [
    (4096, 122, 7, 0), (4096, 122, 7, 1), (14336, 430, 2**63 + 5, 3), (256, 0, 1, 0), (256, 256, 9, 2),
    (1000, 37, 0, 12345), (32768, 983, 42, 7),
])
def test_select_random(sf, K, k, seed, step):
    idx = torch.empty(max(k, 1), dtype=torch.int32, device="cuda")
    n = torch.empty(1, dtype=torch.int32, device="cuda")
    sf.select_random(K, k, seed, step, idx, n)
    torch.cuda.synchronize()
    assert int(n.item()) == k
    np.testing.assert_array_equal(idx.cpu().numpy()[:k], ocmp.select_random(K, k, seed, step))


@pytest.mark.parametrize("N,K,G,b_r,b_f", [(256, 1024, 128, 3, 1), (96, 512, 64, 2, 2), (128, 384, 128, 2, 1)])
def test_residual_store(sf, N, K, G, b_r, b_f):
    W = gen_weight(70 + N, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    got = sf.quantize_residual(dev(W), qw)
    torch.cuda.synchronize()
    want = ocmp.residual_fp16(W, oquant.quantize_nested(W, G, b_r, b_f)).T
    np.testing.assert_array_equal(got.cpu().numpy().view(np.uint16), np.ascontiguousarray(want).view(np.uint16))


@pytest.mark.parametrize("N,K,G,b_r,b_f,B,pct", [
    (1024, 4096, 128, 3, 1, 1, 5), (512, 2048, 128, 2, 2, 4, 3), (96, 1024, 64, 3, 1, 9, 5),
])
def test_fp16_fetch_store(sf, N, K, G, b_r, b_f, B, pct):
    W = gen_weight(900 + N, N, K)
    x = gen_activations(910 + B, B, K, outlier_channels(11, K, count_fraction("1/2", K)), 30.0)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    r = sf.quantize_residual(dev(W), qw)
    xd = bf16_dev(x)
    k = count_fraction(pct, K)
    idx, n = sf.select_topk(xd, k)
    y = sf.gemv_fp16_fetch(qw, xd, idx, n, resid=r)
    torch.cuda.synchronize()
    S = oselect.select_topk(x, k)
    np.testing.assert_array_equal(idx.cpu().numpy()[: int(n.item())], S)
    y_ref, a = ocmp.gemv_fp16_fetch(oquant.quantize_nested(W, G, b_r, b_f), W, x, S)
    _check_gemv(y.cpu().numpy(), y_ref, a)


def test_fp16_fetch_cache_random_selection(sf):
    """4096x4096, 3+1 bits, random 3% of channels per step through a 10% LRU
    cache of fp16 residual columns (units of N*2 bytes) over three steps."""
    N = K = 4096
    G, b_r, b_f = 128, 3, 1
    W = gen_weight(4242, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    r = sf.quantize_residual(dev(W), qw)
    master = r.cpu().contiguous().view(torch.uint8).pin_memory()
    k = count_fraction(3, K)
    cap = count_fraction(10, K)
    cache = sf.RefineCache(K, N * 2, cap, k, master)
    orc = ocache.LRUCache(K, cap)
    qz = oquant.quantize_nested(W, G, b_r, b_f)
    idx = torch.empty(k, dtype=torch.int32, device="cuda")
    n = torch.empty(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    for step in range(3):
        x = gen_activations(5000 + step, 1, K, outlier_channels(13, K, count_fraction("1/2", K)), 30.0)
        xd = bf16_dev(x)
        sf.select_random(K, k, 99, step, idx, n)
        cache.prefetch(idx, n, torch.cuda.current_stream(), side)
        y = sf.gemv_fp16_fetch(qw, xd, idx, n, cache=cache)
        torch.cuda.synchronize()
        S = ocmp.select_random(K, k, 99, step)
        want = orc.step(S.tolist())
        got = cache.sets()
        assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
        y_ref, a = ocmp.gemv_fp16_fetch(qz, W, x, S)
        _check_gemv(y.cpu().numpy(), y_ref, a)
    cache.close()
