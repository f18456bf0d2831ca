"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bit-exact: packed codes, fp16 scale/zero, selected channel indices, cache
hit / miss / bypass sets and slot placement, selected token sets.
Tolerance: refined GEMV |y - y_ref| <= 2e-3 * sum_j |w_eff x| per output;
refined attention max-abs error <= 2e-3.
"""

import numpy as np
import pytest
import torch

from oracle import attn as oattn
from oracle import cache as ocache
from oracle import gemv as ogemv
from oracle import quant as oquant
from oracle import select as oselect
from workloads import (count_fraction, gen_activations, gen_kv, gen_query, gen_weight, outlier_channels,
                       f32_to_bf16_bits)

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3
ATTN_TOL = 2e-3


@pytest.fixture(scope="module")
def sf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    return sf


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def f16(t):
    return t.cpu().numpy().view(np.float16)


def bf16_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


# ---- quantization ----------------------------------------------------------

@pytest.mark.parametrize("N,K,G,b_r,b_f,layout", [
    (512, 512, 64, 2, 2, "by_column"),
    (1024, 4096, 128, 2, 2, "by_column"),
    (128, 384, 128, 3, 1, "by_column"),
    (96, 256, 32, 2, 1, "by_column"),
    (40, 256, 128, 2, 2, "by_row"),
    (8, 128, 128, 2, 2, "by_row"),
])
def test_quantize_bit_exact(sf, N, K, G, b_r, b_f, layout):
    W = gen_weight(100 + N + K, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f, layout)
    torch.cuda.synchronize()
    ref = oquant.pack_nested(oquant.quantize_nested(W, G, b_r, b_f), layout)
    np.testing.assert_array_equal(u32(qw.res), ref["res"])
    np.testing.assert_array_equal(u32(qw.ref), ref["ref"])
    np.testing.assert_array_equal(f16(qw.scale).view(np.uint16), ref["scale"].view(np.uint16))
    np.testing.assert_array_equal(f16(qw.zero).view(np.uint16), ref["zero"].view(np.uint16))


def test_quantize_worked_examples(sf):
    import json
    import os
    cases = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quant_worked.json")))["cases"]
    for c in cases:
        if c["b_r"] + c["b_f"] != 4:
            continue
        row = np.tile(np.array(c["w"], np.float32), 8)     # one group of 32 with the same min/max
        W = np.tile(row, (32, 1))
        qw = sf.quantize_nested(dev(W), 32, c["b_r"], c["b_f"])
        torch.cuda.synchronize()
        codes = oquant.unpack_bits(u32(qw.res)[:1], 32, c["b_r"])[0]
        assert codes[:4].tolist() == c["q_r"], c["name"]
        assert float(f16(qw.scale)[0, 0]) == pytest.approx(c["scale"], abs=1e-12)
        assert float(f16(qw.zero)[0, 0]) == c["zero"]
        fcodes = oquant.unpack_bits(u32(qw.ref)[:4], 32, c["b_f"])[:, 0]
        assert fcodes.tolist() == c["q_f"], c["name"]


# ---- selection ------------------------------------------------------------

@pytest.mark.parametrize("B,K,pct", [(1, 512, 5), (1, 4096, 3), (1, 14336, 3), (4, 4096, 5), (16, 12288, 5),
                                     (3, 1000, 10), (1, 64, 100), (2, 32768, 3), (16, 32768, 1), (16, 40000, 2)])
def test_select_exact(sf, B, K, pct):
    k = count_fraction(pct, K)
    x = gen_activations(200 + K + B, B, K, outlier_channels(7, K, max(1, K // 200)), 30.0)
    idx, n = sf.select_topk(bf16_dev(x), k)
    torch.cuda.synchronize()
    want = oselect.select_topk(x, k)
    got = idx.cpu().numpy()[: int(n.item())]
    np.testing.assert_array_equal(got, want)


def test_select_ties_and_edges(sf):
    rng = np.random.default_rng(5)
    K = 4096
    levels = np.array([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0], np.float32)
    x = f32_to_bf16_bits(rng.choice(levels, size=(4, K)))
    for k in (0, 1, 7, 100, 1500, K):
        idx, n = sf.select_topk(bf16_dev(x), k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy()[: int(n.item())], oselect.select_topk(x, k))
    bad = x.copy()
    bad[2, 17] = 0x7FC0  # NaN
    idx, n = sf.select_topk(bf16_dev(bad), 10)
    torch.cuda.synchronize()
    assert int(n.item()) == -1


# ---- refinement cache --------------------------------------------------------

def _steps(seed, K, n_steps, k, hot):
    rng = np.random.default_rng(seed)
    hot_set = rng.choice(K, size=hot, replace=False)
    for i in range(n_steps):
        kk = k if i % 7 else 3 * k      # every 7th step overflows small caches (bypass)
        rest = rng.choice(K, size=kk, replace=False)
        yield np.array(sorted(set(hot_set.tolist()) | set(rest[:kk - hot].tolist())), np.int32)


@pytest.mark.parametrize("K,N,b_f,C,k,hot", [(512, 256, 2, 40, 30, 5), (4096, 1024, 2, 410, 123, 20),
                                             (1024, 128, 1, 16, 24, 4), (300, 128, 2, 300, 20, 3)])
def test_cache_sets_and_slots(sf, K, N, b_f, C, k, hot):
    unit_bytes = N * b_f // 8
    rng = np.random.default_rng(K + C)
    master = torch.from_numpy(rng.integers(0, 2 ** 31, size=(K, unit_bytes // 4), dtype=np.int64).astype(np.int32))
    master = master.pin_memory()
    max_sel = 3 * k + hot
    cache = sf.RefineCache(K, unit_bytes, C, max_sel, master)
    orc = ocache.LRUCache(K, C)
    idx = torch.zeros(max_sel, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    for S in _steps(K, K, 25, k, hot):
        idx[: len(S)].copy_(dev(S))
        n.fill_(len(S))
        cache.prefetch(idx, n, torch.cuda.current_stream(), side)
        got = cache.sets()
        want = orc.step(S.tolist())
        assert got["hits"] == want["hits"]
        assert got["misses"] == want["misses"]
        assert got["bypass"] == want["bypass"]
        slots = cache.slots()
        snap = orc.snapshot()
        assert {u: s for s, u in enumerate(slots) if u >= 0} == snap
    st = cache.stats()
    assert st.steps == 25 and st.hits == orc.hits and st.misses == orc.misses and st.bypass == orc.bypass
    assert st.h2d_bytes == orc.misses * unit_bytes
    cache.reset()
    assert cache.stats().steps == 0
    cache.close()


# ---- refined GEMV ----------------------------------------------------------------

def _check_gemv(y_gpu, y_ref, abs_sum):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bound = GEMV_TOL * abs_sum
    worst = (err / np.maximum(bound, 1e-300)).max()
    assert np.all(err <= bound), f"worst err/bound = {worst:.3g}"


def _host_master(qw):
    return qw.ref.cpu().contiguous().pin_memory()


def test_gemv_linear_512_preloaded_cache(sf):
    """512x512, group 64, 2+2, 1% outliers x20, top-26, cache holds every column."""
    N = K = 512
    W = gen_weight(1000, N, K)
    x = gen_activations(2000, 1, K, outlier_channels(5000, K, count_fraction(1, K)), 20.0)
    qw = sf.quantize_nested(dev(W), 64, 2, 2)
    k = count_fraction(5, K)
    cache = sf.RefineCache(K, N * 2 // 8, K, k, _host_master(qw))
    cache.preload(torch.arange(K, dtype=torch.int32, device="cuda"))
    xd = bf16_dev(x)
    idx, n = sf.select_topk(xd, k)
    cache.prefetch(idx, n)
    y = sf.gemv_refine(qw, xd, idx, n, cache=cache)
    torch.cuda.synchronize()
    assert cache.sets()["hits"] == oselect.select_topk(x, k).tolist()
    qz = oquant.quantize_nested(W, 64, 2, 2)
    y_ref, a = ogemv.gemv_refine(qz, x, oselect.select_topk(x, k))
    _check_gemv(y.cpu().numpy(), y_ref, a)
    # resident-only and every column refined (store read directly)
    y0 = sf.gemv_refine(qw, xd)
    all_idx = torch.arange(K, dtype=torch.int32, device="cuda")
    all_n = torch.tensor([K], dtype=torch.int32, device="cuda")
    y1 = sf.gemv_refine(qw, xd, all_idx, all_n, use_ref_store=True)
    torch.cuda.synchronize()
    r0, a0 = ogemv.gemv_refine(qz, x, [])
    r1, a1 = ogemv.gemv_refine(qz, x, np.arange(K))
    _check_gemv(y0.cpu().numpy(), r0, a0)
    _check_gemv(y1.cpu().numpy(), r1, a1)
    cache.close()


@pytest.mark.parametrize("N,K,G,b_r,b_f,B,pct", [
    (1024, 4096, 128, 3, 1, 1, 5), (1024, 4096, 128, 3, 1, 4, 5), (512, 4096, 128, 3, 1, 16, 5),
    (256, 14336, 128, 2, 2, 1, 3), (4096, 1024, 128, 2, 2, 2, 3), (96, 2048, 64, 2, 1, 7, 5),
    (256, 2048, 64, 3, 1, 16, 5), (128, 1024, 32, 2, 2, 9, 5),
])
def test_gemv_store(sf, N, K, G, b_r, b_f, B, pct):
    W = gen_weight(300 + N + K + B, N, K)
    x = gen_activations(400 + B, B, K, outlier_channels(9, K, count_fraction("1/2", K)), 30.0)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    k = count_fraction(pct, K)
    xd = bf16_dev(x)
    idx, n = sf.select_topk(xd, k)
    y = sf.gemv_refine(qw, xd, idx, n, use_ref_store=True)
    torch.cuda.synchronize()
    S = oselect.select_topk(x, k)
    np.testing.assert_array_equal(idx.cpu().numpy()[: int(n.item())], S)
    y_ref, a = ogemv.gemv_refine(oquant.quantize_nested(W, G, b_r, b_f), x, S)
    _check_gemv(y.cpu().numpy(), y_ref, a)


@pytest.mark.parametrize("N,K,G,b_r,b_f,B,pct", [
    (1024, 4096, 128, 3, 1, 16, 5), (1024, 4096, 128, 3, 1, 8, 5), (96, 2048, 128, 2, 2, 9, 3),
    (512, 6144, 128, 2, 1, 12, 5), (256, 12288, 256, 3, 1, 16, 5), (160, 1024, 128, 3, 1, 16, 0),
])
def test_gemv_batch_tensor_cores(sf, N, K, G, b_r, b_f, B, pct):
    """Batches of 8-16 rows run the resident part on the tensor cores (f16
    MMAs over exact code values, one selection for the batch): several K
    chunks, a half-filled last row tile (N = 96, 160), group 256, and no
    selection at all (pct 0)."""
    W = gen_weight(700 + N + K + B, N, K)
    x = gen_activations(710 + B, B, K, outlier_channels(19, K, count_fraction("1/2", K)), 30.0)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    xd = bf16_dev(x)
    qz = oquant.quantize_nested(W, G, b_r, b_f)
    if pct:
        k = count_fraction(pct, K)
        idx, n = sf.select_topk(xd, k)
        y = sf.gemv_refine(qw, xd, idx, n, use_ref_store=True)
        S = oselect.select_topk(x, k)
    else:
        y = sf.gemv_refine(qw, xd)
        S = np.zeros(0, np.int64)
    torch.cuda.synchronize()
    y_ref, a = ogemv.gemv_refine(qz, x, S)
    _check_gemv(y.cpu().numpy(), y_ref, a)


def test_gemv_batch_tensor_cores_cache(sf):
    """Qwen3-8B's gate shape at 3+1 bits, batch 16, top 5% of channels as the
    union over the batch, 25% LRU cache, three steps; the oracle checks 128
    sampled rows each step."""
    N, K, G, b_r, b_f, B = 12288, 4096, 128, 3, 1, 16
    W = gen_weight(4321, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    k = count_fraction(5, K)
    cap = count_fraction(25, K)
    cache = sf.RefineCache(K, N * b_f // 8, cap, min(K, B * k), _host_master(qw))  # the union: up to B k channels
    orc = ocache.LRUCache(K, cap)
    rows = np.sort(np.random.default_rng(7).choice(N, size=128, replace=False))
    qz = oquant.quantize_nested(W[rows], G, b_r, b_f)
    outl = outlier_channels(77, K, count_fraction("1/2", K))
    for step in range(3):
        x = gen_activations(3100 + step, B, K, outl, 30.0)
        xd = bf16_dev(x)
        idx, n = sf.select_topk(xd, k)
        cache.prefetch(idx, n)
        y = sf.gemv_refine(qw, xd, idx, n, cache=cache)
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        want = orc.step(S.tolist())
        got = cache.sets()
        assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
        y_ref, a = ogemv.gemv_refine(qz, x, S)
        _check_gemv(y.cpu().numpy()[:, rows], y_ref, a)
    cache.close()


@pytest.mark.parametrize("N,K,cap_pct", [(14336, 4096, 10), (4096, 14336, 10)])
def test_gemv_full_size_cache_sampled_rows(sf, N, K, cap_pct):
    """Llama-3.1-8B gate/down shapes, 2+2, group 128, top 3%, 10% LRU cache,
    several steps; the oracle checks 192 sampled rows each step."""
    G, b_r, b_f = 128, 2, 2
    W = gen_weight(1000 + N, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    k = count_fraction(3, K)
    cap = count_fraction(cap_pct, K)
    cache = sf.RefineCache(K, N * b_f // 8, cap, k, _host_master(qw))
    orc = ocache.LRUCache(K, cap)
    rows = np.sort(np.random.default_rng(N).choice(N, size=192, replace=False))
    qz = oquant.quantize_nested(W[rows], G, b_r, b_f)
    outl = outlier_channels(5000 + K, K, count_fraction("1/2", K))
    side = torch.cuda.Stream()
    for step in range(3):
        x = gen_activations(2000 + step, 1, K, outl, 30.0)
        xd = bf16_dev(x)
        idx, n = sf.select_topk(xd, k)
        cache.prefetch(idx, n, torch.cuda.current_stream(), side)
        y = sf.gemv_refine(qw, xd, idx, n, cache=cache)
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        want = orc.step(S.tolist())
        got = cache.sets()
        assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
        y_ref, a = ogemv.gemv_refine(qz, x, S)
        _check_gemv(y.cpu().numpy()[:, rows], y_ref, a)
    cache.close()


# ---- refined attention -------------------------------------------------------------

def _kv(sf, Hkv, T, d, seed, n_out=4):
    Kf, Vf, _ = gen_kv(seed, Hkv, T, d, n_outlier_ch=n_out)
    Kf2, Vf2 = Kf.reshape(Hkv * T, d), Vf.reshape(Hkv * T, d)
    qk = sf.quantize_nested(dev(Kf2), d, 2, 2, "by_row")
    qv = sf.quantize_nested(dev(Vf2), d, 2, 2, "by_row")
    ok = oquant.quantize_nested(Kf2, d, 2, 2)
    ov = oquant.quantize_nested(Vf2, d, 2, 2)
    return sf.QKV(qk, qv), ok, ov


def _cluster_applies(Hq, Hkv, T):
    return T <= 16 * (2048 if Hq // Hkv <= 4 else 1024)


@pytest.fixture(params=["pipeline", "cluster"])
def attn_path(request, sf):
    """Runs a test once per attention implementation (the multi-kernel
    pipeline and the single cluster kernel per KV head); restores the
    automatic choice afterwards."""
    sf.attn_set_path(sf.ATTN_PIPELINE if request.param == "pipeline" else sf.ATTN_CLUSTER)
    yield request.param
    sf.attn_set_path(sf.ATTN_AUTO)


def _skip_unless_applies(path, Hq, Hkv, T):
    if path == "cluster" and not _cluster_applies(Hq, Hkv, T):
        pytest.skip("the cluster kernel does not apply to this size")


@pytest.mark.parametrize("Hq,Hkv,T,pct", [(8, 2, 1000, 1), (32, 8, 4099, 1), (4, 4, 77, 10), (16, 2, 33, 100),
                                          (8, 1, 512, 0), (8, 2, 8192, 30), (8, 2, 40961, 1), (4, 1, 32768, 2),
                                          (4, 1, 70001, 1), (8, 8, 65536, 1), (64, 8, 16384, 1), (16, 8, 300, 5),
                                          (8, 2, 32768, 1), (32, 8, 1, 100), (8, 1, 20000, 2),
                                          (16, 2, 40000, 100)])
def test_attn_small(sf, attn_path, Hq, Hkv, T, pct):
    """Both implementations against the oracle: the pipeline's compaction,
    finish, refine and output kernels at every size, the cluster kernel up
    to its limit (including clusters with empty CTAs at tiny T, eight query
    heads per KV head, k = T and k = 0), the pairwise ranking of few
    candidates and the radix ranking of many (30% of 8192); eight query
    heads per KV head beyond the cluster kernel's limit, and k = T at 40K
    (every token refined by the refine kernel)."""
    _skip_unless_applies(attn_path, Hq, Hkv, T)
    d = 128
    kv, ok, ov = _kv(sf, Hkv, T, d, 3000 + T)
    qb = gen_query(4000 + T, Hq, d)
    k = count_fraction(pct, T)
    out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
    sel_n = sel_n.cpu().numpy()
    sel = sel.cpu().numpy()
    for g in range(Hkv):
        assert sel_n[g] == len(ref["union"][g])
        np.testing.assert_array_equal(sel[g, : sel_n[g]], ref["union"][g])
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref["out"]).max()
    assert err <= ATTN_TOL, err


def test_attn_32k(sf, attn_path):
    """32K context, 32 query / 8 KV heads, head_dim 128, 2+2 K/V with 4
    outlier key channels x10, top 1% tokens per query head."""
    Hq, Hkv, T, d = 32, 8, 32768, 128
    kv, ok, ov = _kv(sf, Hkv, T, d, 3000)
    qb = gen_query(4000, Hq, d)
    k = count_fraction(1, T)
    out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
    sel_n = sel_n.cpu().numpy()
    sel = sel.cpu().numpy()
    for g in range(Hkv):
        np.testing.assert_array_equal(sel[g, : sel_n[g]], ref["union"][g])
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref["out"]).max()
    assert err <= ATTN_TOL, err


def test_attn_128k_sampled_groups(sf, attn_path):
    """The bench's long-context launch configuration: 128K context, 32 query /
    8 KV heads, top 1% tokens per query head, all eight groups on the GPU;
    the oracle checks the first and the last KV head (union and outputs of
    their four query heads).  Quantization is per token-head row, so each
    sampled group is quantized on its own for the oracle."""
    Hq, Hkv, T, d = 32, 8, 131072, 128
    _skip_unless_applies(attn_path, Hq, Hkv, T)
    Kf, Vf, _ = gen_kv(3128, Hkv, T, d)
    kv = sf.QKV(sf.quantize_nested(dev(Kf.reshape(Hkv * T, d)), d, 2, 2, "by_row"),
                sf.quantize_nested(dev(Vf.reshape(Hkv * T, d)), d, 2, 2, "by_row"))
    qb = gen_query(4128, Hq, d)
    k = count_fraction(1, T)
    out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    out, sel, sel_n = out.cpu().numpy(), sel.cpu().numpy(), sel_n.cpu().numpy()
    grp = Hq // Hkv
    for g in (0, Hkv - 1):
        ok, ov = oquant.quantize_nested(Kf[g], d, 2, 2), oquant.quantize_nested(Vf[g], d, 2, 2)
        ref = oattn.attn_decode_refine(qb[g * grp:(g + 1) * grp], ok, ov, 1, T, k)
        assert sel_n[g] == len(ref["union"][0])
        np.testing.assert_array_equal(sel[g, : sel_n[g]], ref["union"][0])
        err = np.abs(out[g * grp:(g + 1) * grp].astype(np.float64) - ref["out"]).max()
        assert err <= ATTN_TOL, err


def test_attn_band_overflow(sf, attn_path):
    """Half the tokens of each KV head are copies of one token, and k puts the
    k-th largest key of query head 0 inside that tie: thousands of exactly
    tied candidates straddle the threshold (the cluster kernel's band then
    overflows its owner's shared memory into the workspace)."""
    Hq, Hkv, T, d = 8, 2, 8192, 128
    Kf, Vf, _ = gen_kv(91, Hkv, T, d)
    Kf[:, 0::2] = Kf[:, :1]
    Kf2, Vf2 = Kf.reshape(Hkv * T, d), Vf.reshape(Hkv * T, d)
    kv = sf.QKV(sf.quantize_nested(dev(Kf2), d, 2, 2, "by_row"), sf.quantize_nested(dev(Vf2), d, 2, 2, "by_row"))
    ok, ov = oquant.quantize_nested(Kf2, d, 2, 2), oquant.quantize_nested(Vf2, d, 2, 2)
    qb = gen_query(92, Hq, d)
    kap = oattn.selection_keys(oattn.bf16_to_f64(qb)[0], ok, slice(0, T))
    above = int((kap > kap[0]).sum())  # tokens ranked above the tied copies
    k = min(T // 2, above + 100)
    out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
    for g in range(Hkv):
        n = sel_n.cpu().numpy()[g]
        np.testing.assert_array_equal(sel.cpu().numpy()[g, :n], ref["union"][g])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() <= ATTN_TOL


def _wide_query(seed, Hq, d, scale_exp):
    """N(0, 1) query heads with one entry of each head scaled by 2^-scale_exp,
    so the nonzero exponents span about scale_exp binades or a few more."""
    q = np.random.default_rng(seed).standard_normal((Hq, d)).astype(np.float32)
    q[:, 5] = np.ldexp(np.where(q[:, 5] >= 0, 1.0, -1.0), -scale_exp).astype(np.float32) * np.abs(q[:, 0])
    return f32_to_bf16_bits(q)


def test_attn_wide_query_span(sf, attn_path):
    """Query heads whose exponents span 26 binades: beyond the integer-key
    range (15), within the exact fp64 range (33): the band is re-keyed with
    fp64 products and the selection must still equal the exact one."""
    Hq, Hkv, T, d = 8, 2, 6000, 128
    kv, ok, ov = _kv(sf, Hkv, T, d, 515)
    qb = _wide_query(516, Hq, d, 26)
    k = count_fraction(2, T)
    out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
    for g in range(Hkv):
        n = sel_n.cpu().numpy()[g]
        assert n == len(ref["union"][g])
        np.testing.assert_array_equal(sel.cpu().numpy()[g, :n], ref["union"][g])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() <= ATTN_TOL


def test_attn_flags_inexact_query_span(sf):
    """Query heads spanning 40 binades (beyond 33, where fp64 keys stop being
    exact): the definition's oracle refuses them, and every KV group reports
    -1 - (union length) in sel_n on both implementations."""
    Hq, Hkv, T, d = 8, 2, 4000, 128
    kv, ok, ov = _kv(sf, Hkv, T, d, 517)
    qb = _wide_query(518, Hq, d, 40)
    with pytest.raises(ValueError):
        oattn.attn_decode_refine(qb, ok, ov, Hkv, T, 40)
    for path in (sf.ATTN_PIPELINE, sf.ATTN_CLUSTER):
        sf.attn_set_path(path)
        try:
            out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, 40)
            torch.cuda.synchronize()
        finally:
            sf.attn_set_path(sf.ATTN_AUTO)
        sel_n = sel_n.cpu().numpy()
        sel = sel.cpu().numpy()
        for g in range(Hkv):
            assert sel_n[g] < 0
            U = -1 - sel_n[g]
            assert 40 <= U <= (Hq // Hkv) * 40
            u = sel[g, :U]
            assert np.all(np.diff(u) > 0) and u[0] >= 0 and u[-1] < T
        assert np.isfinite(out.cpu().numpy()).all()


def test_attn_ties(sf, attn_path):
    """Duplicate tokens give exactly tied keys; the lower token index wins."""
    Hq, Hkv, T, d = 8, 2, 600, 128
    Kf, Vf, _ = gen_kv(77, Hkv, T, d)
    for t in range(0, T, 5):
        Kf[:, t] = Kf[:, 0]
    Kf2, Vf2 = Kf.reshape(Hkv * T, d), Vf.reshape(Hkv * T, d)
    kv = sf.QKV(sf.quantize_nested(dev(Kf2), d, 2, 2, "by_row"), sf.quantize_nested(dev(Vf2), d, 2, 2, "by_row"))
    ok, ov = oquant.quantize_nested(Kf2, d, 2, 2), oquant.quantize_nested(Vf2, d, 2, 2)
    qb = gen_query(78, Hq, d)
    for k in (1, 13, 60, 200):
        out, sel, sel_n = sf.attn_decode_refine(bf16_dev(qb), kv, Hkv, T, k)
        torch.cuda.synchronize()
        ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
        for g in range(Hkv):
            n = sel_n.cpu().numpy()[g]
            np.testing.assert_array_equal(sel.cpu().numpy()[g, :n], ref["union"][g])
        assert np.abs(out.cpu().numpy() - ref["out"]).max() <= ATTN_TOL


@pytest.mark.parametrize("N,K,cap,pct", [(1024, 4096, 30, 3), (4096, 4096, 410, 3), (512, 8192, 50, 4),
                                         (2048, 14336, 1434, 3)])
def test_gemv_batch1_integer_path(sf, N, K, cap, pct):
    """Batch 1, 2-bit, K a multiple of 1024: the fixed-point DP4A kernel.  The
    activations mix zeros, values 2^-100 and outliers of 3e4 inside the same
    32-column slabs; the cache is small enough that some steps bypass."""
    G, b_r, b_f = 128, 2, 2
    W = gen_weight(700 + N + K, N, K)
    qw = sf.quantize_nested(dev(W), G, b_r, b_f)
    qz = oquant.quantize_nested(W, G, b_r, b_f)
    k = count_fraction(pct, K)
    cache = sf.RefineCache(K, N * b_f // 8, cap, k, _host_master(qw))
    orc = ocache.LRUCache(K, cap)
    outl = outlier_channels(800 + K, K, count_fraction("1/2", K))
    side = torch.cuda.Stream()
    for step in range(4):
        x = gen_activations(900 + step, 1, K, outl, 30.0)
        rng = np.random.default_rng(step)
        pos = rng.choice(K, size=24, replace=False)
        x[0, pos[:8]] = 0
        x[0, pos[8:16]] = f32_to_bf16_bits(np.full(8, 2.0 ** -100, np.float32))
        x[0, pos[16:]] = f32_to_bf16_bits(np.array([3e4, -3e4] * 4, np.float32))
        xd = bf16_dev(x)
        idx, n = sf.select_topk(xd, k)
        cache.prefetch(idx, n, torch.cuda.current_stream(), side)
        y = sf.gemv_refine(qw, xd, idx, n, cache=cache)
        y0 = sf.gemv_refine(qw, xd)
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        want = orc.step(S.tolist())
        assert cache.sets()["bypass"] == want["bypass"]
        y_ref, a = ogemv.gemv_refine(qz, x, S)
        _check_gemv(y.cpu().numpy(), y_ref, a)
        r0, a0 = ogemv.gemv_refine(qz, x, [])
        _check_gemv(y0.cpu().numpy(), r0, a0)
    cache.close()


def test_cache_group_matches_oracle(sf):
    """A group prefetch of three caches (different unit sizes and capacities,
    one of them overflowing into bypass) equals three independent LRU steps."""
    specs = [(4096, 1024, 410, 123), (4096, 256, 40, 123), (14336, 1024, 200, 430)]
    side = torch.cuda.Stream()
    entries, orcs, masters, xs = [], [], [], []
    for i, (K, unit, cap, k) in enumerate(specs):
        rng = np.random.default_rng(50 + i)
        m = torch.from_numpy(rng.integers(0, 2 ** 31, size=(K, unit // 4), dtype=np.int64).astype(np.int32))
        masters.append(m.pin_memory())
        cache = sf.RefineCache(K, unit, cap, k, masters[-1])
        idx = torch.zeros(k, dtype=torch.int32, device="cuda")
        n = torch.zeros(1, dtype=torch.int32, device="cuda")
        entries.append((cache, idx, n))
        orcs.append(ocache.LRUCache(K, cap))
    grp = sf.RefineGroup(entries)
    for step in range(6):
        sels = []
        for i, (K, unit, cap, k) in enumerate(specs):
            x = gen_activations(60 + 10 * step + i, 1, K, outlier_channels(70 + i, K, count_fraction("1/2", K)), 30.0)
            sf.select_topk(bf16_dev(x), k, entries[i][1], entries[i][2])
            sels.append(oselect.select_topk(x, k))
        grp.prefetch(torch.cuda.current_stream(), side)
        torch.cuda.synchronize()
        for i, (cache, idx, n) in enumerate(entries):
            want = orcs[i].step(sels[i].tolist())
            got = cache.sets()
            assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
            assert got["bypass"] == want["bypass"]
            assert {u: s for s, u in enumerate(cache.slots()) if u >= 0} == orcs[i].snapshot()
    grp.close()
    for cache, _, _ in entries:
        cache.close()


# ---- batch-1 fast path (prepared activations, several matrices per launch) -----

@pytest.mark.parametrize("K,pct", [(4096, 3), (14336, 3), (1024, 10)])
def test_select_act_matches_select(sf, K, pct):
    k = count_fraction(pct, K)
    x = gen_activations(31 + K, 1, K, outlier_channels(32, K, count_fraction("1/2", K)), 30.0)
    x[0, 5] = 0
    xd = bf16_dev(x)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    sf.select_topk_act(xd, k, idx, n, act)
    torch.cuda.synchronize()
    S = oselect.select_topk(x, k)
    np.testing.assert_array_equal(idx.cpu().numpy()[: int(n.item())], S)
    _check_prepared(act, x[0], S, K)
    act0 = torch.zeros_like(act)
    sf.act_prepare(xd, act0)
    torch.cuda.synchronize()
    _check_prepared(act0, x[0], [], K)


def _check_prepared(act, x_row, S, K):
    """The prepared activations against their documented layout: per
    256-channel slice, MMA B fragments holding balanced base-256 digits of
    per-group fixed point, group scale and sum, selection mask and counts."""
    a = act.cpu().numpy().view(np.uint32).reshape(K // 256, 528)
    mask = a[:, 520:528]
    sel = [256 * s + 32 * w + i for s in range(K // 256) for w in range(8) for i in range(32)
           if (int(mask[s, w]) >> i) & 1]
    assert sel == list(S)
    counts = np.array([sum(bin(int(m)).count("1") for m in mask[s]) for s in range(K // 256)])
    np.testing.assert_array_equal(a[:, 517], counts)
    np.testing.assert_array_equal(a[:, 516], np.concatenate([[0], np.cumsum(counts)[:-1]]))
    xf = (x_row.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for s in range(0, K // 256, max(1, K // 256 // 8)):
        digits = np.zeros((256, 3), dtype=np.int64)
        seen = np.zeros((256, 3), dtype=np.int64)
        for m in range(8):
            for lane in range(32):
                n, t = lane >> 2, lane & 3
                slot, mm, plane = m >> 2, m & 3, n & 3
                for r in range(2):
                    word = int(a[s, (m * 32 + lane) * 2 + r])
                    if (n >> 2) != slot or plane == 3:
                        assert word == 0
                        continue
                    for b in range(4):
                        ch = 128 * slot + 16 * (2 * t + (mm >> 1)) + 4 * b + 2 * (mm & 1) + r
                        d = (word >> (8 * b)) & 0xFF
                        digits[ch, plane] = d - 256 if d >= 128 else d
                        seen[ch, plane] += 1
        assert (seen == 1).all()
        assert np.abs(digits[:, 2]).max() <= 65
        X = digits[:, 0] + 256 * digits[:, 1] + 65536 * digits[:, 2]
        for grp in range(2):
            fscale = float(a[s, 512 + 2 * grp:513 + 2 * grp].view(np.float32)[0])
            gsum = float(a[s, 513 + 2 * grp:514 + 2 * grp].view(np.float32)[0])
            xs = xf[256 * s + 128 * grp:256 * s + 128 * grp + 128]
            Xg = X[128 * grp:128 * grp + 128]
            amax = np.abs(xs).max()
            if amax > 0:
                e = int(np.frexp(amax)[1])
                assert fscale == 2.0 ** (e - 22)
            assert np.all(np.abs(Xg * fscale - xs) <= fscale / 2)
            assert gsum == float(np.float32(float(np.float32(Xg.sum())) * fscale))


@pytest.mark.parametrize("K,Ns,cap_pct,pct", [(4096, (4096, 1024, 1024), 10, 3), (14336, (4096,), 10, 3),
                                              (4096, (2048, 512), 25, 5)])
def test_gemv_batch1_jobs_with_caches(sf, K, Ns, cap_pct, pct):
    G, b_r, b_f = 128, 2, 2
    k = count_fraction(pct, K)
    cap = count_fraction(cap_pct, K)
    mats = []
    for i, N in enumerate(Ns):
        W = gen_weight(1100 + 7 * i + K, N, K)
        qw = sf.quantize_nested(dev(W), G, b_r, b_f)
        rows = np.sort(np.random.default_rng(N + i).choice(N, size=min(N, 160), replace=False))
        mats.append(dict(qw=qw, qz=oquant.quantize_nested(W[rows], G, b_r, b_f), rows=rows,
                         cache=sf.RefineCache(K, N * b_f // 8, cap, k, _host_master(qw)),
                         orc=ocache.LRUCache(K, cap), y=torch.empty(N, dtype=torch.float32, device="cuda"),
                         y0=torch.empty(N, dtype=torch.float32, device="cuda")))
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    act0 = torch.zeros_like(act)
    grp = sf.RefineGroup([(m["cache"], idx, n) for m in mats])
    jobs = sf.Batch1Jobs([(m["qw"], m["cache"], False, m["y"]) for m in mats])
    jobs0 = sf.Batch1Jobs([(m["qw"], None, False, m["y0"]) for m in mats])
    side = torch.cuda.Stream()
    outl = outlier_channels(1200 + K, K, count_fraction("1/2", K))
    for step in range(3):
        x = gen_activations(1300 + step, 1, K, outl, 30.0)
        xd = bf16_dev(x)
        sf.select_topk_act(xd, k, idx, n, act)
        grp.prefetch(torch.cuda.current_stream(), side)
        jobs.run(xd, idx, n)
        jobs0.run(xd)
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        for m in mats:
            want = m["orc"].step(S.tolist())
            assert m["cache"].sets()["misses"] == want["misses"]
            y_ref, a = ogemv.gemv_refine(m["qz"], x, S)
            _check_gemv(m["y"].cpu().numpy()[None, m["rows"]], y_ref, a)
            r0, a0 = ogemv.gemv_refine(m["qz"], x, [])
            _check_gemv(m["y0"].cpu().numpy()[None, m["rows"]], r0, a0)
    grp.close()
    for m in mats:
        m["cache"].close()


@pytest.mark.parametrize("N,K,b_f", [(1024, 8192, 1), (512, 1024, 2), (2048, 4096, 1)])
def test_gemv_batch1_store_mode(sf, N, K, b_f):
    """Refinement read from the HBM store; b_f = 1 packs 16 rows in half a word."""
    G = 128
    W = gen_weight(1400 + K, N, K)
    qw = sf.quantize_nested(dev(W), G, 2, b_f)
    x = gen_activations(1401, 1, K, outlier_channels(1402, K, 40), 30.0)
    k = count_fraction(5, K)
    xd = bf16_dev(x)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    sf.select_topk_act(xd, k, idx, n, act)
    sf.gemv_refine_batch1([(qw, None, True, y)], xd, idx, n)
    torch.cuda.synchronize()
    y_ref, a = ogemv.gemv_refine(oquant.quantize_nested(W, G, 2, b_f), x, oselect.select_topk(x, k))
    _check_gemv(y.cpu().numpy()[None, :], y_ref, a)


def test_select_act_many_matches_single(sf):
    """One launch selecting four rows of different lengths equals four
    single-row selections (indices and prepared bytes) and the oracle."""
    specs = [(4096, 123), (4096, 123), (4096, 123), (14336, 430)]
    xs, single, many = [], [], []
    for i, (K, k) in enumerate(specs):
        x = gen_activations(1500 + i, 1, K, outlier_channels(1510 + i, K, count_fraction("1/2", K)), 30.0)
        xs.append(x)
        bufs = []
        for _ in range(2):
            bufs.append((torch.zeros(k, dtype=torch.int32, device="cuda"), torch.zeros(1, dtype=torch.int32, device="cuda"),
                         torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")))
        single.append(bufs[0])
        many.append(bufs[1])
    xds = [bf16_dev(x) for x in xs]
    for (K, k), xd, (idx, n, act) in zip(specs, xds, single):
        sf.select_topk_act(xd, k, idx, n, act)
    jobs = sf.SelectJobs([(xd, k, idx, n, act) for (K, k), xd, (idx, n, act) in zip(specs, xds, many)])
    jobs.run()
    torch.cuda.synchronize()
    for (K, k), x, a, b in zip(specs, xs, single, many):
        want = oselect.select_topk(x, k)
        np.testing.assert_array_equal(b[0].cpu().numpy()[: int(b[1].item())], want)
        np.testing.assert_array_equal(a[0].cpu().numpy()[: int(a[1].item())], want)
        np.testing.assert_array_equal(a[2].cpu().numpy(), b[2].cpu().numpy())
