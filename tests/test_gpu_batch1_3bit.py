"""GPU parity of the batch-1 tensor-core GEMV with 3-bit resident codes
(3-bit resident + 1-bit refinement, the full decode step's weight format)
and of its repacked resident layout.

Bit-exact: the repacked codes against the layout sf.h documents; selected
channels and cache sets.  Tolerance: |y - y_ref| <= 2e-3 * sum_j |w_eff x|
per output against the CPU oracle.
"""

import numpy as np
import pytest
import torch

from oracle import cache as ocache
from oracle import gemv as ogemv
from oracle import quant as oquant
from oracle import select as oselect
from workloads import count_fraction, f32_to_bf16_bits, gen_activations, gen_weight, outlier_channels

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
    worst = (err / np.maximum(bound, 1e-300)).max()
    assert np.all(err <= bound), f"worst err/bound = {worst:.3g}"


def _expected_pack3(codes):
    """The split layout of sf_gemv_pack_batch1 written out from its
    definition: per row and 256-channel slice, 16 words of low 2 bits
    (channel 16 w + 4 b + j at word w, bits 8 b + 2 j) and 8 words of high
    bits (word 16 + 2 t + slot, bit 8 b + 4 h + j for channel
    16 (8 slot + 2 t + h) + 4 b + j)."""
    N, K = codes.shape
    out = np.zeros((N, K // 256, 24), dtype=np.uint64)
    for c in range(256):
        v = codes[:, c::256].astype(np.uint64)  # [N][slices]
        w, b, j = c >> 4, (c >> 2) & 3, c & 3
        out[:, :, w] |= (v & 3) << np.uint64(8 * b + 2 * j)
        slot, t, h = w >> 3, (w & 7) >> 1, w & 1
        out[:, :, 16 + 2 * t + slot] |= (v >> 2) << np.uint64(8 * b + 4 * h + j)
    return out.astype(np.uint32).reshape(N, K * 3 // 32)


def test_pack_batch1_layout(sf):
    N, K = 96, 1024
    W = gen_weight(77, N, K)
    qw = sf.quantize_nested(dev(W), 128, 3, 1)
    sf.pack_batch1(qw)
    torch.cuda.synchronize()
    qz = oquant.quantize_nested(W, 128, 3, 1)
    np.testing.assert_array_equal(qw.res_b1.cpu().numpy().view(np.uint32), _expected_pack3(qz["q_r"]))
    # the canonical codes are left as they were
    np.testing.assert_array_equal(qw.res.cpu().numpy().view(np.uint32), oquant.pack_bits(qz["q_r"], 3))
    q2 = sf.quantize_nested(dev(W), 128, 2, 2)
    sf.pack_batch1(q2)
    assert q2.res_b1 is q2.res


def _mats(sf, K, Ns, seed, b_r=3, b_f=1, nrows=160):
    mats = []
    for i, N in enumerate(Ns):
        W = gen_weight(seed + 7 * i, N, K)
        qw = sf.pack_batch1(sf.quantize_nested(dev(W), 128, b_r, b_f))
        rows = np.sort(np.random.default_rng(N + i + seed).choice(N, size=min(N, nrows), replace=False))
        mats.append(dict(qw=qw, qz=oquant.quantize_nested(W[rows], 128, b_r, b_f), rows=rows,
                         y=torch.empty(N, dtype=torch.float32, device="cuda"),
                         y0=torch.empty(N, dtype=torch.float32, device="cuda")))
    return mats


@pytest.mark.parametrize("K,Ns,cap_pct,pct", [(4096, (4096, 1024, 1024), 10, 3), (14336, (4096,), 10, 3),
                                              (4096, (14336, 14336), 10, 3), (4096, (2048, 512), 25, 5)])
def test_gemv_batch1_3bit_jobs_with_caches(sf, K, Ns, cap_pct, pct):
    """Llama-3.1-8B q/k/v, down and gate/up shapes at 3+1 bits, top 3%, 10%
    LRU caches over three steps, plus the resident-only launch."""
    b_r, b_f = 3, 1
    k = count_fraction(pct, K)
    cap = count_fraction(cap_pct, K)
    mats = _mats(sf, K, Ns, 2100 + K)
    for m in mats:
        N = m["qw"].N
        m["cache"] = sf.RefineCache(K, N * b_f // 8, cap, k, m["qw"].ref.cpu().contiguous().pin_memory())
        m["orc"] = ocache.LRUCache(K, cap)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    act0 = torch.zeros_like(act)
    grp = sf.RefineGroup([(m["cache"], idx, n) for m in mats])
    jobs = sf.Batch1Jobs([(m["qw"], m["cache"], False, m["y"]) for m in mats])
    jobs0 = sf.Batch1Jobs([(m["qw"], None, False, m["y0"]) for m in mats])
    side = torch.cuda.Stream()
    outl = outlier_channels(2200 + K, K, count_fraction("1/2", K))
    for step in range(3):
        x = gen_activations(2300 + step, 1, K, outl, 30.0)
        xd = bf16_dev(x)
        sf.select_topk_act(xd, k, idx, n, act)
        grp.prefetch(torch.cuda.current_stream(), side)
        jobs.run(xd, idx, n)
        jobs0.run(xd)
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        for m in mats:
            want = m["orc"].step(S.tolist())
            got = m["cache"].sets()
            assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
            y_ref, a = ogemv.gemv_refine(m["qz"], x, S)
            _check_gemv(m["y"].cpu().numpy()[None, m["rows"]], y_ref, a)
            r0, a0 = ogemv.gemv_refine(m["qz"], x, [])
            _check_gemv(m["y0"].cpu().numpy()[None, m["rows"]], r0, a0)
    grp.close()
    for m in mats:
        m["cache"].close()


def test_gemv_batch1_3bit_lm_head_size(sf):
    """The LM head of the full decode step: 128256 x 4096, 3+1 bits, top 3%
    refined from the HBM store; 256 sampled rows checked, spread over the
    whole output (8016 row tiles on the grid)."""
    N, K = 128256, 4096
    k = count_fraction(3, K)
    mats = _mats(sf, K, (N,), 2500, nrows=256)
    m = mats[0]
    x = gen_activations(2501, 1, K, outlier_channels(2502, K, count_fraction("1/2", K)), 30.0)
    xd = bf16_dev(x)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    sf.select_topk_act(xd, k, idx, n, act)
    sf.gemv_refine_batch1([(m["qw"], None, True, m["y"])], xd, idx, n)
    torch.cuda.synchronize()
    y_ref, a = ogemv.gemv_refine(m["qz"], x, oselect.select_topk(x, k))
    _check_gemv(m["y"].cpu().numpy()[None, m["rows"]], y_ref, a)


@pytest.mark.parametrize("b_r,b_f", [(3, 1), (2, 2), (2, 1)])
def test_gemv_batch1_huge_selected_outliers(sf, b_r, b_f):
    """Selected channels of magnitude 1e5 (beyond the f16 range of the
    correction's operand split) in some slices, 3e4 in others: every output
    stays within the tolerance, none is NaN."""
    N, K = 1024, 4096
    k = count_fraction(3, K)
    mats = _mats(sf, K, (N,), 2600 + b_r + b_f, b_r=b_r, b_f=b_f, nrows=N)
    m = mats[0]
    x = gen_activations(2601, 1, K, outlier_channels(2602, K, count_fraction("1/2", K)), 30.0)
    x[0, [5, 300, 1800, 4000]] = f32_to_bf16_bits(np.array([1e5, -1e5, 2.5e5, -7e4], np.float32))
    x[0, [700, 2900]] = f32_to_bf16_bits(np.array([3e4, -3e4], np.float32))
    xd = bf16_dev(x)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    sf.select_topk_act(xd, k, idx, n, act)
    sf.gemv_refine_batch1([(m["qw"], None, True, m["y"])], xd, idx, n)
    torch.cuda.synchronize()
    S = oselect.select_topk(x, k)
    assert {5, 300, 1800, 4000} <= set(S.tolist())
    y = m["y"].cpu().numpy()
    assert np.all(np.isfinite(y))
    y_ref, a = ogemv.gemv_refine(m["qz"], x, S)
    _check_gemv(y[None, :], y_ref, a)


@pytest.mark.parametrize("b_r,b_f", [(3, 1), (2, 2)])
def test_gemv_batch1_deadline_caches(sf, b_r, b_f):
    """The deadline reading: each GEMV refines only the selected columns its
    cache held when the step started (oracle: C8), then the step's prefetch
    fetches the misses for later steps; four steps over q/k/v-shaped jobs."""
    K, Ns = 4096, (4096, 1024, 1024)
    k = count_fraction(3, K)
    cap = count_fraction(10, K)
    mats = _mats(sf, K, Ns, 2700 + b_r, b_r=b_r, b_f=b_f)
    for m in mats:
        N = m["qw"].N
        m["cache"] = sf.RefineCache(K, N * b_f // 8, cap, k, m["qw"].ref.cpu().contiguous().pin_memory())
        m["cache"].set_deadline(True)
        m["orc"] = ocache.LRUCache(K, cap)
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    grp = sf.RefineGroup([(m["cache"], idx, n) for m in mats])
    jobs = sf.Batch1Jobs([(m["qw"], m["cache"], False, m["y"]) for m in mats])
    side = torch.cuda.Stream()
    outl = outlier_channels(2800 + K, K, count_fraction("1/2", K))
    refined = 0
    for step in range(4):
        x = gen_activations(2900 + step, 1, K, outl, 30.0)
        xd = bf16_dev(x)
        sf.select_topk_act(xd, k, idx, n, act)
        jobs.run(xd, idx, n)                               # refines S ∩ cached
        grp.prefetch(torch.cuda.current_stream(), side)    # then fetches the misses
        torch.cuda.synchronize()
        S = oselect.select_topk(x, k)
        for m in mats:
            E = ocache.effective_set(S, m["orc"].snapshot())
            y_ref, a = ogemv.gemv_refine(m["qz"], x, E)
            _check_gemv(m["y"].cpu().numpy()[None, m["rows"]], y_ref, a)
            want = m["orc"].step(S.tolist())
            got = m["cache"].sets()
            assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
        refined += len(E)
    assert refined > 0                                     # later steps do refine cached columns
    # the generic GEMV refuses a cache in the deadline reading
    with pytest.raises(sf.SfError, match="deadline"):
        sf.gemv_refine(mats[0]["qw"], xd, idx, n, cache=mats[0]["cache"])
    grp.close()
    for m in mats:
        m["cache"].close()
