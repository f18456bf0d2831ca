"""GPU parity of sf_gemv_refine_batch1_produce: the batch-1 GEMV that makes
its own input row (residual add + RMSNorm, bf16 rounding, or the SiLU
product) and the row's top-k selection inside the launch.

Its contract is equality, bit for bit, with the stand-alone producer
(sf_norm_select, sf_round_select, sf_silu_mul_select) followed by
sf_gemv_refine_batch1 on the same row and selection, so the comparison is
exact: the bf16 row, the selection and its length, the updated residual and
every GEMV output.  Both paths are also checked against the CPU oracle on
sampled rows (2e-3 * sum |w_eff x|, as the other GEMV tests).
"""

import numpy as np
import pytest
import torch

from oracle import cache as ocache
from oracle import gemv as ogemv
from oracle import quant as oquant
from oracle import select as oselect
from workloads import count_fraction, gen_weight

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


def _mats(sf, K, Ns, seed, b_r, b_f, nrows=128):
    mats = []
    for i, N in enumerate(Ns):
        W = gen_weight(seed + 7 * i, N, K)
        qw = sf.pack_batch1(sf.quantize_nested(dev(W), 128, b_r, b_f))
        rows = np.sort(np.random.default_rng(seed + N + i).choice(N, size=min(N, nrows), replace=False))
        mats.append(dict(qw=qw, qz=oquant.quantize_nested(W[rows], 128, b_r, b_f), rows=rows,
                         y1=torch.empty(N, dtype=torch.float32, device="cuda"),
                         y2=torch.empty(N, dtype=torch.float32, device="cuda")))
    return mats


def _inputs(op, K, seed):
    """fp32 producer inputs on the device: a heavy-tailed row (a few channels
    x30) and, per op, the delta / weights / up projection."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(K, generator=g)
    hot = torch.randperm(K, generator=g)[: max(1, K // 200)]
    x[hot] *= 30.0
    extra = {}
    if op == "norm":
        extra["delta"] = torch.randn(K, generator=g) * 0.5
        extra["w"] = 0.5 + torch.rand(K, generator=g)
    elif op == "silu":
        extra["u"] = torch.randn(K, generator=g)
    return x.cuda(), {k: v.cuda() for k, v in extra.items()}


def _run_both(sf, op, K, k, x, extra, jobs1, jobs2, with_delta=True):
    """The stand-alone producer + GEMV (outputs y1) and the fused launch
    (outputs y2); returns both rows, selections, lengths and residuals."""
    rows = [torch.zeros(K, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    idx = [torch.full((max(k, 1),), -7, dtype=torch.int32, device="cuda") for _ in range(2)]
    n = [torch.full((1,), -9, dtype=torch.int32, device="cuda") for _ in range(2)]
    delta = extra.get("delta") if with_delta else None
    res1 = x.clone()
    res2 = torch.full_like(x, float("nan"))
    if op == "norm":
        sf.norm_select(res1, extra["w"], rows[0], k, idx[0], n[0], None, delta=delta)
        jobs2.run_produce(sf.PRODUCE_NORM, x, rows[1], k, idx[1], n[1], delta=delta, w=extra["w"], x_out=res2)
    elif op == "round":
        sf.round_select(x, rows[0], k, idx[0], n[0], None)
        jobs2.run_produce(sf.PRODUCE_ROUND, x, rows[1], k, idx[1], n[1])
    else:
        sf.silu_mul_select(x, extra["u"], rows[0], k, idx[0], n[0], None)
        jobs2.run_produce(sf.PRODUCE_SILU_MUL, x, rows[1], k, idx[1], n[1], u=extra["u"])
    jobs1.run(rows[0], idx[0], n[0])
    torch.cuda.synchronize()
    return rows, idx, n, res1, res2


def _assert_same(op, k, rows, idx, n, res1, res2, mats):
    assert torch.equal(rows[0].view(torch.int16), rows[1].view(torch.int16))
    assert int(n[0]) == int(n[1])
    m = max(int(n[0]), 0)
    assert torch.equal(idx[0][:m], idx[1][:m])
    if op == "norm":
        assert torch.equal(res1.view(torch.int32), res2.view(torch.int32))
    for mt in mats:
        assert torch.equal(mt["y1"].view(torch.int32), mt["y2"].view(torch.int32))


def _bits(row):
    return row.view(torch.int16).cpu().numpy().view(np.uint16).reshape(1, -1)


def _check_oracle(mt, xbits, S):
    y_ref, a = ogemv.gemv_refine(mt["qz"], xbits, S)
    err = np.abs(mt["y2"].cpu().numpy()[None, mt["rows"]].astype(np.float64) - y_ref)
    assert np.all(err <= GEMV_TOL * a)


@pytest.mark.parametrize("op,K,Ns,bits,pct", [
    ("norm", 4096, (4096, 1024, 1024), (3, 1), 3),     # q/k/v, Llama-3.1-8B at 3+1
    ("norm", 4096, (14336, 14336), (3, 1), 3),         # gate/up
    ("round", 4096, (4096,), (3, 1), 3),               # o
    ("silu", 14336, (4096,), (3, 1), 3),               # down: two K halves as a cluster pair
    ("norm", 4096, (4096, 1024, 1024), (2, 2), 3),     # 2+2 weights
    ("silu", 14336, (4096,), (2, 2), 3),               # 2+2 down: shared histogram rows
    ("round", 4096, (2048,), (2, 1), 20),              # a larger selection
    ("norm", 4096, (1024,), (3, 1), 0),                # nothing selected
])
def test_produce_matches_separate_store(sf, op, K, Ns, bits, pct):
    b_r, b_f = bits
    k = count_fraction(pct, K)
    mats = _mats(sf, K, Ns, 3100 + K + b_r, b_r, b_f)
    jobs1 = sf.Batch1Jobs([(m["qw"], None, True, m["y1"]) for m in mats])
    jobs2 = sf.Batch1Jobs([(m["qw"], None, True, m["y2"]) for m in mats])
    for rep, with_delta in enumerate((True, False) if op == "norm" else (True,)):
        x, extra = _inputs(op, K, 3200 + K + rep)
        got = _run_both(sf, op, K, k, x, extra, jobs1, jobs2, with_delta)
        _assert_same(op, k, *got, mats)
        xbits = _bits(got[0][0])
        S = oselect.select_topk(xbits, k)
        np.testing.assert_array_equal(got[1][1][: len(S)].cpu().numpy(), S)
        for mt in mats:
            _check_oracle(mt, xbits, S)


@pytest.mark.parametrize("op,K,Ns", [("norm", 4096, (4096, 1024, 1024)), ("silu", 14336, (4096,))])
def test_produce_matches_separate_deadline_caches(sf, op, K, Ns):
    """Deadline caches over four steps: each step both paths read the cache
    state as the step found it (the GEMVs run before the step's prefetch),
    and the cache sets follow the oracle's LRU."""
    b_r, b_f = 3, 1
    k = count_fraction(3, K)
    cap = count_fraction(10, K)
    mats = _mats(sf, K, Ns, 3300 + K, b_r, b_f)
    for m in mats:
        N = m["qw"].N
        m["cache"] = sf.RefineCache(K, N * b_f // 8, cap, k, m["qw"].ref.cpu().contiguous().pin_memory())
        m["cache"].set_deadline(True)
        m["orc"] = ocache.LRUCache(K, cap)
    jobs1 = sf.Batch1Jobs([(m["qw"], m["cache"], False, m["y1"]) for m in mats])
    jobs2 = sf.Batch1Jobs([(m["qw"], m["cache"], False, m["y2"]) for m in mats])
    side = torch.cuda.Stream()
    for step in range(4):
        x, extra = _inputs(op, K, 3400 + step)
        rows, idx, n, res1, res2 = _run_both(sf, op, K, k, x, extra, jobs1, jobs2)
        _assert_same(op, k, rows, idx, n, res1, res2, mats)
        # the step's prefetch from the fused launch's selection, for later steps
        grp = sf.RefineGroup([(m["cache"], idx[1], n[1]) for m in mats])
        grp.prefetch(torch.cuda.current_stream(), side)
        torch.cuda.synchronize()
        S = oselect.select_topk(_bits(rows[1]), k)
        for m in mats:
            want = m["orc"].step(S.tolist())
            got = m["cache"].sets()
            assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
        grp.close()
    for m in mats:
        m["cache"].close()


def test_produce_nan_row(sf):
    """A NaN in the row: both paths report n = -1 and fall back to the
    resident-only GEMV, with the same outputs."""
    K = 4096
    k = count_fraction(3, K)
    mats = _mats(sf, K, (1024,), 3500, 3, 1)
    jobs1 = sf.Batch1Jobs([(m["qw"], None, True, m["y1"]) for m in mats])
    jobs2 = sf.Batch1Jobs([(m["qw"], None, True, m["y2"]) for m in mats])
    x, extra = _inputs("round", K, 3501)
    x[1234] = float("nan")
    rows, idx, n, res1, res2 = _run_both(sf, "round", K, k, x, extra, jobs1, jobs2)
    assert int(n[0]) == -1 and int(n[1]) == -1
    assert torch.equal(rows[0].view(torch.int16), rows[1].view(torch.int16))
    for m in mats:  # the same bits, NaNs included
        assert torch.equal(m["y1"].view(torch.int32), m["y2"].view(torch.int32))


def test_produce_argument_checks(sf):
    """SF_EINVAL for an updated residual overlapping its inputs, a selection
    beyond the launch's scratch, and a cache in the blocking reading."""
    K = 4096
    mats = _mats(sf, K, (1024,), 3600, 2, 2)
    jobs = sf.Batch1Jobs([(m["qw"], None, True, m["y2"]) for m in mats])
    x, extra = _inputs("norm", K, 3601)
    row = torch.zeros(K, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(K, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="x_out"):
        jobs.run_produce(sf.PRODUCE_NORM, x, row, 10, idx, n, delta=extra["delta"], w=extra["w"], x_out=x)
    with pytest.raises(RuntimeError, match="k must be"):
        jobs.run_produce(sf.PRODUCE_ROUND, x, row, K, idx, n)
    m = mats[0]
    cache = sf.RefineCache(K, m["qw"].N * 2 // 8, 100, 10, m["qw"].ref.cpu().contiguous().pin_memory())
    try:
        jb = sf.Batch1Jobs([(m["qw"], cache, False, m["y2"])])
        with pytest.raises(RuntimeError, match="deadline"):
            jb.run_produce(sf.PRODUCE_ROUND, x, row, 10, idx, n)
    finally:
        cache.close()
