"""Parity of the decode-step elementwise operations (sf_add_rmsnorm, sf_rope,
sf_silu_mul) with the decode oracle (oracle.decode) on the GPU.

bf16 outputs are compared as bit patterns: the library rounds an fp64 value
once, the oracle rounds its own fp64 value once, so they agree except where
the two fp64 values straddle a rounding boundary; every output must be within
one bf16 step and almost all identical.  fp32 outputs are compared with the
oracle's fp64 values to fp32 precision."""

import numpy as np
import pytest
import torch

from oracle import decode as od

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    return sf


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _close_bf16(got, ref):
    diff = np.abs(got.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1, diff.max()
    assert np.mean(diff == 0) >= 0.999


@pytest.mark.parametrize("B,H,with_delta", [(1, 4096, True), (3, 4096, False), (2, 14336, True), (1, 33, True)])
def test_add_rmsnorm(sf, B, H, with_delta):
    rng = np.random.default_rng(100 + H + B)
    x = (rng.standard_normal((B, H)) * 3).astype(np.float32)
    delta = (rng.standard_normal((B, H)) * 0.5).astype(np.float32) if with_delta else None
    w = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    xd = torch.from_numpy(x.copy()).cuda()
    y = sf.add_rmsnorm(xd, torch.from_numpy(w).cuda(), 1e-5,
                       delta=torch.from_numpy(delta).cuda() if with_delta else None)
    torch.cuda.synchronize()
    xs = (x + delta).astype(np.float32) if with_delta else x   # the fp32 addition
    np.testing.assert_array_equal(xd.cpu().numpy(), xs)
    ref = od.f64_to_bf16_bits(od.rms_norm(xs.astype(np.float64), w.astype(np.float64), 1e-5))
    _close_bf16(_bits(y), ref)


@pytest.mark.parametrize("pos", [0, 1, 4097, 131071])
def test_rope(sf, pos):
    rng = np.random.default_rng(7 + pos)
    Hq, d = 32, 128
    x = rng.standard_normal((Hq, d)).astype(np.float32)
    xd = torch.from_numpy(x.copy()).cuda()
    y = torch.empty((Hq, d), dtype=torch.bfloat16, device="cuda")
    sf.rope(xd, pos, 500000.0, y=y)
    torch.cuda.synchronize()
    ref = od.rope(x.astype(np.float64), pos)
    np.testing.assert_allclose(xd.cpu().numpy(), ref, rtol=2 ** -23, atol=1e-7)
    _close_bf16(_bits(y), od.f64_to_bf16_bits(ref))


def test_rope_odd_head_count_and_small_dim(sf):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 6)).astype(np.float32)
    xd = torch.from_numpy(x.copy()).cuda()
    sf.rope(xd, 12345, 10000.0)
    torch.cuda.synchronize()
    np.testing.assert_allclose(xd.cpu().numpy(), od.rope(x.astype(np.float64), 12345, 10000.0), rtol=2 ** -23,
                               atol=1e-7)


@pytest.mark.parametrize("n", [1, 14336, 100003])
def test_silu_mul(sf, n):
    rng = np.random.default_rng(n)
    g = (rng.standard_normal(n) * 4).astype(np.float32)
    u = rng.standard_normal(n).astype(np.float32)
    y = sf.silu_mul(torch.from_numpy(g).cuda(), torch.from_numpy(u).cuda())
    torch.cuda.synchronize()
    ref = od.f64_to_bf16_bits(od.silu(g.astype(np.float64)) * u.astype(np.float64))
    _close_bf16(_bits(y), ref)


@pytest.mark.parametrize("Hkv,d,cap,t,b_r,b_f", [(8, 128, 64, 17, 2, 2), (8, 128, 64, 0, 2, 2),
                                                (8, 128, 64, 63, 2, 2), (3, 96, 5, 4, 3, 1), (1, 512, 2, 1, 2, 1)])
def test_kv_append_bit_exact(sf, Hkv, d, cap, t, b_r, b_f):
    """Token t of every head equals the oracle's packed quantization of the
    new rows; every other cache row keeps its sentinel."""
    from oracle import quant as oquant
    rng = np.random.default_rng(1000 + d + t)
    src = (rng.standard_normal((Hkv, d)) * 2).astype(np.float32)
    rows = Hkv * cap
    res = torch.full((rows, d * b_r // 32), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    ref = torch.full((rows, d * b_f // 32), 0x3C3C3C3C, dtype=torch.int32, device="cuda")
    scale = torch.full((rows,), 7.0, dtype=torch.float16, device="cuda")
    zero = torch.full((rows,), 9.0, dtype=torch.float16, device="cuda")
    sf.kv_append(torch.from_numpy(src).cuda(), res, ref, scale, zero, cap, t, b_r, b_f)
    torch.cuda.synchronize()
    want = oquant.pack_nested(oquant.quantize_nested(src, d, b_r, b_f), "by_row")
    res_np = res.cpu().numpy().view(np.uint32).reshape(Hkv, cap, -1)
    ref_np = ref.cpu().numpy().view(np.uint32).reshape(Hkv, cap, -1)
    sc_np = scale.cpu().numpy().view(np.uint16).reshape(Hkv, cap)
    z_np = zero.cpu().numpy().view(np.uint16).reshape(Hkv, cap)
    np.testing.assert_array_equal(res_np[:, t], want["res"])
    np.testing.assert_array_equal(ref_np[:, t], want["ref"])
    np.testing.assert_array_equal(sc_np[:, t], want["scale"][0].view(np.uint16))
    np.testing.assert_array_equal(z_np[:, t], want["zero"][0].view(np.uint16))
    keep = np.ones(cap, bool)
    keep[t] = False
    assert np.all(res_np[:, keep] == 0x5A5A5A5A) and np.all(ref_np[:, keep] == 0x3C3C3C3C)
    assert np.all(sc_np[:, keep] == np.float16(7.0).view(np.uint16)) and \
        np.all(z_np[:, keep] == np.float16(9.0).view(np.uint16))


def test_decode_ops_reject_bad_sizes(sf):
    x = torch.zeros((2, 7), dtype=torch.float32, device="cuda")
    with pytest.raises(sf.SfError):
        sf.rope(x, 0)                   # odd head dim
    with pytest.raises(sf.SfError):
        sf.rope(torch.zeros((2, 8), dtype=torch.float32, device="cuda"), -1)


# ---- producer + selection in one launch ---------------------------------------

def _selection_and_act(sf, y_bits_dev, K, k):
    """The stand-alone selection of a bf16 row (sf_select_topk_act)."""
    idx = torch.zeros(max(k, 1), dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda")
    if k > 0:
        sf.select_topk_act(y_bits_dev.view(1, K), k, idx, n, act)
    else:
        sf.act_prepare(y_bits_dev.view(1, K), act)
    return idx, n, act


def _fused_buffers(sf, K, k):
    return (torch.zeros(K, dtype=torch.bfloat16, device="cuda"), torch.full((max(k, 1),), -1, dtype=torch.int32,
            device="cuda"), torch.full((1,), -7, dtype=torch.int32, device="cuda"),
            torch.zeros(sf.act_bytes(K) // 4, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("H,k,with_delta", [(4096, 123, True), (14336, 430, False), (4096, 0, True)])
def test_norm_select_equals_norm_then_select(sf, H, k, with_delta):
    from oracle import select as oselect
    rng = np.random.default_rng(300 + H + k)
    x = (rng.standard_normal(H) * 3).astype(np.float32)
    x[rng.choice(H, 20, replace=False)] *= 30
    d = (rng.standard_normal(H)).astype(np.float32) if with_delta else None
    w = (1 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    x1, x2 = torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda()
    dd = torch.from_numpy(d).cuda() if with_delta else None
    wd = torch.from_numpy(w).cuda()
    y_ref = sf.add_rmsnorm(x1.view(1, H), wd, 1e-5, delta=dd.view(1, H) if with_delta else None)
    y, idx, n, act = _fused_buffers(sf, H, k)
    sf.norm_select(x2, wd, y, k, idx, n, act, eps=1e-5, delta=dd)
    torch.cuda.synchronize()
    assert torch.equal(x1, x2)                       # the residual update is the same fp32 addition
    _close_bf16(_bits(y), _bits(y_ref.view(-1)))
    yb = _bits(y)
    S = oselect.select_topk(yb[None, :], k)
    assert int(n.item()) == len(S)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(S)], S)
    i2, n2, act2 = _selection_and_act(sf, y, H, k)   # same row, same prepared bytes
    torch.cuda.synchronize()
    assert torch.equal(act, act2)


@pytest.mark.parametrize("K,k", [(4096, 123), (4096, 0)])
def test_round_select_equals_round_then_select(sf, K, k):
    rng = np.random.default_rng(400 + K + k)
    a = torch.from_numpy((rng.standard_normal(K) * 2).astype(np.float32)).cuda()
    y_ref = sf.round_bf16(a)
    y, idx, n, act = _fused_buffers(sf, K, k)
    sf.round_select(a, y, k, idx, n, act)
    i2, n2, act2 = _selection_and_act(sf, y_ref, K, k)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    if k:
        assert int(n.item()) == int(n2.item()) == k
        assert torch.equal(idx[:k], i2[:k])
    assert torch.equal(act, act2)


def test_silu_mul_select_equals_silu_mul_then_select(sf):
    K, k = 14336, 430
    rng = np.random.default_rng(500)
    g = torch.from_numpy((rng.standard_normal(K) * 2).astype(np.float32)).cuda()
    u = torch.from_numpy((rng.standard_normal(K) * 2).astype(np.float32)).cuda()
    y_ref = sf.silu_mul(g, u)
    y, idx, n, act = _fused_buffers(sf, K, k)
    sf.silu_mul_select(g, u, y, k, idx, n, act)
    i2, n2, act2 = _selection_and_act(sf, y_ref, K, k)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(idx[:k], i2[:k]) and int(n.item()) == k
    assert torch.equal(act, act2)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_silu_mul_select_wide_range(sf, seed):
    """The fused SiLU product takes an fp32 path with a rounding test and
    falls back to fp64 near bf16 midpoints: over gates in [-100, 100] and up
    projections spanning 60 binades (overflow and subnormal products
    included) it must match the stand-alone fp64 evaluation bit for bit."""
    K, k = 32768, 983
    rng = np.random.default_rng(700 + seed)
    g = torch.from_numpy(rng.uniform(-100.0, 100.0, K).astype(np.float32)).cuda()
    u = torch.from_numpy((np.sign(rng.standard_normal(K)) * 10.0 ** rng.uniform(-30, 30, K)).astype(np.float32)).cuda()
    y_ref = sf.silu_mul(g, u)
    y, idx, n, act = _fused_buffers(sf, K, k)
    sf.silu_mul_select(g, u, y, k, idx, n, act)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


def test_rope_qk_equals_two_ropes(sf):
    rng = np.random.default_rng(600)
    q = torch.from_numpy(rng.standard_normal((32, 128)).astype(np.float32)).cuda()
    k = torch.from_numpy(rng.standard_normal((8, 128)).astype(np.float32)).cuda()
    q2, k2 = q.clone(), k.clone()
    qb = torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda")
    qb2 = torch.zeros_like(qb)
    sf.rope(q, 131071, y=qb)
    sf.rope(k, 131071)
    sf.rope_qk(q2, k2, 131071, q_bf16=qb2)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(qb.view(torch.int16), qb2.view(torch.int16))
