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


def test_decode_ops_reject_bad_sizes(sf):
    x = torch.zeros((2, 7), dtype=torch.float32, device="cuda")
    with pytest.raises(sf.SfError):
        sf.rope(x, 0)                   # odd head dim
    with pytest.raises(sf.SfError):
        sf.rope(torch.zeros((2, 8), dtype=torch.float32, device="cuda"), -1)
