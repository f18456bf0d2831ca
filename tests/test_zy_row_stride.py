"""Attention over K/V views with a row stride: a cache allocated for more
tokens per KV head than the call reads (token t of head g at row
g * row_stride + t), as a decode loop that appends one token per step keeps
it.  Both implementations against the oracle on the T tokens read, and a
stride below T refused.

Collected after the parity suite and before the allocation-free entry
point's file, which runs last."""

import numpy as np
import pytest
import torch

from oracle import attn as oattn
from oracle import quant as oquant
from workloads import count_fraction, gen_kv, gen_query

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3


@pytest.fixture(scope="module")
def sf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    return sf


@pytest.fixture(params=["pipeline", "cluster"])
def attn_path(request, sf):
    sf.attn_set_path(sf.ATTN_PIPELINE if request.param == "pipeline" else sf.ATTN_CLUSTER)
    yield request.param
    sf.attn_set_path(sf.ATTN_AUTO)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16_dev(bits):
    return _dev(bits.view(np.int16)).view(torch.bfloat16)


def _cluster_applies(Hq, Hkv, T):
    return T <= 16 * (2048 if Hq // Hkv <= 4 else 1024)


@pytest.mark.parametrize("Hq,Hkv,T,cap", [(32, 8, 5000, 6144), (8, 2, 40000, 40960)])
def test_attn_row_stride(sf, attn_path, Hq, Hkv, T, cap):
    """K/V views of a cache allocated for cap tokens per KV head, of which
    the first T are read: equal to the oracle on those T."""
    if attn_path == "cluster" and not _cluster_applies(Hq, Hkv, T):
        pytest.skip("the cluster kernel does not apply to this size")
    d = 128
    Kf, Vf, _ = gen_kv(700 + T, Hkv, cap, d)
    kv = sf.QKV(sf.quantize_nested(_dev(Kf.reshape(Hkv * cap, d)), d, 2, 2, "by_row"),
                sf.quantize_nested(_dev(Vf.reshape(Hkv * cap, d)), d, 2, 2, "by_row"), row_stride=cap)
    qb = gen_query(701 + T, Hq, d)
    k = count_fraction(1, T)
    out, sel, sel_n = sf.attn_decode_refine(_bf16_dev(qb), kv, Hkv, T, k)
    torch.cuda.synchronize()
    ok = oquant.quantize_nested(Kf[:, :T].reshape(Hkv * T, d), d, 2, 2)
    ov = oquant.quantize_nested(Vf[:, :T].reshape(Hkv * T, d), d, 2, 2)
    ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k)
    sel_n, sel = sel_n.cpu().numpy(), sel.cpu().numpy()
    for g in range(Hkv):
        assert sel_n[g] == len(ref["union"][g])
        np.testing.assert_array_equal(sel[g, : sel_n[g]], ref["union"][g])
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref["out"]).max() <= ATTN_TOL


def test_attn_row_stride_below_t_is_rejected(sf):
    Kf, Vf, _ = gen_kv(5, 2, 300, 128)
    kv = sf.QKV(sf.quantize_nested(_dev(Kf.reshape(600, 128)), 128, 2, 2, "by_row"),
                sf.quantize_nested(_dev(Vf.reshape(600, 128)), 128, 2, 2, "by_row"), row_stride=299)
    with pytest.raises(sf.SfError):
        sf.attn_decode_refine(_bf16_dev(gen_query(6, 8, 128)), kv, 2, 300, 3)
