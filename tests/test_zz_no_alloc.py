"""The allocation-free attention entry point.

Callers that cannot allocate device memory when attention runs (a fixed,
pre-reserved memory pool, a plugin handed no scratch) use
sf_attn_decode_refine_noalloc, whose scratch is an array compiled into the
library.  Through the C ABI it must give the same selected tokens and the
same outputs (within the attention tolerance) as sf_attn_decode_refine with a
caller workspace, on two calls in a row -- the second call runs on whatever
the first left in the shared array -- and refuse sizes the array cannot hold.

This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _qkv(sf, Hkv, T, d, seed):
    from workloads import gen_kv
    Kf, Vf, _ = gen_kv(seed, Hkv, T, d)
    return sf.QKV(sf.quantize_nested(_dev(Kf.reshape(-1, d)), d, 2, 2, "by_row"),
                  sf.quantize_nested(_dev(Vf.reshape(-1, d)), d, 2, 2, "by_row"))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    from workloads import count_fraction, gen_query
    Hq, Hkv, d = 32, 8, 128
    for call, (T, seed) in enumerate([(8192, 11), (5000, 12)]):
        kv = _qkv(sf, Hkv, T, d, seed)
        q = _dev(gen_query(seed + 100, Hq, d).view(np.int16)).view(torch.bfloat16)
        k = count_fraction(1, T)
        ref_out, ref_sel, ref_n = sf.attn_decode_refine(q, kv, Hkv, T, k)
        out = torch.full((Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        sel = torch.full((Hkv, Hq // Hkv * k), -7, dtype=torch.int32, device="cuda")
        sel_n = torch.full((Hkv,), -7, dtype=torch.int32, device="cuda")
        sf.attn_decode_refine_noalloc(q, kv, Hkv, T, k, out, sel, sel_n)
        torch.cuda.synchronize()
        n_ref = ref_n.cpu().numpy()
        np.testing.assert_array_equal(sel_n.cpu().numpy(), n_ref)
        for g in range(Hkv):
            np.testing.assert_array_equal(sel[g, : n_ref[g]].cpu().numpy(), ref_sel[g, : n_ref[g]].cpu().numpy())
        err = (out - ref_out).abs().max().item()
        assert err <= ATTN_TOL, f"call {call}: max-abs difference {err}"


def test_noalloc_refuses_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    Hq, Hkv, d, T = 32, 8, 128, 131072
    need = sf.attn_workspace_size(Hq, Hkv, d, T, 1311)
    assert need > 24 * 2 ** 20
    kv = _qkv(sf, Hkv, 64, d, 5)        # the size check fires before any pointer is used
    q = torch.zeros((Hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((Hq, d), dtype=torch.float32, device="cuda")
    sel = torch.empty((Hkv, 4 * 1311), dtype=torch.int32, device="cuda")
    sel_n = torch.empty((Hkv,), dtype=torch.int32, device="cuda")
    with pytest.raises(sf.SfError, match="built-in array"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, T, 1311, out, sel, sel_n)


def test_noalloc_pipeline_path_against_oracle_on_two_calls():
    """The multi-kernel pipeline leans on the built-in array far more than the
    cluster kernel (scores, candidate lists, exact keys, split partials).  At
    Hq 32 and T 40000 its scratch still fits the array: two calls in a row
    through the pipeline must give the oracle's union sets and outputs for the
    sampled KV heads, and agree with the workspace entry point everywhere."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    from oracle import attn as oattn, quant as oquant
    from workloads import count_fraction, gen_kv, gen_query
    Hq, Hkv, d = 32, 8, 128
    grp = Hq // Hkv
    sf.attn_set_path(sf.ATTN_PIPELINE)
    try:
        for call, (T, seed) in enumerate([(34000, 21), (30001, 22)]):
            k = count_fraction(1, T)
            assert sf.attn_workspace_size(Hq, Hkv, d, T, k) <= 24 * 2 ** 20
            Kf, Vf, _ = gen_kv(seed, Hkv, T, d)
            kv = sf.QKV(sf.quantize_nested(_dev(Kf.reshape(-1, d)), d, 2, 2, "by_row"),
                        sf.quantize_nested(_dev(Vf.reshape(-1, d)), d, 2, 2, "by_row"))
            qb = gen_query(seed + 100, Hq, d)
            q = _dev(qb.view(np.int16)).view(torch.bfloat16)
            out = torch.full((Hq, d), float("nan"), dtype=torch.float32, device="cuda")
            sel = torch.full((Hkv, grp * k), -7, dtype=torch.int32, device="cuda")
            sel_n = torch.full((Hkv,), -7, dtype=torch.int32, device="cuda")
            sf.attn_decode_refine_noalloc(q, kv, Hkv, T, k, out, sel, sel_n)
            ref_out, ref_sel, ref_n = sf.attn_decode_refine(q, kv, Hkv, T, k)
            torch.cuda.synchronize()
            o, s, n = out.cpu().numpy(), sel.cpu().numpy(), sel_n.cpu().numpy()
            np.testing.assert_array_equal(n, ref_n.cpu().numpy())
            rs = ref_sel.cpu().numpy()
            for g in range(Hkv):
                np.testing.assert_array_equal(s[g, : n[g]], rs[g, : n[g]])
            assert np.abs(o - ref_out.cpu().numpy()).max() <= ATTN_TOL
            for g in (call, Hkv - 1 - call):
                ok, ov = oquant.quantize_nested(Kf[g], d, 2, 2), oquant.quantize_nested(Vf[g], d, 2, 2)
                ref = oattn.attn_decode_refine(qb[g * grp:(g + 1) * grp], ok, ov, 1, T, k)
                assert n[g] == len(ref["union"][0])
                np.testing.assert_array_equal(s[g, : n[g]], ref["union"][0])
                err = np.abs(o[g * grp:(g + 1) * grp].astype(np.float64) - ref["out"]).max()
                assert err <= ATTN_TOL, f"call {call}, KV head {g}: max-abs error {err}"
    finally:
        sf.attn_set_path(sf.ATTN_AUTO)
