"""Pins for the oracle's refined decode attention (CPU only).

* refining every token (k = T) equals torch's scaled_dot_product_attention
  in fp64 on full-code K/V (a library routine); k = 0 equals it on
  resident K/V;
* the selection key is checked against exact rational arithmetic
  (fractions.Fraction) on a small case, including the tie-break;
* selected tokens are the ones with the largest resident attention scores
  computed independently with torch in fp64;
* the exactness precondition on the query's exponent span is enforced.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import attn, quant
from workloads import gen_kv, gen_query, count_fraction, f32_to_bf16_bits


def _quant_kv(Kf, Vf, b_r=2, b_f=2):
    Hkv, T, d = Kf.shape
    qk = quant.quantize_nested(Kf.reshape(Hkv * T, d), d, b_r, b_f)
    qv = quant.quantize_nested(Vf.reshape(Hkv * T, d), d, b_r, b_f)
    return qk, qv


def _sdpa(q, k, v, Hkv):
    Hq, d = q.shape
    grp = Hq // Hkv
    qt = torch.from_numpy(q).reshape(Hkv, grp, 1, d)
    kt = torch.from_numpy(k).reshape(Hkv, 1, -1, d).expand(Hkv, grp, -1, d)
    vt = torch.from_numpy(v).reshape(Hkv, 1, -1, d).expand(Hkv, grp, -1, d)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    return o.reshape(Hq, d).numpy()


@pytest.mark.parametrize("Hq,Hkv,T,d", [(8, 2, 96, 64), (4, 4, 50, 32)])
def test_all_and_none_match_sdpa(Hq, Hkv, T, d):
    Kf, Vf, _ = gen_kv(71, Hkv, T, d, n_outlier_ch=2)
    qb = gen_query(72, Hq, d)
    qk, qv = _quant_kv(Kf, Vf)
    q = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r_all = attn.attn_decode_refine(qb, qk, qv, Hkv, T, T)
    np.testing.assert_allclose(r_all["out"], _sdpa(q, quant.dequant_full(qk), quant.dequant_full(qv), Hkv),
                               rtol=1e-10, atol=1e-12)
    assert all(len(u) == T for u in r_all["union"])
    r_none = attn.attn_decode_refine(qb, qk, qv, Hkv, T, 0)
    np.testing.assert_allclose(r_none["out"], _sdpa(q, quant.dequant_resident(qk),
                                                    quant.dequant_resident(qv), Hkv), rtol=1e-10, atol=1e-12)
    assert all(len(u) == 0 for u in r_none["union"])


def test_keys_exact_rational_and_tiebreak():
    Hkv, T, d, Hq = 1, 40, 16, 2
    Kf, Vf, _ = gen_kv(81, Hkv, T, d, n_outlier_ch=1)
    Kf[0, 7] = Kf[0, 3]          # duplicate tokens -> identical codes -> exact key ties
    Kf[0, 30] = Kf[0, 3]
    qk, qv = _quant_kv(Kf, Vf)
    qb = gen_query(82, Hq, d)
    k = 6
    r = attn.attn_decode_refine(qb, qk, qv, Hkv, T, k)
    qf = (qb.astype(np.uint32) << 16).view(np.float32)
    for h in range(Hq):
        keys = []
        for t in range(T):
            s = Fraction(float(qk["scale"][0, t]))
            z = Fraction(float(qk["zero"][0, t]))
            E = sum(Fraction(float(qf[h, j])) * (int(qk["q_r"][t, j]) * 4 + Fraction(3, 2) - z) for j in range(d))
            keys.append(s * E)
        order = sorted(range(T), key=lambda t: (-keys[t], t))
        assert r["sel"][h].tolist() == sorted(order[:k])
        kap = attn.selection_keys(qf[h].astype(np.float64), qk, slice(0, T))
        for t in range(T):   # exact E, then one rounding of s*E
            assert kap[t] == float(keys[t])


def test_selection_follows_resident_scores():
    Hkv, T, d, Hq = 2, 1024, 128, 8
    Kf, Vf, _ = gen_kv(91, Hkv, T, d)
    qk, qv = _quant_kv(Kf, Vf)
    qb = gen_query(92, Hq, d)
    k = count_fraction(1, T)
    r = attn.attn_decode_refine(qb, qk, qv, Hkv, T, k)
    q = torch.from_numpy((qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    kres = torch.from_numpy(quant.dequant_resident(qk)).reshape(Hkv, T, d)
    grp = Hq // Hkv
    for h in range(Hq):
        s = (kres[h // grp] @ q[h]) / math.sqrt(d)
        sel = torch.from_numpy(r["sel"][h].astype(np.int64))
        mask = torch.ones(T, dtype=torch.bool)
        mask[sel] = False
        assert len(sel) == k
        assert s[sel].min() >= s[mask].max() - 1e-9
    for g in range(Hkv):
        want = sorted(set().union(*[set(r["sel"][h].tolist()) for h in range(g * grp, (g + 1) * grp)]))
        assert r["union"][g].tolist() == want


def test_span_precondition():
    q = np.zeros((1, 128))
    q[0, 0] = 2.0 ** 20
    q[0, 1] = 2.0 ** -20
    with pytest.raises(ValueError):
        attn.check_exact_span(q, 4, 128)
    q[0, 1] = 2.0 ** -5
    attn.check_exact_span(q, 4, 128)


def test_refinement_reduces_error():
    Hkv, T, d, Hq = 2, 2048, 128, 8
    Kf, Vf, _ = gen_kv(101, Hkv, T, d)
    qk, qv = _quant_kv(Kf, Vf)
    qb = gen_query(102, Hq, d)
    q = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = _sdpa(q, Kf.reshape(-1, d).astype(np.float64), Vf.reshape(-1, d).astype(np.float64), Hkv)
    e_ref = np.abs(attn.attn_decode_refine(qb, qk, qv, Hkv, T, count_fraction(1, T))["out"] - exact).mean()
    e_res = np.abs(attn.attn_decode_refine(qb, qk, qv, Hkv, T, 0)["out"] - exact).mean()
    assert e_ref < e_res


def test_available_mask_refines_only_cached_union_tokens():
    """A7: with a per-token availability mask the union is unchanged and
    only its available tokens take full-code K and V; all available equals
    A5, none available gives the resident attention.  The mixed case is
    checked against library softmax on K/V assembled here token by token."""
    from scipy.special import softmax
    from oracle.quant import dequant_full, dequant_resident, quantize_nested
    from workloads import gen_kv, gen_query
    Hq, Hkv, T, d, k = 8, 2, 300, 32, 20
    Kf, Vf, _ = gen_kv(71, Hkv, T, d)
    qk, qv = quantize_nested(Kf.reshape(-1, d), d, 2, 2), quantize_nested(Vf.reshape(-1, d), d, 2, 2)
    qb = gen_query(72, Hq, d)
    attn_decode_refine = attn.attn_decode_refine
    full = attn_decode_refine(qb, qk, qv, Hkv, T, k)
    r_all = attn_decode_refine(qb, qk, qv, Hkv, T, k, available=np.ones((Hkv, T), bool))
    np.testing.assert_array_equal(r_all["out"], full["out"])
    r_none = attn_decode_refine(qb, qk, qv, Hkv, T, k, available=np.zeros((Hkv, T), bool))
    res = attn_decode_refine(qb, qk, qv, Hkv, T, k, refine=False)
    np.testing.assert_allclose(r_none["out"], res["out"], rtol=0, atol=1e-12)
    for g in range(Hkv):
        np.testing.assert_array_equal(r_none["union"][g], full["union"][g])
        assert r_none["refined"][g].size == 0
    avail = np.random.default_rng(73).random((Hkv, T)) < 0.5
    r = attn_decode_refine(qb, qk, qv, Hkv, T, k, available=avail)
    kf, kr, vf, vr = dequant_full(qk), dequant_resident(qk), dequant_full(qv), dequant_resident(qv)
    q = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    grp = Hq // Hkv
    for g in range(Hkv):
        U = set(full["union"][g].tolist())
        assert r["refined"][g].tolist() == sorted(t for t in U if avail[g, t])
        use_full = np.array([t in U and avail[g, t] for t in range(T)])
        Kg = np.where(use_full[:, None], kf[g * T:(g + 1) * T], kr[g * T:(g + 1) * T])
        Vg = np.where(use_full[:, None], vf[g * T:(g + 1) * T], vr[g * T:(g + 1) * T])
        for h in range(g * grp, (g + 1) * grp):
            want = softmax(Kg @ q[h] / np.sqrt(d)) @ Vg
            np.testing.assert_allclose(r["out"][h], want, rtol=1e-10, atol=1e-12)
