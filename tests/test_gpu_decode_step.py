"""GPU parity of the full decode step (quantized_gemv_kv_b200.decode): a
reduced Llama-shaped model (2 layers, hidden 512, MLP 1024, 4 query / 2 KV
heads of 128, vocab 1152, 3+1-bit weights, 2+2-bit KV) stepped through the
library, against the oracle.

Every op of the step is checked on the GPU's own inputs (teacher forcing, so
an error is caught where it arises): bf16 activations within one bf16 step of
the oracle and at least 99% identical; selected channels, appended K/V codes,
union token sets and cache hit / miss / bypass sets bit-exact; GEMV outputs
within 2e-3 * sum_j |w_eff x| per output; attention within 2e-3 max-abs.
The logits of one whole step from the embedding are then compared with
oracle.decode.decode_step itself.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import attn as oattn
from oracle import cache as ocache
from oracle import decode as od
from oracle import gemv as ogemv
from oracle import quant as oquant
from oracle import select as oselect
from workloads import f32_to_bf16_bits, gen_activations, gen_kv, gen_weight, outlier_channels

pytestmark = pytest.mark.gpu

GEMV_TOL = 2e-3
ATTN_TOL = 2e-3
P, P_TOK = Fraction(3, 100), Fraction(5, 100)
NL, H, F, HQ, HKV, D, V = 2, 512, 1024, 4, 2, 128, 1152
T0, CAP = 300, 320


@pytest.fixture(scope="module")
def sf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import quantized_gemv_kv_b200 as sf
    return sf


def _shape(sf):
    from quantized_gemv_kv_b200.decode import Shape
    return Shape(layers=NL, hidden=H, mlp=F, n_q=HQ, n_kv=HKV, head_dim=D, vocab=V)


def _host_model():
    """Seeded fp32 weights, norms and initial K/V (numpy), shared by the GPU
    model and the oracle."""
    rng = np.random.default_rng(4242)
    W, norms, kvs = {}, {}, {}
    shapes = dict(q=(HQ * D, H), k=(HKV * D, H), v=(HKV * D, H), o=(H, HQ * D), gate=(F, H), up=(F, H), down=(H, F))
    for l in range(NL):
        for i, (n, (N, K)) in enumerate(shapes.items()):
            W[(l, n)] = gen_weight(6000 + 16 * l + i, N, K)
        norms[(l, "norm1")] = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
        norms[(l, "norm2")] = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
        Kf, Vf, _ = gen_kv(6500 + l, HKV, T0, D)
        kvs[l] = (Kf, Vf)
    W[(-1, "head")] = gen_weight(6999, V, H)
    norms[(-1, "final")] = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    return W, norms, kvs


def _build(sf, host, **kw):
    from quantized_gemv_kv_b200.decode import DecodeModel
    W, norms, kvs = host
    return DecodeModel(_shape(sf), weight=lambda l, n, N, K: torch.from_numpy(W[(l, n)]).cuda(),
                       norm=lambda l, which: torch.from_numpy(norms[(l, which)]),
                       kv=lambda l: (torch.from_numpy(kvs[l][0]), torch.from_numpy(kvs[l][1])),
                       capacity=CAP, p=P, p_tok=P_TOK, record=True, **kw)


def _oracle_model(host):
    W, norms, kvs = host
    layers = []
    for l in range(NL):
        L = {n: oquant.quantize_nested(W[(l, n)], 128, 3, 1) for n in ("q", "k", "v", "o", "gate", "up", "down")}
        L["norm1"], L["norm2"] = norms[(l, "norm1")].astype(np.float64), norms[(l, "norm2")].astype(np.float64)
        layers.append(L)
    head = oquant.quantize_nested(W[(-1, "head")], 128, 3, 1)
    kv0 = [dict(k=oquant.quantize_nested(kvs[l][0].reshape(-1, D), D, 2, 2),
                v=oquant.quantize_nested(kvs[l][1].reshape(-1, D), D, 2, 2)) for l in range(NL)]
    return layers, head, norms[(-1, "final")].astype(np.float64), kv0


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f64(bits):
    return od.bf16_bits_to_f64(bits)


def _check_bf16(got_bits, want_f64):
    want = od.f64_to_bf16_bits(want_f64)
    g = _f64(got_bits)
    ulp = np.abs(od.bf16_bits_to_f64(want)) * 2.0 ** -7 + 1e-38
    assert np.all(np.abs(g - od.bf16_bits_to_f64(want)) <= ulp), "a bf16 value is more than one step off"
    assert np.mean(got_bits == want) >= 0.99


def _check_gemv(y_gpu, y_ref, abs_sum):
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    bound = GEMV_TOL * abs_sum
    assert np.all(err <= bound), f"worst err/bound = {(err / np.maximum(bound, 1e-300)).max():.3g}"


def _linear_check(qz, x_bits, idx, n, y_gpu, k, cached=None):
    """Selection bit-exact; the GEMV refines S, or in the deadline reading
    (``cached``: the units its cache held when the step started) S ∩ cached."""
    S = oselect.select_topk(x_bits[None, :], k)
    np.testing.assert_array_equal(idx[:n], S)
    E = S if cached is None else ocache.effective_set(S, cached)
    y_ref, a = ogemv.gemv_refine(qz, x_bits[None, :], E)
    _check_gemv(np.asarray(y_gpu)[None, :], y_ref, a)
    return S


def _append_rows(kv, new_rows, T):
    """The oracle cache after appending the quantized rows of token T."""
    return od.kv_append(kv, new_rows, HKV, T, 2, 2)


def _check_step(m, olayers, ohead, ofinal, okv, T, available=None, wcached=None):
    """Teacher-forced checks of one recorded step at position T; returns the
    oracle caches with the GPU's new token appended.  ``wcached[(l, slot)]``:
    the deadline reading's cached units of the matrices reading that input."""
    wc = (lambda l, slot: None) if wcached is None else (lambda l, slot: wcached[(l, slot)])
    k_tok = od.count_half_up(P_TOK, T + 1)
    nxt = []
    x_hist = m.x_hist.cpu().numpy().astype(np.float64)
    h_hist = m.h_hist.cpu().numpy().astype(np.float64)
    for l, (L, OL) in enumerate(zip(m.layers, olayers)):
        b = m.buf
        # RMSNorm 1
        n1 = _bits(b["attn_in"]["x"][l])
        _check_bf16(n1, od.rms_norm(x_hist[l], OL["norm1"]))
        # q, k, v
        raw = m.qkv_raw[l].cpu().numpy()
        idx, n = b["attn_in"]["idx"][l].cpu().numpy(), int(b["attn_in"]["n"][l].item())
        k_in = m.k_in["attn_in"]
        _linear_check(OL["q"], n1, idx, n, raw[:HQ * D], k_in, wc(l, "attn_in"))
        _linear_check(OL["k"], n1, idx, n, raw[HQ * D:(HQ + HKV) * D], k_in, wc(l, "attn_in"))
        _linear_check(OL["v"], n1, idx, n, raw[(HQ + HKV) * D:], k_in, wc(l, "attn_in"))
        q_raw = raw[:HQ * D].astype(np.float64).reshape(HQ, D)
        k_raw = raw[HQ * D:(HQ + HKV) * D].astype(np.float64).reshape(HKV, D)
        v_raw = raw[(HQ + HKV) * D:].astype(np.float32).reshape(HKV, D)
        # RoPE, append
        qb = _bits(m.q_bf[l]).reshape(HQ, D)
        _check_bf16(qb.reshape(-1), od.rope(q_raw, T).reshape(-1))
        k_rot = m.k_rot[l].cpu().numpy()
        np.testing.assert_allclose(k_rot, od.rope(k_raw, T), rtol=2.0 ** -22, atol=1e-30)
        okv2 = dict(k=_append_rows(okv[l]["k"], k_rot, T), v=_append_rows(okv[l]["v"], v_raw, T))
        kq, vq = L["kv"].k, L["kv"].v
        codes_k = oquant.pack_bits(oquant.quantize_nested(k_rot, D, 2, 2)["q_r"], 2)
        codes_v = oquant.pack_bits(oquant.quantize_nested(v_raw, D, 2, 2)["q_r"], 2)
        res_k = kq.res.cpu().numpy().view(np.uint32).reshape(HKV, CAP, -1)[:, T]
        res_v = vq.res.cpu().numpy().view(np.uint32).reshape(HKV, CAP, -1)[:, T]
        np.testing.assert_array_equal(res_k, codes_k)
        np.testing.assert_array_equal(res_v, codes_v)
        ref_k = oquant.pack_bits(oquant.quantize_nested(k_rot, D, 2, 2)["q_f"], 2)
        if L["kv_cache"] is None:
            got_ref = kq.ref.cpu().numpy().view(np.uint32).reshape(HKV, CAP, -1)[:, T]
        else:
            got_ref = L["kv_host"].numpy().view(np.uint32).reshape(HKV, CAP, -1)[:, T, :8]
        np.testing.assert_array_equal(got_ref, ref_k)
        # attention over the T + 1 tokens
        avail = None if available is None else available[l]
        ref = oattn.attn_decode_refine(qb, okv2["k"], okv2["v"], HKV, T + 1, k_tok, available=avail)
        un = m.union(l)
        for g in range(HKV):
            np.testing.assert_array_equal(un[g], ref["union"][g])
        att = m.att[l].cpu().numpy()
        assert np.abs(att - ref["out"]).max() <= ATTN_TOL
        # o projection and the residual
        ab = _bits(b["attn_out"]["x"][l])
        np.testing.assert_array_equal(ab, f32_to_bf16_bits(att.reshape(-1)))
        idx, n = b["attn_out"]["idx"][l].cpu().numpy(), int(b["attn_out"]["n"][l].item())
        _linear_check(OL["o"], ab, idx, n, L["o"].y.cpu().numpy(), m.k_in["attn_out"], wc(l, "attn_out"))
        np.testing.assert_array_equal(h_hist[l], (x_hist[l].astype(np.float32) + L["o"].y.cpu().numpy()))
        # MLP
        n2 = _bits(b["mlp_in"]["x"][l])
        _check_bf16(n2, od.rms_norm(h_hist[l], OL["norm2"]))
        idx, n = b["mlp_in"]["idx"][l].cpu().numpy(), int(b["mlp_in"]["n"][l].item())
        g = L["gate"].y.cpu().numpy()
        u = L["up"].y.cpu().numpy()
        _linear_check(OL["gate"], n2, idx, n, g, m.k_in["mlp_in"], wc(l, "mlp_in"))
        _linear_check(OL["up"], n2, idx, n, u, m.k_in["mlp_in"], wc(l, "mlp_in"))
        mid = _bits(b["mlp_mid"]["x"][l])
        _check_bf16(mid, od.silu(g.astype(np.float64)) * u.astype(np.float64))
        idx, n = b["mlp_mid"]["idx"][l].cpu().numpy(), int(b["mlp_mid"]["n"][l].item())
        dn = L["down"].y.cpu().numpy()
        _linear_check(OL["down"], mid, idx, n, dn, m.k_in["mlp_mid"], wc(l, "mlp_mid"))
        np.testing.assert_array_equal(x_hist[l + 1], h_hist[l].astype(np.float32) + dn)
        nxt.append(okv2)
    # final norm and LM head
    nf = _bits(m.buf["head"]["x"][0])
    _check_bf16(nf, od.rms_norm(x_hist[NL], ofinal))
    idx, n = m.buf["head"]["idx"][0].cpu().numpy(), int(m.buf["head"]["n"][0].item())
    _linear_check(ohead, nf, idx, n, m.logits.cpu().numpy(), m.k_in["head"], wc(-1, "head"))
    return nxt


def _embedding(seed):
    bits = gen_activations(seed, 1, H, outlier_channels(7100, H, 3), 30.0)[0]
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("fused", [False, True])
def test_decode_step_store_mode_against_oracle(sf, fused):
    """Refinement stores in device memory: the teacher-forced checks of one
    step, the logits of the whole step against oracle.decode.decode_step, and
    a graph replay that reproduces the eager step bit for bit; with the input
    rows made by stand-alone producers or inside the GEMV launches."""
    host = _host_model()
    m = _build(sf, host, fused_producers=fused)
    olayers, ohead, ofinal, okv = _oracle_model(host)
    x0 = _embedding(7000)
    m.x_in.copy_(torch.from_numpy(x0))
    T = T0
    m.step(T)
    torch.cuda.synchronize()
    _check_step(m, olayers, ohead, ofinal, okv, T)
    # the whole step from the embedding, as the oracle defines it
    logits, _ = od.decode_step(x0.astype(np.float64), olayers, okv, T, HQ, HKV, ofinal, ohead, P, P_TOK)
    got = m.logits.cpu().numpy().astype(np.float64)
    xb = m.buf["head"]["x"][0]
    S = oselect.select_topk(_bits(xb)[None, :], m.k_in["head"])
    _, a = ogemv.gemv_refine(ohead, _bits(xb)[None, :], S)
    # bound: the LM head's own tolerance, twice (its input is itself the end
    # of a chain of tolerances, re-rounded to bf16)
    _check_gemv(got[None, :], logits[None, :], 2 * a)
    # a captured graph of the same step gives the same bits
    first = m.logits.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        g.capture_begin(capture_error_mode="relaxed")
        m.step(T)
        g.capture_end()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(m.logits, first)
    del g
    m.close()


@pytest.mark.parametrize("deadline,lead,fused", [(False, False, False), (True, False, False), (True, True, False),
                                                 (True, True, True)])
def test_decode_step_cache_mode_against_oracle(sf, deadline, lead, fused):
    """Weight refinements behind 25% LRU caches and K/V refinements behind a
    20% KV refinement cache per layer with a fetch budget, over three decode
    steps at positions T0, T0+1, T0+2: every op of every step, the attention
    refining only the union tokens cached when the step starts, and the cache
    sets of one weight matrix per input and of each layer's KV cache.  With
    the deadline reading the GEMVs refine only the selected columns cached
    when the step starts (and never wait for a fetch); with fetch lead the
    q/k/v, gate/up and LM-head caches are first stepped with the channels
    predicted from the residual stream a block ahead.  ``fused``: the GEMVs
    make their input rows and selections in their own launches."""
    host = _host_model()
    budget = 12                                   # per KV head and step
    m = _build(sf, host, weight_cache_pct=25, kv_cache_pct=20, kv_budget=budget, weight_deadline=deadline,
               fetch_lead=lead, fused_producers=fused)
    olayers, ohead, ofinal, okv = _oracle_model(host)
    # oracle LRUs: q (attn_in), o, gate (mlp_in), down, head; the KV caches
    worcs = {slot: [ocache.LRUCache(K, od.count_half_up(Fraction(25, 100), K)) for _ in range(NL)]
             for slot, K in (("attn_in", H), ("attn_out", HQ * D), ("mlp_in", H), ("mlp_mid", F))}
    horc = ocache.LRUCache(H, od.count_half_up(Fraction(25, 100), H))
    # one LRU per layer and KV head, over the head's units [g CAP, (g + 1) CAP)
    kcap = od.count_half_up(Fraction(20, 100), CAP)
    korcs = [[ocache.LRUCache(HKV * CAP, kcap) for _ in range(HKV)] for _ in range(NL)]
    first_of = {"attn_in": "q", "attn_out": "o", "mlp_in": "gate", "mlp_mid": "down"}
    for step in range(3):
        T = T0 + step
        avail = []
        for l in range(NL):
            a = np.zeros((HKV, T + 1), dtype=bool)
            for o in korcs[l]:
                for u in o.snapshot():
                    gh, t = divmod(u, CAP)
                    if t <= T:
                        a[gh, t] = True
            avail.append(a)
        m.x_in.copy_(torch.from_numpy(_embedding(7200 + step)))
        m.step(T)
        torch.cuda.synchronize()
        m.sync()
        if lead:
            # the predictions: each from the residual as it stood (teacher
            # forced), selected exactly, and stepped into the caches first
            xh, hh = m.x_hist.cpu().numpy().astype(np.float64), m.h_hist.cpu().numpy().astype(np.float64)
            preds = [("mlp_in", l, xh[l], olayers[l]["norm2"]) for l in range(NL)]
            preds += [("attn_in", l + 1, hh[l], olayers[l + 1]["norm1"]) for l in range(NL - 1)]
            preds += [("head", -1, hh[NL - 1], ofinal)]
            for slot, l, resid, wn in preds:
                pr = m.pred[slot]
                li = max(l, 0)
                pb = _bits(pr["x"][li])
                _check_bf16(pb, od.rms_norm(resid, wn))
                S = oselect.select_topk(pb[None, :], m.k_in[slot])
                np.testing.assert_array_equal(pr["idx"][li].cpu().numpy()[: int(pr["n"][li].item())], S)
                (horc if slot == "head" else worcs[slot][l]).step(S.tolist())
        wcached = None
        if deadline:
            wcached = {(l, slot): set(orcs[l].snapshot()) for slot, orcs in worcs.items() for l in range(NL)}
            wcached[(-1, "head")] = set(horc.snapshot())
        okv = _check_step(m, olayers, ohead, ofinal, okv, T, available=avail, wcached=wcached)
        for slot, orcs in worcs.items():
            for l in range(NL):
                b = m.buf[slot]
                S = b["idx"][l].cpu().numpy()[: int(b["n"][l].item())].tolist()
                want = orcs[l].step(S)
                got = m.layers[l][first_of[slot]].cache.sets()
                assert got["hits"] == want["hits"] and got["misses"] == want["misses"]
                assert got["bypass"] == want["bypass"]
        hb = m.buf["head"]
        want = horc.step(hb["idx"][0].cpu().numpy()[: int(hb["n"][0].item())].tolist())
        assert m.head.cache.sets()["misses"] == want["misses"]
        for l in range(NL):
            wants = [korcs[l][g].step([g * CAP + int(t) for t in u], budget=budget)
                     for g, u in enumerate(m.union(l))]
            got = m.layers[l]["kv_cache"].sets()
            assert got["hits"] == sum((w["hits"] for w in wants), [])
            assert got["misses"] == sum((w["misses"] for w in wants), [])
            assert got["bypass"] == sum((w["bypass"] for w in wants), [])
    ko = [o for lo in korcs for o in lo]
    assert sum(o.late for o in ko) > 0 and sum(o.hits for o in ko) > 0
    assert m.cache_totals("kv")["late"] == sum(o.late for o in ko)
    m.close()
