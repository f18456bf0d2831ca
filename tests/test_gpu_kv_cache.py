"""GPU parity of refined attention that reads its refinement bits from a KV
refinement cache (sf_qkv.ref_cache): one cache unit per token-head, the
deadline reading (only the union tokens cached when the step starts are
refined; the misses are fetched for later steps, at most a budget per step,
the rest late), against the oracle's attention with an availability mask and
its LRU with a fetch budget.

Bit-exact: union sets, cache hit / miss / bypass sets, late counts.
Tolerance: attention max-abs error <= 2e-3.
"""

import numpy as np
import pytest
import torch

from oracle import attn as oattn
from oracle import cache as ocache
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _setup(sf, Hq, Hkv, T, S, d, seed, cap_pct):
    Kf, Vf, _ = gen_kv(seed, Hkv, S, d)           # S tokens allocated per head, the first T used
    k = sf.quantize_nested(dev(Kf.reshape(-1, d)), d, 2, 2, "by_row")
    v = sf.quantize_nested(dev(Vf.reshape(-1, d)), d, 2, 2, "by_row")
    master = torch.cat([k.ref.view(-1, 8), v.ref.view(-1, 8)], dim=1).cpu().contiguous().pin_memory()
    k_tokens = count_fraction(1, T)
    grp = Hq // Hkv
    cap = count_fraction(cap_pct, T)                # per KV head: one LRU each
    cache = sf.RefineCache(Hkv * S, 64, cap, grp * k_tokens, master, parts=Hkv)
    k.ref = v.ref = None                            # the stores are not read
    kvc = sf.QKV(k, v, row_stride=S, ref_cache=cache)
    ok = oquant.quantize_nested(Kf[:, :T].reshape(-1, d), d, 2, 2)
    ov = oquant.quantize_nested(Vf[:, :T].reshape(-1, d), d, 2, 2)
    return kvc, cache, ok, ov, k_tokens, cap


@pytest.mark.parametrize("path", ["auto", "pipeline"])
def test_attention_with_kv_refinement_cache(sf, path):
    Hq, Hkv, d, T, S = 32, 8, 128, 6000, 6040
    kvc, cache, ok, ov, k_tokens, cap = _setup(sf, Hq, Hkv, T, S, d, 811, 10)
    budget = 90                                     # per KV head and step
    cache.set_budget(budget)
    orcs = [ocache.LRUCache(Hkv * S, cap) for _ in range(Hkv)]   # the parts: units [g S, (g + 1) S)
    grp = Hq // Hkv
    units = torch.zeros(Hkv * grp * k_tokens, dtype=torch.int32, device="cuda")
    n_units = torch.zeros(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    sf.attn_set_path(sf.ATTN_PIPELINE if path == "pipeline" else sf.ATTN_AUTO)
    late = 0
    try:
        for step, qseed in enumerate([901, 901, 902, 901, 901]):
            qb = gen_query(qseed, Hq, d)
            avail = np.zeros((Hkv, T), dtype=bool)
            for orc in orcs:
                for u in orc.snapshot():
                    g, t = divmod(u, S)
                    if t < T:
                        avail[g, t] = True
            out, sel, sel_n = sf.attn_decode_refine(dev(qb.view(np.int16)).view(torch.bfloat16), kvc, Hkv, T,
                                                    k_tokens)
            sf.attn_union_units(sel, sel_n, Hkv, grp * k_tokens, S, units, n_units)
            cache.prefetch(units, n_units, torch.cuda.current_stream(), side)
            torch.cuda.synchronize()
            ref = oattn.attn_decode_refine(qb, ok, ov, Hkv, T, k_tokens, available=avail)
            sel_c, n_c = sel.cpu().numpy(), sel_n.cpu().numpy()
            want_units = []
            for g in range(Hkv):
                np.testing.assert_array_equal(sel_c[g, : n_c[g]], ref["union"][g])
                want_units += [g * S + int(t) for t in ref["union"][g]]
            assert int(n_units.item()) == len(want_units)
            np.testing.assert_array_equal(units.cpu().numpy()[: len(want_units)], want_units)
            err = np.abs(out.cpu().numpy().astype(np.float64) - ref["out"]).max()
            assert err <= ATTN_TOL, f"step {step}: max-abs error {err}"
            wants = [orcs[g].step([u for u in want_units if u // S == g], budget=budget) for g in range(Hkv)]
            got = cache.sets()
            assert got["hits"] == sum((w["hits"] for w in wants), [])
            assert got["misses"] == sum((w["misses"] for w in wants), [])
            assert got["bypass"] == sum((w["bypass"] for w in wants), [])
            late += sum(len(w["late"]) for w in wants)
            assert cache.stats().late == late
            if step == 0:
                assert not any(len(e) for e in ref["refined"])        # a cold cache refines nothing
            if step == 1:
                for g in range(Hkv):
                    assert len(ref["refined"][g]) == min(budget, len(ref["union"][g]))
        assert late > 0 and sum(o.hits for o in orcs) > 0
        got_slots = {u: s for s, u in enumerate(cache.slots()) if u >= 0}
        want_slots = {u: g * cap + sl for g, o in enumerate(orcs) for u, sl in o.snapshot().items()}
        assert got_slots == want_slots
    finally:
        sf.attn_set_path(sf.ATTN_AUTO)
        cache.close()


def test_kv_cache_refusals(sf):
    Hq, Hkv, d, T, S = 8, 2, 128, 512, 512
    kvc, cache, ok, ov, k_tokens, cap = _setup(sf, Hq, Hkv, T, S, d, 812, 10)
    q = torch.zeros((Hq, d), dtype=torch.bfloat16, device="cuda")
    sf.attn_set_path(sf.ATTN_CLUSTER)
    try:
        with pytest.raises(sf.SfError, match="ref_cache"):
            sf.attn_decode_refine(q, kvc, Hkv, T, k_tokens)
    finally:
        sf.attn_set_path(sf.ATTN_AUTO)
    # a cache with a fetch budget cannot serve a GEMV
    W = torch.randn(256, 256, device="cuda") * 0.02
    qw = sf.quantize_nested(W, 128, 2, 2)
    wc = sf.RefineCache(256, 256 * 2 // 8, 32, 8, qw.ref.cpu().contiguous().pin_memory())
    wc.set_budget(4)
    x = torch.randn(1, 256, device="cuda").to(torch.bfloat16)
    idx, n = sf.select_topk(x, 8)
    wc.prefetch(idx, n)
    with pytest.raises(sf.SfError, match="fetch budget"):
        sf.gemv_refine(qw, x, idx, n, cache=wc)
    torch.cuda.synchronize()
    wc.close()
    cache.close()


@pytest.mark.parametrize("t,b_f", [(17, 2), (0, 2), (63, 1)])
def test_kv_append_pair_cached(sf, t, b_f):
    """Key and value rows of token t in one launch: resident codes, scale and
    zero bit-exact against the oracle's quantizer; the refinement words reach
    the host master (K half, then V half of unit g S + t) through the side
    stream's copy; every other unit of the master keeps its sentinel."""
    Hkv, d, S, b_r = 8, 128, 64, 2
    rng = np.random.default_rng(900 + t + b_f)
    ksrc = (rng.standard_normal((Hkv, d)) * 2).astype(np.float32)
    vsrc = (rng.standard_normal((Hkv, d)) * 2).astype(np.float32)
    fw = d * b_f // 32
    unit = 2 * fw * 4
    master = torch.full((Hkv * S * unit,), 0xA5, dtype=torch.uint8).pin_memory()
    cache = sf.RefineCache(Hkv * S, unit, 8, 8, master)
    cache.preload(torch.tensor([2 * S + t, 5 * S + 3], dtype=torch.int32, device="cuda"))

    rows = Hkv * S
    kres = torch.full((rows, d * b_r // 32), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    vres = torch.full((rows, d * b_r // 32), 0x1E1E1E1E, dtype=torch.int32, device="cuda")
    ksc = torch.full((rows,), 7.0, dtype=torch.float16, device="cuda")
    kz = torch.full((rows,), 9.0, dtype=torch.float16, device="cuda")
    vsc = torch.full((rows,), 3.0, dtype=torch.float16, device="cuda")
    vz = torch.full((rows,), 5.0, dtype=torch.float16, device="cuda")

    class _Q:  # the views the binding reads
        def __init__(self, res, scale, zero):
            self.res, self.scale, self.zero = res, scale, zero

    side = torch.cuda.Stream()
    sf.kv_append_pair_cached(dev(ksrc), dev(vsrc), _Q(kres, ksc, kz), _Q(vres, vsc, vz), cache, S, t, b_r, b_f,
                             side=side)
    side.synchronize()
    torch.cuda.synchronize()
    for src, res, sc, z, half in ((ksrc, kres, ksc, kz, 0), (vsrc, vres, vsc, vz, 1)):
        want = oquant.pack_nested(oquant.quantize_nested(src, d, b_r, b_f), "by_row")
        res_np = res.cpu().numpy().view(np.uint32).reshape(Hkv, S, -1)
        np.testing.assert_array_equal(res_np[:, t], want["res"])
        np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint16).reshape(Hkv, S)[:, t],
                                      want["scale"][0].view(np.uint16))
        np.testing.assert_array_equal(z.cpu().numpy().view(np.uint16).reshape(Hkv, S)[:, t],
                                      want["zero"][0].view(np.uint16))
        m = master.numpy().view(np.uint32).reshape(Hkv, S, 2 * fw)
        np.testing.assert_array_equal(m[:, t, half * fw:(half + 1) * fw], want["ref"])
    keep = np.ones(S, bool)
    keep[t] = False
    assert np.all(master.numpy().reshape(Hkv, S, unit)[:, keep] == 0xA5)
    cache.close()


@pytest.mark.parametrize("t,pos", [(0, 0), (17, 131071), (63, 5)])
def test_rope_kv_append_pair_cached_equals_separate(sf, t, pos):
    """RoPE of q and k and the append of the rotated key and value rows in one
    launch equal sf_rope_qk followed by sf_kv_append_pair_cached, bit for bit:
    q, its bf16 copy, the rotated k, the resident codes, scales and zeros and
    the refinement words in the host master."""
    Hq, Hkv, d, S, b_r, b_f = 32, 8, 128, 64, 2, 2
    rng = np.random.default_rng(1300 + t)
    q0 = (rng.standard_normal((Hq, d)) * 3).astype(np.float32)
    k0 = (rng.standard_normal((Hkv, d)) * 3).astype(np.float32)
    v0 = (rng.standard_normal((Hkv, d)) * 3).astype(np.float32)
    fw = d * b_f // 32
    unit = 2 * fw * 4

    class _Q:  # the views the binding reads
        def __init__(self, res, scale, zero):
            self.res, self.scale, self.zero = res, scale, zero

    outs = []
    for fused in (False, True):
        master = torch.full((Hkv * S * unit,), 0xA5, dtype=torch.uint8).pin_memory()
        cache = sf.RefineCache(Hkv * S, unit, 8, 8, master)
        cache.preload(torch.tensor([3 * S + t], dtype=torch.int32, device="cuda"))
        rows = Hkv * S
        kq = _Q(torch.zeros((rows, d * b_r // 32), dtype=torch.int32, device="cuda"),
                torch.zeros((rows,), dtype=torch.float16, device="cuda"),
                torch.zeros((rows,), dtype=torch.float16, device="cuda"))
        vq = _Q(torch.zeros((rows, d * b_r // 32), dtype=torch.int32, device="cuda"),
                torch.zeros((rows,), dtype=torch.float16, device="cuda"),
                torch.zeros((rows,), dtype=torch.float16, device="cuda"))
        q, k, v = dev(q0), dev(k0), dev(v0)
        qb = torch.zeros((Hq, d), dtype=torch.bfloat16, device="cuda")
        side = torch.cuda.Stream()
        if fused:
            sf.rope_kv_append_pair_cached(q, k, v, kq, vq, cache, S, t, pos, b_r, b_f, q_bf16=qb, side=side)
        else:
            sf.rope_qk(q, k, pos, q_bf16=qb)
            sf.kv_append_pair_cached(k, v, kq, vq, cache, S, t, b_r, b_f, side=side)
        side.synchronize()
        torch.cuda.synchronize()
        outs.append([q.cpu(), qb.view(torch.int16).cpu(), k.cpu()] +
                    [a.cpu().view(torch.int16) if a.dtype == torch.float16 else a.cpu()
                     for a in (kq.res, kq.scale, kq.zero, vq.res, vq.scale, vq.zero)] + [master.clone()])
        cache.close()
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                           b.view(torch.int32) if b.dtype == torch.float32 else b)
