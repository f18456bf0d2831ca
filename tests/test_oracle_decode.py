"""Pins of the decode-step oracle (oracle.decode): closed forms, identities
and the two extremes of refinement against a plain transformer layer written
independently here (RoPE by complex multiplication, library softmax and
sigmoid)."""

from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit, softmax

from oracle import decode as od
from oracle.quant import dequant_full, dequant_resident, quantize_nested
from workloads import f32_to_bf16_bits


def test_bf16_rounding_ties_to_even():
    one = 1.0
    ulp = 2.0 ** -7                      # bf16 spacing at 1
    vals = np.array([one, one + ulp / 2, one + 1.5 * ulp, -(one + ulp / 2), 3.0, 0.0])
    bits = od.f64_to_bf16_bits(vals)
    # 1 + ulp/2 ties to 1 (even), 1 + 1.5 ulp ties to 1 + 2 ulp (even)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xBF80, 0x4040, 0x0000]


def test_bf16_rounding_matches_fp32_path_on_fp32_values():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(10000).astype(np.float32)
    np.testing.assert_array_equal(od.f64_to_bf16_bits(x.astype(np.float64)), f32_to_bf16_bits(x))


def test_count_half_up():
    assert od.count_half_up(Fraction(5, 100), 512) == 26
    assert od.count_half_up(Fraction(3, 100), 4096) == 123
    assert od.count_half_up(Fraction(3, 100), 14336) == 430
    assert od.count_half_up(Fraction(1, 100), 32768) == 328
    assert od.count_half_up(Fraction(1, 100), 131072) == 1311
    assert od.count_half_up(Fraction(1, 2), 1) == 1       # exact half rounds up
    assert od.count_half_up(Fraction(0), 100) == 0


def test_rms_norm_closed_forms():
    c = -2.5
    y = od.rms_norm(np.full(8, c), np.ones(8), eps=0.0)
    np.testing.assert_allclose(y, np.full(8, -1.0), rtol=0, atol=1e-15)
    y = od.rms_norm(np.array([3.0, 4.0]), np.array([1.0, 2.0]), eps=0.0)
    r = np.sqrt(12.5)                    # mean of 9 and 16
    np.testing.assert_allclose(y, [3.0 / r, 8.0 / r], rtol=1e-15)
    # eps enters under the root
    y = od.rms_norm(np.array([1.0, 1.0]), np.ones(2), eps=1.0)
    np.testing.assert_allclose(y, [1.0 / np.sqrt(2.0)] * 2, rtol=1e-15)


def test_rope_values_and_identities():
    x = np.zeros((1, 4))
    x[0, 0] = 1.0
    y = od.rope(x, 1)                    # dims 0 and 2 rotate by 1 radian
    np.testing.assert_allclose(y[0], [0.5403023058681398, 0.0, 0.8414709848078965, 0.0], atol=1e-15)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((3, 128))
    np.testing.assert_array_equal(od.rope(q, 0), q)
    y = od.rope(q, 777)
    np.testing.assert_allclose(np.hypot(y[:, :64], y[:, 64:]), np.hypot(q[:, :64], q[:, 64:]), rtol=1e-13)
    # scores depend on the position difference only
    k = rng.standard_normal((3, 128))
    for m, n in ((5, 2), (1000, 17), (131071, 130000)):
        a = np.sum(od.rope(q, m) * od.rope(k, n), axis=1)
        b = np.sum(od.rope(q, m - n) * k, axis=1)
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)


def test_silu_identities():
    rng = np.random.default_rng(5)
    z = rng.standard_normal(1000) * 4
    np.testing.assert_allclose(od.silu(z) - od.silu(-z), z, rtol=1e-13, atol=1e-13)
    assert od.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(od.silu(np.array([40.0])), [40.0], rtol=1e-15)


def test_kv_append_inserts_token_rows():
    rng = np.random.default_rng(11)
    Hkv, T, d = 2, 5, 16
    old = rng.standard_normal((Hkv * T, d)).astype(np.float32)
    qz = quantize_nested(old, d, 2, 2)
    new = rng.standard_normal((Hkv, d)).astype(np.float32)
    out = od.kv_append(qz, new, Hkv, T, 2, 2)
    ref = quantize_nested(np.concatenate([old.reshape(Hkv, T, d), new[:, None, :]], axis=1).reshape(-1, d),
                          d, 2, 2)
    for key in ("q", "q_r", "q_f", "scale", "zero"):
        np.testing.assert_array_equal(out[key], ref[key])


# ---- the two extremes of refinement against a plain layer --------------------

def _bf16(v):
    return (f32_to_bf16_bits(np.asarray(v, dtype=np.float32)).astype(np.uint32) << 16).view(np.float32) \
        .astype(np.float64)


def _rope_complex(x, pos, theta=500000.0):
    d = x.shape[-1]
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    z = z * np.exp(1j * pos * theta ** (-np.arange(d // 2) * 2.0 / d))
    return np.concatenate([z.real, z.imag], axis=-1)


def _plain_layer(x, W, K, V, Hq, Hkv, T, eps=1e-5):
    """Textbook pre-norm Llama layer on dequantized weights W[name] and the
    cache's K, V values [Hkv][T + 1][d] (the new token's rows included)."""
    d = W["q"].shape[0] // Hq

    def norm(v, w):
        return w * v / np.sqrt(np.dot(v, v) / v.size + eps)

    n1 = _bf16(norm(x, W["norm1"]))
    q = _bf16(_rope_complex((W["q"] @ n1).reshape(Hq, d), T))
    att = np.empty((Hq, d))
    for h in range(Hq):
        g = h // (Hq // Hkv)
        att[h] = softmax(K[g] @ q[h] / np.sqrt(d)) @ V[g]
    hres = x + W["o"] @ _bf16(att.reshape(-1))
    n2 = _bf16(norm(hres, W["norm2"]))
    a, b = W["gate"] @ n2, W["up"] @ n2
    return hres + W["down"] @ _bf16(a * expit(a) * b)


def _tiny_model(seed, hidden=64, mlp=128, Hq=4, Hkv=2, d=16, T=12, G=16):
    rng = np.random.default_rng(seed)
    shapes = dict(q=(Hq * d, hidden), k=(Hkv * d, hidden), v=(Hkv * d, hidden), o=(hidden, Hq * d),
                  gate=(mlp, hidden), up=(mlp, hidden), down=(hidden, mlp))
    layer = {n: quantize_nested((rng.standard_normal(s) * 0.1).astype(np.float32), G, 3, 1)
             for n, s in shapes.items()}
    layer["norm1"] = 1.0 + 0.1 * rng.standard_normal(hidden)
    layer["norm2"] = 1.0 + 0.1 * rng.standard_normal(hidden)
    Kc = rng.standard_normal((Hkv * T, d)).astype(np.float32)
    Vc = rng.standard_normal((Hkv * T, d)).astype(np.float32)
    kv = dict(k=quantize_nested(Kc, d, 2, 2), v=quantize_nested(Vc, d, 2, 2))
    x = rng.standard_normal(hidden)
    return layer, kv, x


@pytest.mark.parametrize("refined", [True, False])
def test_layer_extremes_equal_plain_layer(refined):
    """p = 1 (every channel, every token refined): full-code weights and K/V;
    p = 0 (none): resident values everywhere."""
    Hq, Hkv, T = 4, 2, 12
    layer, kv, x = _tiny_model(19)
    p = Fraction(1) if refined else Fraction(0)
    out, kv2 = od.decode_layer(x, layer, kv, T, Hq, Hkv, p, p)
    deq = dequant_full if refined else dequant_resident
    W = {n: deq(layer[n]) for n in ("q", "k", "v", "o", "gate", "up", "down")}
    W["norm1"], W["norm2"] = layer["norm1"], layer["norm2"]
    d = 16
    K = deq(kv2["k"]).reshape(Hkv, T + 1, d)
    V = deq(kv2["v"]).reshape(Hkv, T + 1, d)
    ref = _plain_layer(x, W, K, V, Hq, Hkv, T)
    np.testing.assert_allclose(out, ref, rtol=1e-9, atol=1e-9)
    # the appended token is the quantized, rotated k and the v of the new token
    n1 = _bf16(W["norm1"] * x / np.sqrt(np.dot(x, x) / x.size + 1e-5))
    k_new = _rope_complex((W["k"] @ n1).reshape(Hkv, d), T)
    v_new = (W["v"] @ n1).reshape(Hkv, d)
    np.testing.assert_array_equal(kv2["k"]["q"].reshape(Hkv, T + 1, d)[:, T],
                                  quantize_nested(k_new.astype(np.float32), d, 2, 2)["q"])
    np.testing.assert_array_equal(kv2["v"]["q"].reshape(Hkv, T + 1, d)[:, T],
                                  quantize_nested(v_new.astype(np.float32), d, 2, 2)["q"])


def test_decode_step_runs_two_layers():
    Hq, Hkv, T = 4, 2, 12
    l0, kv0, x = _tiny_model(23)
    l1, kv1, _ = _tiny_model(29)
    rng = np.random.default_rng(31)
    head = quantize_nested((rng.standard_normal((96, 64)) * 0.1).astype(np.float32), 16, 3, 1)
    logits, kvs = od.decode_step(x, [l0, l1], [kv0, kv1], T, Hq, Hkv, np.ones(64), head, Fraction(3, 100),
                                 Fraction(1, 100))
    assert logits.shape == (96,) and np.all(np.isfinite(logits))
    assert all(kv["k"]["q"].shape == (Hkv * (T + 1), 16) for kv in kvs)


# ---- the whole step (layers chained, final norm, LM head) against a plain model ----

def _plain_step(x, layers, kvs, Hq, Hkv, T, final_w, Whead, refined, d=16, eps=1e-5):
    """Textbook chain written without the oracle's decode code: each layer
    appends its own rotated k and its v (quantized per token-head, then taken
    at full code or resident value), runs the plain layer, and the final
    RMSNorm feeds a dense LM head.  Returns (logits, appended K rows, appended
    V rows) -- the rows as quantized codes [layer][Hkv][d]."""
    deq = dequant_full if refined else dequant_resident
    k_rows, v_rows = [], []
    for layer, kv in zip(layers, kvs):
        W = {n: deq(layer[n]) for n in ("q", "k", "v", "o", "gate", "up", "down")}
        W["norm1"], W["norm2"] = layer["norm1"], layer["norm2"]
        n1 = _bf16(W["norm1"] * x / np.sqrt(np.dot(x, x) / x.size + eps))
        k_new = quantize_nested(_rope_complex((W["k"] @ n1).reshape(Hkv, d), T).astype(np.float32), d, 2, 2)
        v_new = quantize_nested((W["v"] @ n1).reshape(Hkv, d).astype(np.float32), d, 2, 2)
        k_rows.append(k_new["q"])
        v_rows.append(v_new["q"])
        K = np.concatenate([deq(kv["k"]).reshape(Hkv, T, d), deq(k_new).reshape(Hkv, 1, d)], axis=1)
        V = np.concatenate([deq(kv["v"]).reshape(Hkv, T, d), deq(v_new).reshape(Hkv, 1, d)], axis=1)
        x = _plain_layer(x, W, K, V, Hq, Hkv, T)
    nf = _bf16(final_w * x / np.sqrt(np.dot(x, x) / x.size + eps))
    return deq(Whead) @ nf, k_rows, v_rows


def _two_layer_model():
    l0, kv0, x = _tiny_model(23)
    l1, kv1, _ = _tiny_model(29)
    rng = np.random.default_rng(31)
    head = quantize_nested((rng.standard_normal((96, 64)) * 0.1).astype(np.float32), 16, 3, 1)
    final_w = 1.0 + 0.2 * rng.standard_normal(64)
    return [l0, l1], [kv0, kv1], x, head, final_w


@pytest.mark.parametrize("refined", [True, False])
def test_decode_step_equals_plain_two_layer_model(refined):
    """p = 1 refines every channel and token (full-code weights and K/V
    everywhere); p = 0 refines none (resident values everywhere).  Either way
    the oracle's step must equal the plain chain: both layers in order, each
    with its own cache, then the final RMSNorm and the LM head on its output."""
    Hq, Hkv, T = 4, 2, 12
    layers, kvs, x, head, final_w = _two_layer_model()
    p = Fraction(1) if refined else Fraction(0)
    logits, kvs2 = od.decode_step(x, layers, kvs, T, Hq, Hkv, final_w, head, p, p)
    ref, k_rows, v_rows = _plain_step(x, layers, kvs, Hq, Hkv, T, final_w, head, refined)
    np.testing.assert_allclose(logits, ref, rtol=1e-9, atol=1e-9)
    for li, kv2 in enumerate(kvs2):
        np.testing.assert_array_equal(kv2["k"]["q"].reshape(Hkv, T + 1, 16)[:, T], k_rows[li])
        np.testing.assert_array_equal(kv2["v"]["q"].reshape(Hkv, T + 1, 16)[:, T], v_rows[li])
        # the old tokens are untouched
        np.testing.assert_array_equal(kv2["k"]["q"].reshape(Hkv, T + 1, 16)[:, :T],
                                      kvs[li]["k"]["q"].reshape(Hkv, T, 16))


def _step_with_mistake(x, layers, kvs, T, Hq, Hkv, final_w, head, p, mistake):
    """The oracle's step assembled from its own pieces with one planted
    mistake: the pin above must tell each of them apart from the plain model."""
    if mistake == "caches_swapped":
        kvs = kvs[::-1]
    if mistake == "layers_reversed":
        layers = layers[::-1]
    for layer, kv in zip(layers, kvs):
        x, _ = od.decode_layer(x, layer, kv, T, Hq, Hkv, p, p)
    if mistake == "no_final_norm":
        n = x
    elif mistake == "final_norm_unit_weight":
        n = od.rms_norm(x, np.ones_like(final_w))
    else:
        n = od.rms_norm(x, final_w)
    return od.refined_linear(head, n, p)


@pytest.mark.parametrize("mistake", ["caches_swapped", "layers_reversed", "no_final_norm",
                                     "final_norm_unit_weight"])
def test_decode_step_pin_catches_planted_mistakes(mistake):
    Hq, Hkv, T = 4, 2, 12
    layers, kvs, x, head, final_w = _two_layer_model()
    p = Fraction(1)
    ref, _, _ = _plain_step(x, layers, kvs, Hq, Hkv, T, final_w, head, True)
    good = _step_with_mistake(x, layers, kvs, T, Hq, Hkv, final_w, head, p, None)
    np.testing.assert_allclose(good, ref, rtol=1e-9, atol=1e-9)
    bad = _step_with_mistake(x, layers, kvs, T, Hq, Hkv, final_w, head, p, mistake)
    assert np.max(np.abs(bad - ref)) > 1e-3 * np.max(np.abs(ref))
