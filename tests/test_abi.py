"""The C-ABI library loads on a machine without a GPU, exports every entry
point that include/sf.h declares, and rejects bad arguments on the host with
a status code and a message (no device work is started by these calls)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(sf_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def sf():
    import quantized_gemv_kv_b200 as sf
    return sf


def test_header_declares_the_hot_path():
    names = _declared()
    for want in ("sf_quantize_nested", "sf_select_topk", "sf_gemv_refine", "sf_attn_decode_refine",
                 "sf_refine_cache_create", "sf_refine_cache_prefetch", "sf_refine_cache_destroy"):
        assert want in names


def test_every_declared_symbol_is_exported(sf):
    lib = ctypes.CDLL(sf.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) <= set(sf.EXPORTED)


def test_version_and_status_strings(sf):
    assert "sm_100a" in sf.version()
    assert sf._lib.sf_status_string(sf.SF_EINVAL) == b"SF_EINVAL"


def _err(sf):
    buf = ctypes.create_string_buffer(512)
    sf._lib.sf_last_error(buf, len(buf))
    return buf.value.decode()


def test_host_validation(sf):
    L = sf._lib
    p = ctypes.c_void_p(16)
    # bad bit widths, bad group size, misaligned layouts: rejected before any launch
    assert L.sf_quantize_nested(p, 64, 64, 32, 5, 2, 0, p, p, p, p, None) == sf.SF_EINVAL
    assert "b_r" in _err(sf)
    assert L.sf_quantize_nested(p, 64, 64, 48, 2, 2, 0, p, p, p, p, None) == sf.SF_EINVAL
    assert L.sf_quantize_nested(p, 48, 64, 32, 2, 2, 0, p, p, p, p, None) == sf.SF_EINVAL
    assert L.sf_quantize_nested(None, 64, 64, 32, 2, 2, 0, p, p, p, p, None) == sf.SF_EINVAL
    assert L.sf_select_topk(p, 17, 64, 4, p, p, None) == sf.SF_EINVAL
    assert L.sf_select_topk(p, 1, 64, 65, p, p, None) == sf.SF_EINVAL
    qw = sf._QWeight(16, 16, 16, None, 64, 64, 32, 2, 2)
    assert L.sf_gemv_refine(ctypes.byref(qw), p, 17, None, None, None, p, None) == sf.SF_EINVAL
    qw = sf._QWeight(16, 16, 16, None, 48, 64, 32, 2, 2)
    assert L.sf_gemv_refine(ctypes.byref(qw), p, 1, None, None, None, p, None) == sf.SF_EINVAL
    out = ctypes.c_size_t()
    assert L.sf_attn_workspace_size(32, 8, 64, 1024, 10, ctypes.byref(out)) == sf.SF_EINVAL
    assert L.sf_attn_workspace_size(32, 8, 128, 1024, 10, ctypes.byref(out)) == sf.SF_OK
    assert out.value > 32 * 1024 * 4
    h = ctypes.c_void_p()
    assert L.sf_refine_cache_create(ctypes.byref(h), 64, 24, 8, 8, p, 0) == sf.SF_EINVAL
    assert L.sf_refine_cache_destroy(None) == sf.SF_OK


def test_attn_path_switch(sf):
    """The implementation switch accepts its three values and refuses others
    (no GPU needed: nothing is enqueued)."""
    L = ctypes.CDLL(sf.LIB_PATH)
    assert L.sf_attn_set_path(7) == sf.SF_EINVAL
    assert L.sf_attn_set_path(-1) == sf.SF_EINVAL
    for p in (sf.ATTN_PIPELINE, sf.ATTN_CLUSTER, sf.ATTN_AUTO):
        assert L.sf_attn_set_path(p) == sf.SF_OK


def test_host_validation_decode_step_ops(sf):
    """The decode-step entry points and the K/V row stride reject bad sizes
    on the host, before any device work."""
    L = sf._lib
    p = ctypes.c_void_p(256)
    assert L.sf_add_rmsnorm(p, None, p, 0, 4096, ctypes.c_float(1e-5), p, None) == sf.SF_EINVAL
    assert L.sf_add_rmsnorm(p, None, p, 1, 4096, ctypes.c_float(-1.0), p, None) == sf.SF_EINVAL
    assert L.sf_add_rmsnorm(None, None, p, 1, 4096, ctypes.c_float(1e-5), p, None) == sf.SF_EINVAL
    assert L.sf_rope(p, 8, 127, 0, ctypes.c_double(500000.0), None, None) == sf.SF_EINVAL
    assert "even d" in _err(sf)
    assert L.sf_rope(p, 8, 128, -1, ctypes.c_double(500000.0), None, None) == sf.SF_EINVAL
    assert L.sf_rope(p, 8, 128, 0, ctypes.c_double(0.0), None, None) == sf.SF_EINVAL
    assert L.sf_silu_mul(p, p, 0, p, None) == sf.SF_EINVAL
    # append: t must lie inside the stride, d a multiple of 32, widths as the quantizer's
    assert L.sf_kv_append(p, 8, 128, 64, 64, 2, 2, p, p, p, p, None) == sf.SF_EINVAL
    assert L.sf_kv_append(p, 8, 100, 64, 3, 2, 2, p, p, p, p, None) == sf.SF_EINVAL
    assert L.sf_kv_append(p, 8, 128, 64, 3, 3, 2, p, p, p, p, None) == sf.SF_EINVAL
    # attention over a strided cache: a stride below T is refused
    kv = sf._QKV(256, 256, 256, 256, 256, 256, 256, 256, 2, 2, 299)
    assert L.sf_attn_decode_refine(p, 8, 2, 128, 300, ctypes.byref(kv), 3, p, p, p, p,
                                   ctypes.c_size_t(1 << 30), None) == sf.SF_EINVAL
    assert "row_stride" in _err(sf)


def test_attention_binding_refuses_bad_output_buffers_before_any_call(sf):
    """An undersized or mistyped output would be written out of bounds by the
    kernels: the binding refuses it before the library is reached (so this
    runs without a GPU)."""
    import torch
    Hq, Hkv, d, k = 32, 8, 128, 10
    q = torch.zeros((Hq, d), dtype=torch.bfloat16)
    out = torch.empty((Hq, d), dtype=torch.float32)
    sel = torch.empty((Hkv, Hq // Hkv * k), dtype=torch.int32)
    sel_n = torch.empty((Hkv,), dtype=torch.int32)
    kv = None  # never reached
    with pytest.raises(ValueError, match="sel_out"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, 64, k, out, sel[:, :-1].contiguous(), sel_n)
    with pytest.raises(ValueError, match="sel_out"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, 64, k, out, sel.to(torch.int64), sel_n)
    with pytest.raises(ValueError, match="out must be"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, 64, k, out[:-1], sel, sel_n)
    with pytest.raises(ValueError, match="sel_n"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, 64, k, out, sel, sel_n[:-1])
    with pytest.raises(ValueError, match="q must be"):
        sf.attn_decode_refine_noalloc(q.float(), kv, Hkv, 64, k, out, sel, sel_n)
    # well-formed buffers still stop at the device check on a CPU tensor
    with pytest.raises(ValueError, match="CUDA"):
        sf.attn_decode_refine_noalloc(q, kv, Hkv, 64, k, out, sel, sel_n)


def test_host_validation_gemv_produce(sf):
    """sf_gemv_refine_batch1_produce checks its producer on the host, before
    any device work: the op, its pointers, y's alignment, the selection's
    room in the launch's scratch, and an updated residual that overlaps x."""
    L = sf._lib
    qw = sf._QWeight(256, 256, 256, 256, 64, 4096, 128, 2, 2)
    job = sf._GemvJob(ctypes.pointer(qw), None, 1, 256, None)
    jp = ctypes.cast(ctypes.pointer(job), ctypes.c_void_p)

    def call(op=sf.PRODUCE_ROUND, k=10, x=4096, w=None, u=None, x_out=None, y=8192):
        pr = sf._GemvProducer(op, k, 1e-5, x, None, w, u, x_out, y, 256, 256)
        return L.sf_gemv_refine_batch1_produce(jp, 1, ctypes.cast(ctypes.pointer(pr), ctypes.c_void_p), None)

    assert L.sf_gemv_refine_batch1_produce(jp, 1, None, None) == sf.SF_EINVAL
    assert call(op=7) == sf.SF_EINVAL
    assert "unknown producer op" in _err(sf)
    assert call(op=sf.PRODUCE_NORM) == sf.SF_EINVAL
    assert "needs w" in _err(sf)
    assert call(op=sf.PRODUCE_SILU_MUL) == sf.SF_EINVAL
    assert "needs u" in _err(sf)
    assert call(y=8194) == sf.SF_EINVAL
    assert "aligned" in _err(sf)
    # 2-bit codes at K = 4096: the whole row is more than the scratch holds
    assert call(k=4096) == sf.SF_EINVAL
    assert "k must be" in _err(sf)
    assert call(k=-1) == sf.SF_EINVAL
    assert call(op=sf.PRODUCE_NORM, w=4096, x_out=4096 + 4 * 100) == sf.SF_EINVAL
    assert "x_out" in _err(sf)


def test_host_validation_rope_kv_append(sf):
    """sf_rope_kv_append_pair_cached refuses, on the host and before it
    touches the cache: a head dim that is not a multiple of 64 (a lane must
    hold both dims of its pairs), a negative position, theta <= 0, no query
    heads, and the append's own bad sizes."""
    L = sf._lib
    p = ctypes.c_void_p(256)
    good = dict(Hq=32, Hkv=8, d=128, pos=5, theta=500000.0, S=64, t=3, b_r=2, b_f=2)

    def call(**kw):
        a = dict(good, **kw)
        return L.sf_rope_kv_append_pair_cached(p, a["Hq"], None, p, p, a["Hkv"], a["d"], a["pos"],
                                               ctypes.c_double(a["theta"]), a["S"], a["t"], a["b_r"], a["b_f"],
                                               p, p, p, p, p, p, p, None, None)

    assert call(d=96) == sf.SF_EINVAL
    assert "multiple of 64" in _err(sf)
    assert call(pos=-1) == sf.SF_EINVAL
    assert call(theta=0.0) == sf.SF_EINVAL
    assert call(Hq=0) == sf.SF_EINVAL
    assert call(t=64) == sf.SF_EINVAL
    assert call(b_r=3, b_f=2) == sf.SF_EINVAL
    assert L.sf_rope_kv_append_pair_cached(None, 32, None, p, p, 8, 128, 5, ctypes.c_double(1e4), 64, 3, 2, 2,
                                           p, p, p, p, p, p, p, None, None) == sf.SF_EINVAL
