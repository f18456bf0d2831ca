"""Python binding of libsf, the StrataFlux selective-precision-streaming hot
path for B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels
of ``libsf.so``.  PyTorch provides device memory and the current CUDA stream.
The functions mirror the C ABI declared in ``include/sf.h``:

  quantize_nested, select_topk, gemv_refine, attn_decode_refine,
  attn_workspace_size, RefineCache (sf_refine_cache_*).

Importing fails loudly when the library has not been built (``build()`` in
``quantized_gemv_kv_b200.build``); there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsf.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m quantized_gemv_kv_b200.build` "
                      "(nvcc, sm_100a); there is no fallback path")

_lib = ctypes.CDLL(LIB_PATH)

SF_OK, SF_EINVAL, SF_ENOMEM, SF_ECUDA, SF_ETIMEOUT, SF_ENOTIMPL = range(6)
SF_REF_BY_COLUMN, SF_REF_BY_ROW = 0, 1
_LAYOUTS = {"by_column": SF_REF_BY_COLUMN, "by_row": SF_REF_BY_ROW}

_p = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t


class SfError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_lib.sf_status_string(status).decode()}: {msg}")
        self.status = status


class _QWeight(ctypes.Structure):
    _fields_ = [("res", _p), ("scale", _p), ("zero", _p), ("ref", _p),
                ("N", _i), ("K", _i), ("G", _i), ("b_r", _i), ("b_f", _i)]


class _QKV(ctypes.Structure):
    _fields_ = [("k_res", _p), ("k_ref", _p), ("v_res", _p), ("v_ref", _p),
                ("k_scale", _p), ("k_zero", _p), ("v_scale", _p), ("v_zero", _p),
                ("b_r", _i), ("b_f", _i), ("row_stride", _i), ("ref_cache", _p)]


class _GemvJob(ctypes.Structure):
    _fields_ = [("W", ctypes.POINTER(_QWeight)), ("cache", _p), ("use_ref_store", _i), ("y", _p), ("res_b1", _p)]


class _GemvProducer(ctypes.Structure):
    _fields_ = [("op", _i), ("k", _i), ("eps", ctypes.c_float), ("x", _p), ("delta", _p), ("w", _p), ("u", _p),
                ("x_out", _p), ("y", _p), ("idx", _p), ("n", _p)]


PRODUCE_NORM, PRODUCE_ROUND, PRODUCE_SILU_MUL = 0, 1, 2


class _SelectJob(ctypes.Structure):
    _fields_ = [("x", _p), ("K", _i), ("k", _i), ("idx_out", _p), ("n_out", _p), ("act", _p)]


class CacheStats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int64), ("hits", ctypes.c_int64), ("misses", ctypes.c_int64),
                ("bypass", ctypes.c_int64), ("h2d_bytes", ctypes.c_int64), ("late", ctypes.c_int64)]


_SIGS = {
    "sf_version": ([], ctypes.c_char_p),
    "sf_status_string": ([_i], ctypes.c_char_p),
    "sf_last_error": ([ctypes.c_char_p, _sz], _sz),
    "sf_quantize_nested": ([_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p], _i),
    "sf_select_topk": ([_p, _i, _i, _i, _p, _p, _p], _i),
    "sf_refine_cache_create": ([ctypes.POINTER(_p), _i, _sz, _i, _i, _p, _i], _i),
    "sf_refine_cache_create_parts": ([ctypes.POINTER(_p), _i, _sz, _i, _i, _i, _p, _i], _i),
    "sf_refine_cache_preload": ([_p, _p, _i, _p], _i),
    "sf_refine_cache_prefetch": ([_p, _p, _p, _p, _p], _i),
    "sf_refine_cache_sets": ([_p, _p, _p, _p, _p], _i),
    "sf_refine_cache_slots": ([_p, _p], _i),
    "sf_refine_cache_stats": ([_p, ctypes.POINTER(CacheStats)], _i),
    "sf_refine_cache_reset": ([_p], _i),
    "sf_refine_cache_destroy": ([_p], _i),
    "sf_refine_cache_set_budget": ([_p, _i], _i),
    "sf_refine_cache_set_deadline": ([_p, _i], _i),
    "sf_refine_group_create": ([ctypes.POINTER(_p), ctypes.POINTER(_p), ctypes.POINTER(_p), ctypes.POINTER(_p), _i],
                               _i),
    "sf_refine_group_prefetch": ([_p, _p, _p], _i),
    "sf_refine_group_destroy": ([_p], _i),
    "sf_gemv_refine": ([ctypes.POINTER(_QWeight), _p, _i, _p, _p, _p, _p, _p], _i),
    "sf_act_bytes": ([_i], _sz),
    "sf_select_random": ([_i, _i, ctypes.c_uint64, ctypes.c_uint64, _p, _p, _p], _i),
    "sf_quantize_residual": ([_p, ctypes.POINTER(_QWeight), _p, _p], _i),
    "sf_gemv_fp16_fetch": ([ctypes.POINTER(_QWeight), _p, _i, _p, _p, _p, _p, _p, _p], _i),
    "sf_select_topk_act": ([_p, _i, _i, _p, _p, _p, _p], _i),
    "sf_act_prepare": ([_p, _i, _p, _p], _i),
    "sf_select_topk_act_many": ([_p, _i, _p], _i),
    "sf_gemv_refine_batch1": ([_p, _i, _p, _p, _p, _p], _i),
    "sf_gemv_refine_batch1_produce": ([_p, _i, _p, _p], _i),
    "sf_gemv_pack_batch1": ([_p, _i, _i, _i, _p, _p], _i),
    "sf_attn_workspace_size": ([_i, _i, _i, _i, _i, ctypes.POINTER(_sz)], _i),
    "sf_attn_decode_refine": ([_p, _i, _i, _i, _i, ctypes.POINTER(_QKV), _i, _p, _p, _p, _p, _sz, _p], _i),
    "sf_attn_decode_refine_noalloc": ([_p, _i, _i, _i, _i, ctypes.POINTER(_QKV), _i, _p, _p, _p, _p], _i),
    "sf_attn_set_path": ([_i], _i),
    "sf_attn_union_units": ([_p, _p, _i, _i, _i, _p, _p, _p], _i),
    "sf_add_rmsnorm": ([_p, _p, _p, _i, _i, ctypes.c_float, _p, _p], _i),
    "sf_rope": ([_p, _i, _i, _i, ctypes.c_double, _p, _p], _i),
    "sf_silu_mul": ([_p, _p, _i, _p, _p], _i),
    "sf_round_bf16": ([_p, _i, _p, _p], _i),
    "sf_norm_select": ([_p, _p, _p, _i, ctypes.c_float, _p, _i, _p, _p, _p, _p], _i),
    "sf_round_select": ([_p, _i, _p, _i, _p, _p, _p, _p], _i),
    "sf_silu_mul_select": ([_p, _p, _i, _p, _i, _p, _p, _p, _p], _i),
    "sf_rope_qk": ([_p, _i, _p, _i, _i, _i, ctypes.c_double, _p, _p], _i),
    "sf_kv_append": ([_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p], _i),
    "sf_kv_append_cached": ([_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _i, _p], _i),
    "sf_gemv_set_launch_overlap": ([_i], _i),
    "sf_kv_append_pair_cached": ([_p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i),
    "sf_rope_kv_append_pair_cached": ([_p, _i, _p, _p, _p, _i, _i, _i, ctypes.c_double, _i, _i, _i, _i, _p, _p, _p,
                                       _p, _p, _p, _p, _p, _p], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


def version() -> str:
    return _lib.sf_version().decode()


def _check(status: int) -> None:
    if status != SF_OK:
        buf = ctypes.create_string_buffer(1024)
        _lib.sf_last_error(buf, len(buf))
        raise SfError(status, buf.value.decode(errors="replace"))


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libsf must be contiguous")
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


# ---- quantization ------------------------------------------------------------

@dataclass
class QWeight:
    """Packed nested-quantized matrix (see ``sf_quantize_nested``)."""
    res: torch.Tensor      # int32 [N][K*b_r/32] (uint32 words)
    ref: torch.Tensor      # int32 [K][N*b_f/32] (by_column) or [N][K*b_f/32] (by_row)
    scale: torch.Tensor    # float16 [K/G][N]
    zero: torch.Tensor     # float16 [K/G][N]
    N: int
    K: int
    G: int
    b_r: int
    b_f: int
    layout: str = "by_column"
    res_b1: torch.Tensor | None = None  # resident codes in the batch-1 layout (pack_batch1)

    def c_struct(self, with_ref: bool = False) -> _QWeight:
        return _QWeight(_ptr(self.res), _ptr(self.scale), _ptr(self.zero),
                        _ptr(self.ref) if with_ref else None, self.N, self.K, self.G, self.b_r, self.b_f)


def quantize_nested(W: torch.Tensor, G: int, b_r: int, b_f: int, layout: str = "by_column",
                    stream: torch.cuda.Stream | None = None) -> QWeight:
    """Nested min-max group quantization of fp32 W[N][K] on the device."""
    _dev(W, "W")
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    dev = W.device
    res = torch.empty((N, K * b_r // 32), dtype=torch.int32, device=dev)
    if layout == "by_column":
        ref = torch.empty((K, N * b_f // 32), dtype=torch.int32, device=dev)
    else:
        ref = torch.empty((N, K * b_f // 32), dtype=torch.int32, device=dev)
    scale = torch.empty((K // G, N), dtype=torch.float16, device=dev)
    zero = torch.empty((K // G, N), dtype=torch.float16, device=dev)
    _check(_lib.sf_quantize_nested(_ptr(W), N, K, G, b_r, b_f, _LAYOUTS[layout], _ptr(res), _ptr(ref),
                                   _ptr(scale), _ptr(zero), _stream(stream)))
    return QWeight(res, ref, scale, zero, N, K, G, b_r, b_f, layout)


# ---- selection ---------------------------------------------------------------

def select_topk(x: torch.Tensor, k: int, idx_out: torch.Tensor | None = None, n_out: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k channels by |x| per row of bf16 x[B][K], union ascending.
    Returns (idx int32 [B*k] buffer, n int32 [1] device scalar)."""
    _dev(x, "x")
    if x.dim() == 1:
        x = x.unsqueeze(0)
    B, K = x.shape
    if idx_out is None:
        idx_out = torch.empty(max(B * k, 1), dtype=torch.int32, device=x.device)
    if n_out is None:
        n_out = torch.empty(1, dtype=torch.int32, device=x.device)
    _check(_lib.sf_select_topk(_ptr(x), B, K, k, _ptr(idx_out), _ptr(n_out), _stream(stream)))
    return idx_out, n_out


# ---- refinement cache ----------------------------------------------------------

class RefineCache:
    """LRU refinement cache in device memory fed from a host master copy
    (``sf_refine_cache_*``).  ``host_master`` is a CPU uint8/int32 tensor of
    num_units * unit_bytes bytes; it is kept alive by this object.  With
    parts > 1 the units are split into that many consecutive ranges, each an
    LRU of ``capacity`` slots seeing at most ``max_select`` units per step
    (``sf_refine_cache_create_parts``)."""

    def __init__(self, num_units: int, unit_bytes: int, capacity: int, max_select: int,
                 host_master: torch.Tensor, device: int | None = None, parts: int = 1):
        if host_master.is_cuda or not host_master.is_contiguous():
            raise ValueError("host_master must be a contiguous CPU tensor")
        if host_master.numel() * host_master.element_size() < num_units * unit_bytes:
            raise ValueError("host_master is smaller than num_units * unit_bytes")
        self._master = host_master
        self.num_units, self.unit_bytes, self.capacity, self.max_select = num_units, unit_bytes, capacity, max_select
        self.parts = parts
        self.device = torch.cuda.current_device() if device is None else device
        h = _p()
        _check(_lib.sf_refine_cache_create_parts(ctypes.byref(h), num_units, unit_bytes, parts, capacity, max_select,
                                                 host_master.data_ptr(), self.device))
        self._h = h

    @property
    def handle(self) -> int:
        return self._h.value

    def preload(self, units: torch.Tensor, stream: torch.cuda.Stream | None = None) -> None:
        _dev(units, "units")
        _check(_lib.sf_refine_cache_preload(self._h, _ptr(units), units.numel(), _stream(stream)))

    def prefetch(self, idx: torch.Tensor, n: torch.Tensor, producer: torch.cuda.Stream | None = None,
                 side: torch.cuda.Stream | None = None) -> None:
        _check(_lib.sf_refine_cache_prefetch(self._h, _ptr(idx), _ptr(n), _stream(producer),
                                             _stream(side if side is not None else producer)))

    def sets(self) -> dict:
        import numpy as np
        h = np.zeros(self.max_select * self.parts, np.int32)
        m = np.zeros(self.max_select * self.parts, np.int32)
        b = np.zeros(self.max_select * self.parts, np.int32)
        c = np.zeros(3, np.int32)
        _check(_lib.sf_refine_cache_sets(self._h, h.ctypes.data, m.ctypes.data, b.ctypes.data, c.ctypes.data))
        return dict(hits=h[:c[0]].tolist(), misses=m[:c[1]].tolist(), bypass=b[:c[2]].tolist())

    def slots(self) -> list[int]:
        import numpy as np
        s = np.zeros(max(self.capacity * self.parts, 1), np.int32)
        _check(_lib.sf_refine_cache_slots(self._h, s.ctypes.data))
        return s[:self.capacity * self.parts].tolist()

    def stats(self) -> CacheStats:
        st = CacheStats()
        _check(_lib.sf_refine_cache_stats(self._h, ctypes.byref(st)))
        return st

    def reset(self) -> None:
        _check(_lib.sf_refine_cache_reset(self._h))

    def set_deadline(self, on: bool = True) -> None:
        """Deadline reading for a weight matrix's cache
        (``sf_refine_cache_set_deadline``): the batch-1 GEMV refines only the
        selected columns already cached and does not wait for fetches."""
        _check(_lib.sf_refine_cache_set_deadline(self._h, 1 if on else 0))

    def set_budget(self, budget: int | None) -> None:
        """Per-step fetch budget (``sf_refine_cache_set_budget``); None = no limit."""
        _check(_lib.sf_refine_cache_set_budget(self._h, -1 if budget is None else int(budget)))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            _check(_lib.sf_refine_cache_destroy(self._h))
            self._h = _p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class RefineGroup:
    """Batched prefetch of several caches (``sf_refine_group_*``).  ``entries``
    is a list of (RefineCache, idx tensor, n tensor); the tensors must keep
    their storage for the group's lifetime (their device pointers are fixed at
    creation)."""

    def __init__(self, entries):
        cnt = len(entries)
        self._entries = list(entries)
        caches = (_p * cnt)(*[c.handle for c, _, _ in entries])
        idxs = (_p * cnt)(*[_ptr(i) for _, i, _ in entries])
        ns = (_p * cnt)(*[_ptr(n) for _, _, n in entries])
        h = _p()
        _check(_lib.sf_refine_group_create(ctypes.byref(h), caches, idxs, ns, cnt))
        self._h = h

    def prefetch(self, producer: torch.cuda.Stream | None = None, side: torch.cuda.Stream | None = None) -> None:
        _check(_lib.sf_refine_group_prefetch(self._h, _stream(producer),
                                             _stream(side if side is not None else producer)))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            _check(_lib.sf_refine_group_destroy(self._h))
            self._h = _p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- GEMV ----------------------------------------------------------------------

def gemv_refine(W: QWeight, x: torch.Tensor, idx: torch.Tensor | None = None, n: torch.Tensor | None = None,
                cache: RefineCache | None = None, use_ref_store: bool = False, y: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Refined decode GEMV y[B][N] (fp32).  Refinements come from ``cache``,
    else from W.ref when ``use_ref_store``, else none (resident-only)."""
    _dev(x, "x")
    if x.dim() == 1:
        x = x.unsqueeze(0)
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, W.N), dtype=torch.float32, device=x.device)
    qw = W.c_struct(with_ref=use_ref_store and cache is None)
    _check(_lib.sf_gemv_refine(ctypes.byref(qw), _ptr(x), B, _ptr(idx), _ptr(n),
                               cache.handle if cache is not None else None, _ptr(y), _stream(stream)))
    return y


# ---- attention -----------------------------------------------------------------

@dataclass
class QKV:
    """Quantized K and V, rows = token-heads [Hkv][S] (layout by_row, G = d):
    S = row_stride when it is positive (a cache allocated for row_stride
    tokens per head), else the call's T.  ``ref_cache``: the refinement bits
    live in this RefineCache (units g*S + t of 64 bytes: K words then V
    words) instead of k.ref / v.ref, which may then be None."""
    k: QWeight
    v: QWeight
    row_stride: int = 0
    ref_cache: "RefineCache | None" = None

    def c_struct(self) -> _QKV:
        return _QKV(_ptr(self.k.res), _ptr(self.k.ref), _ptr(self.v.res), _ptr(self.v.ref),
                    _ptr(self.k.scale), _ptr(self.k.zero), _ptr(self.v.scale), _ptr(self.v.zero),
                    self.k.b_r, self.k.b_f, self.row_stride,
                    self.ref_cache.handle if self.ref_cache is not None else None)


ATTN_AUTO, ATTN_CLUSTER, ATTN_PIPELINE = 0, 1, 2


def attn_set_path(path: int) -> None:
    """Process-wide choice of the attention implementation
    (``sf_attn_set_path``): ATTN_AUTO, ATTN_CLUSTER (one thread-block cluster
    per KV head, T <= 32768) or ATTN_PIPELINE (the multi-kernel pipeline)."""
    _check(_lib.sf_attn_set_path(path))


def attn_workspace_size(Hq: int, Hkv: int, d: int, T: int, k_tokens: int) -> int:
    out = _sz()
    _check(_lib.sf_attn_workspace_size(Hq, Hkv, d, T, k_tokens, ctypes.byref(out)))
    return out.value


def attn_decode_refine(q: torch.Tensor, kv: QKV, Hkv: int, T: int, k_tokens: int,
                       workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       sel_out: torch.Tensor | None = None, sel_n: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None):
    """Refined decode attention.  Returns (out fp32 [Hq][d], sel int32
    [Hkv][Hq/Hkv*k], sel_n int32 [Hkv])."""
    _dev(q, "q")
    Hq, d = q.shape
    grp = Hq // Hkv
    dev = q.device
    if workspace is None:
        workspace = torch.empty(attn_workspace_size(Hq, Hkv, d, T, k_tokens), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((Hq, d), dtype=torch.float32, device=dev)
    if sel_out is None:
        sel_out = torch.empty((Hkv, max(grp * k_tokens, 1)), dtype=torch.int32, device=dev)
    if sel_n is None:
        sel_n = torch.empty(Hkv, dtype=torch.int32, device=dev)
    _check_attn_outputs(q, Hkv, k_tokens, out, sel_out, sel_n)
    s = kv.c_struct()
    _check(_lib.sf_attn_decode_refine(_ptr(q), Hq, Hkv, d, T, ctypes.byref(s), k_tokens, _ptr(sel_out),
                                      _ptr(sel_n), _ptr(out), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, sel_out, sel_n


def _check_attn_outputs(q: torch.Tensor, Hkv: int, k_tokens: int, out: torch.Tensor, sel_out: torch.Tensor,
                        sel_n: torch.Tensor) -> None:
    """Shapes, dtypes and devices of the attention's caller-provided buffers,
    checked before anything reaches the library (an undersized output would
    be written out of bounds by the kernels)."""
    if q.dtype != torch.bfloat16 or q.dim() != 2:
        raise ValueError("q must be a 2-D bfloat16 tensor [Hq][d]")
    Hq, d = q.shape
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if out.dtype != torch.float32 or out.numel() < Hq * d:
        raise ValueError(f"out must be float32 with at least Hq*d = {Hq * d} elements")
    need = Hkv * (Hq // Hkv) * k_tokens
    if sel_out.dtype != torch.int32 or sel_out.numel() < need:
        raise ValueError(f"sel_out must be int32 with at least Hkv*(Hq/Hkv)*k_tokens = {need} elements")
    if sel_n.dtype != torch.int32 or sel_n.numel() < Hkv:
        raise ValueError(f"sel_n must be int32 with at least Hkv = {Hkv} elements")
    for name, t in (("q", q), ("out", out), ("sel_out", sel_out), ("sel_n", sel_n)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        _dev(t, name)
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")


def attn_union_units(sel_out: torch.Tensor, sel_n: torch.Tensor, Hkv: int, cap: int, S: int, units: torch.Tensor,
                     n_units: torch.Tensor, stream: torch.cuda.Stream | None = None) -> None:
    """``sf_attn_union_units``: the KV-refinement-cache units (g*S + t) of
    the union an attention call selected, ascending, into units / n_units.
    cap = (Hq/Hkv) * k_tokens of that call (the row stride of sel_out)."""
    if sel_out.numel() < Hkv * cap or units.dtype != torch.int32 or units.numel() < Hkv * cap or \
            n_units.dtype != torch.int32:
        raise ValueError("units must be int32 with room for Hkv * cap entries, n_units int32")
    _check(_lib.sf_attn_union_units(_ptr(sel_out), _ptr(sel_n), Hkv, cap, S, _ptr(units), _ptr(n_units),
                                    _stream(stream)))


def attn_decode_refine_noalloc(q: torch.Tensor, kv: QKV, Hkv: int, T: int, k_tokens: int,
                               out: torch.Tensor, sel_out: torch.Tensor, sel_n: torch.Tensor,
                               stream: torch.cuda.Stream | None = None) -> None:
    """Refined decode attention with the library's built-in scratch
    (``sf_attn_decode_refine_noalloc``): for callers that must not allocate
    device memory at this point.  The caller provides the outputs; nothing
    is allocated by this call."""
    _check_attn_outputs(q, Hkv, k_tokens, out, sel_out, sel_n)
    Hq, d = q.shape
    s = kv.c_struct()
    _check(_lib.sf_attn_decode_refine_noalloc(_ptr(q), Hq, Hkv, d, T, ctypes.byref(s), k_tokens, _ptr(sel_out),
                                              _ptr(sel_n), _ptr(out), _stream(stream)))


# ---- batch-1 fast path ---------------------------------------------------------

def pack_batch1(W: QWeight, drop_canonical: bool = False, stream: torch.cuda.Stream | None = None) -> QWeight:
    """Writes W.res_b1, the resident codes in the layout of the batch-1
    tensor-core GEMV (``sf_gemv_pack_batch1``); for 2-bit codes that is the
    canonical layout itself.  ``drop_canonical`` releases W.res afterwards
    (the batch-1 GEMV then reads only W.res_b1)."""
    _dev(W.res, "W.res")
    if W.b_r == 2:
        W.res_b1 = W.res
    else:
        out = torch.empty_like(W.res)
        _check(_lib.sf_gemv_pack_batch1(_ptr(W.res), W.N, W.K, W.b_r, _ptr(out), _stream(stream)))
        W.res_b1 = out
        if drop_canonical:
            W.res = None
    return W


def act_bytes(K: int) -> int:
    return _lib.sf_act_bytes(K)


def select_topk_act(x: torch.Tensor, k: int, idx_out: torch.Tensor, n_out: torch.Tensor, act: torch.Tensor,
                    stream: torch.cuda.Stream | None = None) -> None:
    """Top-k selection of one activation row plus its prepared form
    (``sf_select_topk_act``)."""
    _dev(x, "x")
    K = x.shape[-1]
    _check(_lib.sf_select_topk_act(_ptr(x), K, k, _ptr(idx_out), _ptr(n_out), _ptr(act), _stream(stream)))


def act_prepare(x: torch.Tensor, act: torch.Tensor, stream: torch.cuda.Stream | None = None) -> None:
    """Prepared form of one activation row with nothing selected."""
    _dev(x, "x")
    _check(_lib.sf_act_prepare(_ptr(x), x.shape[-1], _ptr(act), _stream(stream)))


class Batch1Jobs:
    """A reusable list of (QWeight, cache or None, use_ref_store, y) for
    ``sf_gemv_refine_batch1``; builds the C structs once."""

    def __init__(self, jobs):
        self._w = [W.c_struct(with_ref=bool(store)) for W, cache, store, y in jobs]
        self._keep = jobs
        arr = (_GemvJob * len(jobs))()
        for i, (W, cache, store, y) in enumerate(jobs):
            arr[i].W = ctypes.pointer(self._w[i])
            arr[i].cache = cache.handle if cache is not None else None
            arr[i].use_ref_store = 1 if store else 0
            arr[i].y = _ptr(y)
            arr[i].res_b1 = _ptr(W.res_b1) if W.res_b1 is not None else None
        self._arr = arr
        self.count = len(jobs)

    def run(self, x: torch.Tensor, idx: torch.Tensor | None = None, n: torch.Tensor | None = None,
            stream: torch.cuda.Stream | None = None) -> None:
        """x: the bf16 row; (idx, n): its selection (None: nothing selected)."""
        _check(_lib.sf_gemv_refine_batch1(ctypes.cast(self._arr, _p), self.count, _ptr(x), _ptr(idx), _ptr(n),
                                          _stream(stream)))

    def run_produce(self, op: int, x: torch.Tensor, y: torch.Tensor, k: int, idx: torch.Tensor, n: torch.Tensor,
                    delta: torch.Tensor | None = None, w: torch.Tensor | None = None, u: torch.Tensor | None = None,
                    x_out: torch.Tensor | None = None, eps: float = 1e-5,
                    stream: torch.cuda.Stream | None = None) -> None:
        """``sf_gemv_refine_batch1_produce``: the input row made inside the
        launch by ``op`` (PRODUCE_NORM: bf16(RMSNorm(x + delta) w), x + delta
        to x_out; PRODUCE_ROUND: bf16(x); PRODUCE_SILU_MUL: bf16(silu(x) u)),
        written to y with its top-k selection (idx, n), then the GEMVs."""
        _dev(x, "x")
        if idx.dtype != torch.int32 or idx.numel() < max(k, 1) or n.dtype != torch.int32:
            raise ValueError("idx and n must be int32, idx with room for k entries")
        pr = _GemvProducer(op, k, eps, _ptr(x), _ptr(delta), _ptr(w), _ptr(u), _ptr(x_out), _ptr(y), _ptr(idx),
                           _ptr(n))
        pp = ctypes.cast(ctypes.pointer(pr), _p)
        _check(_lib.sf_gemv_refine_batch1_produce(ctypes.cast(self._arr, _p), self.count, pp, _stream(stream)))


_gemv_overlap = False


def gemv_set_launch_overlap(on: bool) -> bool:
    """``sf_gemv_set_launch_overlap``: batch-1 GEMV launches may overlap the
    previous kernel (which must not write the weights).  Returns the
    previous setting."""
    global _gemv_overlap
    prev = _gemv_overlap
    _check(_lib.sf_gemv_set_launch_overlap(1 if on else 0))
    _gemv_overlap = bool(on)
    return prev


def gemv_refine_batch1(jobs, x: torch.Tensor, idx: torch.Tensor | None = None, n: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None) -> None:
    """Refined GEMVs at batch 1 of up to 4 matrices that read the same x."""
    Batch1Jobs(jobs).run(x, idx, n, stream)


class SelectJobs:
    """A reusable list of single-row selections for
    ``sf_select_topk_act_many``: entries (x, k, idx_out, n_out, act or None)."""

    def __init__(self, jobs):
        self._keep = jobs
        arr = (_SelectJob * len(jobs))()
        for i, (x, k, idx, n, act) in enumerate(jobs):
            arr[i].x = _ptr(x)
            arr[i].K = x.shape[-1]
            arr[i].k = k
            arr[i].idx_out = _ptr(idx)
            arr[i].n_out = _ptr(n)
            arr[i].act = _ptr(act) if act is not None else None
        self._arr = arr
        self.count = len(jobs)

    def run(self, stream: torch.cuda.Stream | None = None) -> None:
        _check(_lib.sf_select_topk_act_many(ctypes.cast(self._arr, _p), self.count, _stream(stream)))


# ---- decode-step elementwise operations ----------------------------------------

def add_rmsnorm(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-5, delta: torch.Tensor | None = None,
                y: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """``sf_add_rmsnorm``: x (fp32 [B][H], updated in place by x += delta
    when delta is given), w fp32 [H]; returns y bf16 [B][H]."""
    _dev(x, "x")
    if x.dtype != torch.float32 or w.dtype != torch.float32 or (delta is not None and delta.dtype != torch.float32):
        raise ValueError("x, w and delta must be float32")
    x2 = x if x.dim() == 2 else x.view(1, -1)
    B, H = x2.shape
    if y is None:
        y = torch.empty((B, H), dtype=torch.bfloat16, device=x.device)
    _check(_lib.sf_add_rmsnorm(_ptr(x2), _ptr(delta), _ptr(w), B, H, eps, _ptr(y), _stream(stream)))
    return y


def rope(x: torch.Tensor, pos: int, theta: float = 500000.0, y: torch.Tensor | None = None,
         stream: torch.cuda.Stream | None = None) -> torch.Tensor | None:
    """``sf_rope``: rotates the heads of x (fp32 [H][d], in place) to
    position pos; when y (bf16 [H][d]) is given the result is also written
    there as bf16.  Returns y."""
    _dev(x, "x")
    if x.dtype != torch.float32 or x.dim() != 2:
        raise ValueError("x must be a 2-D float32 tensor")
    H, d = x.shape
    _check(_lib.sf_rope(_ptr(x), H, d, pos, theta, _ptr(y), _stream(stream)))
    return y


def silu_mul(g: torch.Tensor, u: torch.Tensor, y: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """``sf_silu_mul``: bf16(silu(g) * u) elementwise over fp32 g, u."""
    _dev(g, "g")
    if g.dtype != torch.float32 or u.dtype != torch.float32 or g.numel() != u.numel():
        raise ValueError("g and u must be float32 tensors of the same size")
    if y is None:
        y = torch.empty(g.shape, dtype=torch.bfloat16, device=g.device)
    _check(_lib.sf_silu_mul(_ptr(g), _ptr(u), g.numel(), _ptr(y), _stream(stream)))
    return y


def round_bf16(x: torch.Tensor, y: torch.Tensor | None = None,
               stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """``sf_round_bf16``: bf16 (ties to even) of fp32 x, elementwise."""
    _dev(x, "x")
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    if y is None:
        y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    if y.dtype != torch.bfloat16 or y.numel() < x.numel():
        raise ValueError("y must be bfloat16 with at least x.numel() elements")
    _check(_lib.sf_round_bf16(_ptr(x), x.numel(), _ptr(y), _stream(stream)))
    return y


def kv_append(src: torch.Tensor, res: torch.Tensor, ref: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
              row_stride: int, t: int, b_r: int = 2, b_f: int = 2, stream: torch.cuda.Stream | None = None) -> None:
    """``sf_kv_append``: quantizes src (fp32 [Hkv][d]) and writes it as token
    t of every KV head of the cache (res, ref, scale, zero with rows
    [Hkv][row_stride])."""
    _dev(src, "src")
    if src.dtype != torch.float32 or src.dim() != 2:
        raise ValueError("src must be a 2-D float32 tensor")
    Hkv, d = src.shape
    _check(_lib.sf_kv_append(_ptr(src), Hkv, d, row_stride, t, b_r, b_f, _ptr(res), _ptr(ref), _ptr(scale),
                             _ptr(zero), _stream(stream)))



def kv_append_cached(src: torch.Tensor, res: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                     cache: RefineCache, part: int, row_stride: int, t: int, b_r: int = 2, b_f: int = 2,
                     stream: torch.cuda.Stream | None = None) -> None:
    """``sf_kv_append_cached``: as kv_append, with the refinement bits written
    to the KV refinement cache's host master (part 0: K half, 1: V half)."""
    _dev(src, "src")
    if src.dtype != torch.float32 or src.dim() != 2:
        raise ValueError("src must be a 2-D float32 tensor")
    Hkv, d = src.shape
    _check(_lib.sf_kv_append_cached(_ptr(src), Hkv, d, row_stride, t, b_r, b_f, _ptr(res), _ptr(scale), _ptr(zero),
                                    cache.handle, part, _stream(stream)))


def kv_append_pair_cached(k_src: torch.Tensor, v_src: torch.Tensor, kq: "QWeight", vq: "QWeight", cache: RefineCache,
                          row_stride: int, t: int, b_r: int = 2, b_f: int = 2, stream: torch.cuda.Stream | None = None,
                          side: torch.cuda.Stream | None = None) -> None:
    """``sf_kv_append_pair_cached``: the key and value rows of token t in one
    launch; the host master's copy runs on ``side`` (default: ``stream``)."""
    _dev(k_src, "k_src")
    _dev(v_src, "v_src")
    if k_src.dtype != torch.float32 or k_src.dim() != 2 or v_src.shape != k_src.shape or v_src.dtype != torch.float32:
        raise ValueError("k_src and v_src must be 2-D float32 tensors of one shape")
    Hkv, d = k_src.shape
    st = _stream(stream)
    _check(_lib.sf_kv_append_pair_cached(_ptr(k_src), _ptr(v_src), Hkv, d, row_stride, t, b_r, b_f, _ptr(kq.res),
                                         _ptr(kq.scale), _ptr(kq.zero), _ptr(vq.res), _ptr(vq.scale), _ptr(vq.zero),
                                         cache.handle, st, _stream(side) if side is not None else st))


def rope_kv_append_pair_cached(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kq: "QWeight", vq: "QWeight",
                               cache: RefineCache, row_stride: int, t: int, pos: int, b_r: int = 2, b_f: int = 2,
                               theta: float = 500000.0, q_bf16: torch.Tensor | None = None,
                               stream: torch.cuda.Stream | None = None, side: torch.cuda.Stream | None = None) -> None:
    """``sf_rope_kv_append_pair_cached``: RoPE of q [Hq][d] (in place, and as
    bf16 to q_bf16) and k [Hkv][d] to position pos, then the rotated key and
    the value rows of token t appended, in one launch."""
    for name, a in (("q", q), ("k", k), ("v", v)):
        _dev(a, name)
        if a.dtype != torch.float32 or a.dim() != 2:
            raise ValueError(f"{name} must be a 2-D float32 tensor")
    if v.shape != k.shape or q.shape[1] != k.shape[1]:
        raise ValueError("k and v must have one shape, and q the same head dim")
    if q_bf16 is not None and (q_bf16.dtype != torch.bfloat16 or q_bf16.numel() != q.numel()):
        raise ValueError("q_bf16 must be bfloat16 with q's size")
    Hq, d = q.shape
    Hkv = k.shape[0]
    st = _stream(stream)
    _check(_lib.sf_rope_kv_append_pair_cached(_ptr(q), Hq, _ptr(q_bf16), _ptr(k), _ptr(v), Hkv, d, pos, theta,
                                              row_stride, t, b_r, b_f, _ptr(kq.res), _ptr(kq.scale), _ptr(kq.zero),
                                              _ptr(vq.res), _ptr(vq.scale), _ptr(vq.zero), cache.handle, st,
                                              _stream(side) if side is not None else st))


def norm_select(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, k: int, idx: torch.Tensor, n: torch.Tensor,
                act: torch.Tensor | None, eps: float = 1e-5, delta: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> None:
    """``sf_norm_select``: x += delta, y = bf16(RMSNorm(x) w), then the top-k
    selection of y and its prepared activations, in one launch (batch 1)."""
    _dev(x, "x")
    _check(_lib.sf_norm_select(_ptr(x), _ptr(delta), _ptr(w), x.numel(), eps, _ptr(y), k, _ptr(idx), _ptr(n),
                               _ptr(act), _stream(stream)))


def round_select(a: torch.Tensor, y: torch.Tensor, k: int, idx: torch.Tensor, n: torch.Tensor,
                 act: torch.Tensor | None, stream: torch.cuda.Stream | None = None) -> None:
    """``sf_round_select``: y = bf16(a), then its top-k selection and prepared activations."""
    _dev(a, "a")
    _check(_lib.sf_round_select(_ptr(a), a.numel(), _ptr(y), k, _ptr(idx), _ptr(n), _ptr(act), _stream(stream)))


def silu_mul_select(g: torch.Tensor, u: torch.Tensor, y: torch.Tensor, k: int, idx: torch.Tensor, n: torch.Tensor,
                    act: torch.Tensor | None, stream: torch.cuda.Stream | None = None) -> None:
    """``sf_silu_mul_select``: y = bf16(silu(g) u), then its top-k selection and prepared activations."""
    _dev(g, "g")
    if g.numel() != u.numel():
        raise ValueError("g and u must have the same size")
    _check(_lib.sf_silu_mul_select(_ptr(g), _ptr(u), g.numel(), _ptr(y), k, _ptr(idx), _ptr(n), _ptr(act),
                                   _stream(stream)))


def rope_qk(q: torch.Tensor, k: torch.Tensor, pos: int, theta: float = 500000.0, q_bf16: torch.Tensor | None = None,
            stream: torch.cuda.Stream | None = None) -> None:
    """``sf_rope_qk``: RoPE of q [Hq][d] (and its bf16 copy) and k [Hkv][d] in one launch."""
    _dev(q, "q")
    Hq, d = q.shape
    _check(_lib.sf_rope_qk(_ptr(q), Hq, _ptr(k), k.shape[0], d, pos, theta, _ptr(q_bf16), _stream(stream)))


# ---- comparator modes ------------------------------------------------------------

def select_random(K: int, k: int, seed: int, step: int, idx: torch.Tensor, n: torch.Tensor,
                  stream: torch.cuda.Stream | None = None) -> None:
    """``sf_select_random``: k of K channels from a counter-based draw."""
    _dev(idx, "idx")
    if idx.dtype != torch.int32 or idx.numel() < max(k, 1):
        raise ValueError("idx must be int32 with room for k entries")
    _check(_lib.sf_select_random(K, k, seed, step, _ptr(idx), _ptr(n), _stream(stream)))


def quantize_residual(W: torch.Tensor, qw: QWeight, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """``sf_quantize_residual``: fp16 [K][N] residuals of W against its resident values."""
    _dev(W, "W")
    out = torch.empty((qw.K, qw.N), dtype=torch.float16, device=W.device)
    s = qw.c_struct()
    _check(_lib.sf_quantize_residual(_ptr(W), ctypes.byref(s), _ptr(out), _stream(stream)))
    return out


def gemv_fp16_fetch(W: QWeight, x: torch.Tensor, idx: torch.Tensor, n: torch.Tensor, resid: torch.Tensor | None = None,
                    cache: RefineCache | None = None, y: torch.Tensor | None = None,
                    stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """``sf_gemv_fp16_fetch``: the FP16-fetch comparator GEMV (residual store or a cache of its columns)."""
    _dev(x, "x")
    if x.dim() == 1:
        x = x.unsqueeze(0)
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, W.N), dtype=torch.float32, device=x.device)
    s = W.c_struct()
    _check(_lib.sf_gemv_fp16_fetch(ctypes.byref(s), _ptr(x), B, _ptr(idx), _ptr(n), _ptr(resid),
                                   cache.handle if cache is not None else None, _ptr(y), _stream(stream)))
    return y
