"""One decode step of a Llama-shaped model with nested-refined weights and KV,
chained from the library's calls (argument marshalling only: every step runs
in libsf's kernels).

The pages measure StrataFlux end to end on a decode step of a Llama-3.1-8B
sized model at 128K context (arXiv 2611.08363 abstract: tokens/s and GPU
memory with 3-bit weights and 2-bit KV).  Per layer, batch 1:

  n1 = RMSNorm(x)                         sf_norm_select (adds the previous
                                          layer's MLP output to x first, and
                                          selects n1's top channels)
  q, k, v = refined GEMVs of n1           the weight caches' prefetch,
                                          sf_gemv_refine_batch1
  q, k rotated to position T              sf_rope_qk (q also as bf16)
  k, v quantized, appended as token T     sf_kv_append (with a KV refinement
                                          cache, both rows and the rotation
                                          in one launch:
                                          sf_rope_kv_append_pair_cached)
  a = refined attention over T + 1        sf_attn_decode_refine (+ the KV
                                          refinement cache's prefetch)
  h = x + o(bf16(a))                      sf_round_select, GEMV, sf_norm_select
  n2 = RMSNorm(h)
  x' = h + down(bf16(silu(gate(n2)) up(n2)))   sf_silu_mul_select, GEMVs

then RMSNorm and the refined LM head give the logits.  Each GEMV refines the
top round_half_up(p K) channels of its own input (the explainer's 解説:
weights are refined where the input activation is large); the attention
refines the top round_half_up(p_tok (T + 1)) tokens per query head.

Refinement sources.  ``weight_cache_pct`` None keeps every weight matrix's
refinement store in device memory; a percentage gives each matrix an LRU
cache of that share of its columns fed from page-locked host memory on a side
stream: every fetch completes before its GEMV, or, with
``weight_deadline``, the GEMV refines only the selected columns already
cached and the misses are fetched after it for later steps.  ``kv_cache_pct`` None keeps
the K/V refinement bits in device memory; a percentage keeps them in host
memory behind a KV refinement cache per layer (units = token-heads, 64
bytes; one LRU per KV head holding that share of the head's capacity) that
the attention reads with the deadline reading: only the union tokens cached
when the step starts are refined, the misses are fetched for later steps
(at most ``kv_budget`` per KV head and step; the rest are late).

Every call is enqueued on the current stream (plus the side stream), so a
step can be captured in a CUDA graph; before capturing after eager steps
call :meth:`DecodeModel.sync`.
"""

from __future__ import annotations

from dataclasses import dataclass
from fractions import Fraction

import torch

from . import (PRODUCE_NORM, PRODUCE_ROUND, PRODUCE_SILU_MUL, QKV, Batch1Jobs, RefineCache, RefineGroup, act_bytes,
               attn_decode_refine, attn_union_units, attn_workspace_size, gemv_set_launch_overlap, kv_append,
               norm_select, pack_batch1, quantize_nested, rope_kv_append_pair_cached, rope_qk, round_select,
               silu_mul_select)

MATS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class Shape:
    layers: int = 32
    hidden: int = 4096
    mlp: int = 14336
    n_q: int = 32
    n_kv: int = 8
    head_dim: int = 128
    vocab: int = 128256
    w_bits: tuple = (3, 1)
    kv_bits: tuple = (2, 2)
    group: int = 128
    theta: float = 500000.0
    eps: float = 1e-5

    def mat_shape(self, name: str) -> tuple[int, int]:
        H, F, dq, dkv = self.hidden, self.mlp, self.n_q * self.head_dim, self.n_kv * self.head_dim
        return {"q": (dq, H), "k": (dkv, H), "v": (dkv, H), "o": (H, dq), "gate": (F, H), "up": (F, H),
                "down": (H, F), "head": (self.vocab, H)}[name]


def count_half_up(p: Fraction, n: int) -> int:
    """floor(p n + 1/2) in exact arithmetic (the configurations' count rule)."""
    p = Fraction(p)
    return int((2 * p.numerator * n + p.denominator) // (2 * p.denominator))


class _Matrix:
    """A quantized weight matrix with its refinement source."""

    def __init__(self, W: torch.Tensor, shape: Shape, k_sel: int, cache_pct, device, deadline: bool = False):
        b_r, b_f = shape.w_bits
        N, K = W.shape
        self.qw = pack_batch1(quantize_nested(W, shape.group, b_r, b_f), drop_canonical=True)
        self.cache = None
        self.host = None
        if cache_pct is not None:
            self.host = self.qw.ref.cpu().contiguous().pin_memory()
            self.qw.ref = None
            cap = count_half_up(Fraction(cache_pct) / 100, K)
            self.cache = RefineCache(K, N * b_f // 8, cap, max(k_sel, 1), self.host)
            if deadline:
                self.cache.set_deadline(True)
        self.y = torch.empty(N, dtype=torch.float32, device=device)

    def close(self):
        if self.cache is not None:
            self.cache.close()


class DecodeModel:
    """A Llama-shaped decoder whose step runs through libsf.

    ``weight(l, name, N, K)`` returns fp32 [N][K] device weights (name in
    q, k, v, o, gate, up, down; l = -1 with name "head" for the LM head);
    ``norm(l, which)`` fp32 [hidden] RMSNorm weights (which in norm1, norm2;
    l = -1: the final norm); ``kv(l)`` returns the initial context of layer l
    as fp32 (K, V) [n_kv][T0][head_dim] (K already rotated).  ``capacity``
    is the number of tokens per KV head the cache is allocated for."""

    def __init__(self, shape: Shape, weight, norm, kv, capacity: int, p: Fraction = Fraction(3, 100),
                 p_tok: Fraction = Fraction(1, 100), weight_cache_pct=None, kv_cache_pct=None,
                 kv_budget: int | None = None, weight_deadline: bool = False, fetch_lead: bool = False,
                 record: bool = False, fused_producers: bool = False, device=None):
        self.s = shape
        self.dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.p, self.p_tok = Fraction(p), Fraction(p_tok)
        self.S = capacity
        self.record = record
        self.deadline = weight_deadline and weight_cache_pct is not None
        self.lead = fetch_lead and self.deadline
        # fused_producers: each GEMV makes its own input row and selection in
        # its launch (sf_gemv_refine_batch1_produce); not with a blocking
        # cache prefetch, which needs the selection before the launch
        self.fused = fused_producers and (weight_cache_pct is None or self.deadline)
        H, F, d = shape.hidden, shape.mlp, shape.head_dim
        Hq, Hkv = shape.n_q, shape.n_kv
        dev = self.dev
        self.k_in = {"attn_in": count_half_up(self.p, H), "attn_out": count_half_up(self.p, Hq * d),
                     "mlp_in": count_half_up(self.p, H), "mlp_mid": count_half_up(self.p, F),
                     "head": count_half_up(self.p, H)}
        self.K_in = {"attn_in": H, "attn_out": Hq * d, "mlp_in": H, "mlp_mid": F, "head": H}
        slot_of = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out", "gate": "mlp_in",
                   "up": "mlp_in", "down": "mlp_mid"}
        # side streams at the default (lowest) priority: a step run on a
        # higher-priority stream keeps its critical path ahead of them
        self.side = torch.cuda.Stream(device=dev)      # weight caches' steps and gathers
        self.side_kv = torch.cuda.Stream(device=dev)   # the KV caches' bookkeeping and gathers
        self.layers = []
        kv_b_r, kv_b_f = shape.kv_bits
        self.kv_cache_pct = kv_cache_pct
        for l in range(shape.layers):
            L = {}
            for name in MATS:
                N, K = shape.mat_shape(name)
                W = weight(l, name, N, K)
                L[name] = _Matrix(W, shape, self.k_in[slot_of[name]], weight_cache_pct, dev, self.deadline)
                del W
            L["norm1"] = norm(l, "norm1").to(dev, torch.float32).contiguous()
            L["norm2"] = norm(l, "norm2").to(dev, torch.float32).contiguous()
            Kc, Vc = kv(l)
            T0 = Kc.shape[1]
            if T0 > capacity:
                raise ValueError("initial context longer than the KV capacity")
            L["kv"], L["kv_host"], L["kv_cache"] = self._make_kv(Kc, Vc, capacity, kv_b_r, kv_b_f, kv_cache_pct,
                                                                kv_budget)
            del Kc, Vc
            L["T0"] = T0
            self.layers.append(L)
        Nh, Kh = shape.mat_shape("head")
        self.head = _Matrix(weight(-1, "head", Nh, Kh), shape, self.k_in["head"], weight_cache_pct, dev,
                            self.deadline)
        self.final_norm = norm(-1, "final").to(dev, torch.float32).contiguous()
        self._alloc_buffers()
        self._build_jobs(weight_cache_pct is not None)

    # ---- set-up -----------------------------------------------------------------------

    def _make_kv(self, Kc, Vc, S, b_r, b_f, cache_pct, budget):
        s, dev = self.s, self.dev
        Hkv, T0, d = Kc.shape
        rows = Hkv * S

        def quant(X):
            full = torch.zeros((Hkv, S, d), dtype=torch.float32, device=dev)
            full[:, :T0] = X.to(dev, torch.float32)
            return quantize_nested(full.view(rows, d), d, b_r, b_f, "by_row")
        qk, qv = quant(Kc), quant(Vc)
        host, cache = None, None
        kvq = QKV(qk, qv, row_stride=S)
        if cache_pct is not None:
            host = torch.cat([qk.ref.view(rows, -1), qv.ref.view(rows, -1)], dim=1).cpu().contiguous().pin_memory()
            qk.ref = qv.ref = None
            grp = s.n_q // Hkv
            k_max = count_half_up(self.p_tok, S)
            # one LRU per KV head: its share of the head's token-heads, its own budget
            cap = count_half_up(Fraction(cache_pct) / 100, S)
            cache = RefineCache(rows, host.shape[1] * 4, cap, max(1, grp * k_max), host, parts=Hkv)
            if budget is not None:
                cache.set_budget(budget)
            kvq.ref_cache = cache
        return kvq, host, cache

    def _alloc_buffers(self):
        s, dev = self.s, self.dev
        H, F, d, Hq, Hkv = s.hidden, s.mlp, s.head_dim, s.n_q, s.n_kv
        bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
        nl = s.layers
        # the residual stream, in two buffers: a launch that updates it reads
        # one and writes the other (its thread blocks read the old value)
        self.xr = torch.zeros((2, H), dtype=f32, device=dev)
        self.cur = 0
        self.read_evt = [None, None]
        self.x_in = torch.zeros(H, dtype=f32, device=dev)       # the step's input embedding
        self.buf = {}
        for slot in ("attn_in", "attn_out", "mlp_in", "mlp_mid"):
            K = self.K_in[slot]
            self.buf[slot] = dict(x=torch.zeros((nl, K), dtype=bf, device=dev),
                                  idx=torch.zeros((nl, max(1, self.k_in[slot])), dtype=i32, device=dev),
                                  n=torch.zeros((nl, 1), dtype=i32, device=dev),
                                  act=torch.zeros((nl, act_bytes(K) // 4), dtype=i32, device=dev))
        self.buf["head"] = dict(x=torch.zeros((1, H), dtype=bf, device=dev),
                                idx=torch.zeros((1, max(1, self.k_in["head"])), dtype=i32, device=dev),
                                n=torch.zeros((1, 1), dtype=i32, device=dev),
                                act=torch.zeros((1, act_bytes(H) // 4), dtype=i32, device=dev))
        self.q_bf = torch.zeros((nl, Hq, d), dtype=bf, device=dev)
        self.att = torch.zeros((nl, Hq, d), dtype=f32, device=dev)
        k_max = count_half_up(self.p_tok, self.S)
        grp = Hq // Hkv
        # per layer the union lists, rows of (Hq/Hkv) * k_tokens of the step (see union())
        self.sel = torch.zeros((nl, max(1, Hkv * grp * k_max)), dtype=i32, device=dev)
        self.sel_n = torch.zeros((nl, Hkv), dtype=i32, device=dev)
        self.units = torch.zeros((nl, max(1, Hkv * grp * k_max)), dtype=i32, device=dev)
        self.n_units = torch.zeros((nl, 1), dtype=i32, device=dev)
        self.logits = torch.zeros(s.vocab, dtype=f32, device=dev)
        self.ws = torch.empty(attn_workspace_size(Hq, Hkv, d, self.S, k_max), dtype=torch.uint8, device=dev)
        if self.record:
            self.x_hist = torch.zeros((nl + 1, H), dtype=f32, device=dev)   # x entering layer l; [nl]: final
            self.h_hist = torch.zeros((nl, H), dtype=f32, device=dev)
            self.k_rot = torch.zeros((nl, Hkv, d), dtype=f32, device=dev)
            self.qkv_raw = torch.zeros((nl, (Hq + 2 * Hkv) * d), dtype=f32, device=dev)   # GEMV outputs

    def _build_jobs(self, cached: bool):
        groups = {"attn_in": ("q", "k", "v"), "attn_out": ("o",), "mlp_in": ("gate", "up"), "mlp_mid": ("down",)}
        self.jobs, self.jobs0, self.wgroups = [], [], []
        for l, L in enumerate(self.layers):
            J, J0, G = {}, {}, {}
            for slot, names in groups.items():
                b = self.buf[slot]
                J[slot] = Batch1Jobs([(L[n].qw, L[n].cache, not cached, L[n].y) for n in names])
                J0[slot] = Batch1Jobs([(L[n].qw, None, False, L[n].y) for n in names])
                if cached:
                    G[slot] = RefineGroup([(L[n].cache, b["idx"][l], b["n"][l]) for n in names])
            self.jobs.append(J)
            self.jobs0.append(J0)
            self.wgroups.append(G)
        hb = self.buf["head"]
        self.head_job = Batch1Jobs([(self.head.qw, self.head.cache, not cached, self.logits)])
        self.head_job0 = Batch1Jobs([(self.head.qw, None, False, self.logits)])
        self.head_group = RefineGroup([(self.head.cache, hb["idx"][0], hb["n"][0])]) if cached else None
        # fetch lead: the predicted selections of the inputs fed by the
        # residual stream (q/k/v, gate/up, LM head) and their groups
        self.pred, self.pgroups, self.head_pgroup = {}, [], None
        if self.lead:
            dev, nl = self.dev, self.s.layers
            for slot in ("attn_in", "mlp_in", "head"):
                K, rows = self.K_in[slot], (1 if slot == "head" else nl)
                self.pred[slot] = dict(x=torch.zeros((rows, K), dtype=torch.bfloat16, device=dev),
                                       idx=torch.zeros((rows, max(1, self.k_in[slot])), dtype=torch.int32, device=dev),
                                       n=torch.zeros((rows, 1), dtype=torch.int32, device=dev))
            for l, L in enumerate(self.layers):
                self.pgroups.append({slot: RefineGroup([(L[n].cache, self.pred[slot]["idx"][l], self.pred[slot]["n"][l])
                                                        for n in groups[slot]]) for slot in ("attn_in", "mlp_in")})
            ph = self.pred["head"]
            self.head_pgroup = RefineGroup([(self.head.cache, ph["idx"][0], ph["n"][0])])

    @property
    def x(self) -> torch.Tensor:
        """The residual stream as it stands."""
        return self.xr[self.cur]

    # ---- the step -----------------------------------------------------------------------

    def _sel(self, l, slot, refine):
        """The (idx, n, act, k) arguments of the fused producer + selection
        that makes the input row of `slot` (k = 0: nothing selected)."""
        b = self.buf[slot]
        li = max(l, 0)
        return dict(k=self.k_in[slot] if refine else 0, idx=b["idx"][li], n=b["n"][li], act=None)

    def _linear(self, l, slot, refine, main):
        """The caches' step on the side stream and the batch-1 GEMV launch of
        the matrices reading `slot` (its row, selection and prepared
        activations made by the producer just before)."""
        b = self.buf[slot]
        x = b["x"][l:l + 1] if l >= 0 else b["x"]
        li = max(l, 0)
        if refine:
            grp = self.wgroups[l].get(slot) if l >= 0 else self.head_group
            if grp is not None and not self.deadline:
                grp.prefetch(main, self.side)   # the GEMV waits for these fetches
            (self.jobs[l][slot] if l >= 0 else self.head_job).run(x, b["idx"][li], b["n"][li])
            if grp is not None and self.deadline:
                grp.prefetch(main, self.side)   # for later steps; nothing waits within this one
        else:
            (self.jobs0[l][slot] if l >= 0 else self.head_job0).run(x)

    def _produce_linear(self, l, slot, refine, main, op, x, **kw):
        """The GEMVs of `slot` with their input row made in the same launch by
        ``op`` (sf_gemv_refine_batch1_produce); the caches' step for later
        steps follows on the side stream (deadline reading).  For
        PRODUCE_NORM the residual x + delta goes to the other residual
        buffer, which becomes the current one."""
        b = self.buf[slot]
        li = max(l, 0)
        k = self.k_in[slot] if refine else 0
        jobs = (self.jobs[l][slot] if l >= 0 else self.head_job) if refine else \
            (self.jobs0[l][slot] if l >= 0 else self.head_job0)
        y = b["x"][l] if l >= 0 else b["x"][0]
        if op == PRODUCE_NORM:
            kw["x_out"] = self.xr[1 - self.cur]
        jobs.run_produce(op, x, y, k, b["idx"][li], b["n"][li], eps=self.s.eps, **kw)
        if op == PRODUCE_NORM:
            self.cur ^= 1
        if refine:
            grp = self.wgroups[l].get(slot) if l >= 0 else self.head_group
            if grp is not None:
                grp.prefetch(main, self.side)   # for later steps; nothing waits within this one

    def _norm_linear(self, l, slot, norm_w, delta, refine, main, predict=None):
        """x += delta, RMSNorm, the selection, the GEMVs of `slot`; predict()
        runs once the updated residual is enqueued (before the GEMV launch
        when the producer is a launch of its own).  The residual buffer
        written (the other one when fused, else the current) must first have
        been read by any prediction that reads it."""
        target = 1 - self.cur if self.fused else self.cur
        if self.read_evt[target] is not None:
            main.wait_event(self.read_evt[target])
            self.read_evt[target] = None
        if self.fused:
            self._produce_linear(l, slot, refine, main, PRODUCE_NORM, self.x, delta=delta, w=norm_w)
            if predict is not None:
                predict()
        else:
            b = self.buf[slot]
            norm_select(self.x, norm_w, b["x"][l] if l >= 0 else b["x"], eps=self.s.eps, delta=delta,
                        **self._sel(l, slot, refine))
            if predict is not None:
                predict()
            self._linear(l, slot, refine, main)

    def _predict(self, l, slot, norm_w, main):
        """Fetch lead: select the channels the input of `slot` (layer l; the LM
        head for l < 0) will have, from the residual stream as it is now
        (RMSNorm of the current residual with that input's norm weights), and
        step those matrices' caches with the prediction, on the side stream,
        while the main stream goes on.  The main stream waits for the
        prediction's read of the residual buffer before it next writes that
        buffer."""
        pr = self.pred[slot]
        li = max(l, 0)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            norm_select(self.x, norm_w, pr["x"][li], k=self.k_in[slot], idx=pr["idx"][li], n=pr["n"][li], act=None,
                        eps=self.s.eps, delta=None)
            ev = torch.cuda.Event()
            ev.record(self.side)
        grp = self.pgroups[l][slot] if l >= 0 else self.head_pgroup
        grp.prefetch(self.side, self.side)
        self.read_evt[self.cur] = ev

    def step(self, T: int, refine: bool = True) -> None:
        """One decode step of the token at position T (T tokens already in
        every layer's cache); x_in holds the token's embedding.  refine=False
        is the quantization-only baseline: same kernels, nothing selected,
        fetched or refined."""
        prev = gemv_set_launch_overlap(True)  # no kernel of the step writes weights
        try:
            self._step(T, refine)
        finally:
            gemv_set_launch_overlap(prev)

    def _step(self, T: int, refine: bool) -> None:
        s = self.s
        if T + 1 > self.S:
            raise ValueError("the KV cache is full")
        main = torch.cuda.current_stream()
        H, d, Hq, Hkv = s.hidden, s.head_dim, s.n_q, s.n_kv
        b_r, b_f = s.kv_bits
        k_tok = count_half_up(self.p_tok, T + 1) if refine else 0
        self.k_tok = k_tok
        side_used = refine and any(self.wgroups) or (refine and self.head_group is not None)
        kv_used = False
        lead = refine and self.lead
        self.cur = 0
        self.read_evt = [None, None]  # per residual buffer: the last prediction that reads it
        self.x.copy_(self.x_in)
        prev = None
        for l, L in enumerate(self.layers):
            # lead: gate/up of this layer, predicted from the residual before the attention
            self._norm_linear(l, "attn_in", L["norm1"], prev, refine, main,
                              predict=(lambda: self._predict(l, "mlp_in", L["norm2"], main)) if lead else None)
            if self.record:
                self.x_hist[l].copy_(self.x)
            q, k, v = L["q"].y.view(Hq, d), L["k"].y.view(Hkv, d), L["v"].y.view(Hkv, d)
            if self.record:
                self.qkv_raw[l, :Hq * d].copy_(L["q"].y)
                self.qkv_raw[l, Hq * d:(Hq + Hkv) * d].copy_(L["k"].y)
                self.qkv_raw[l, (Hq + Hkv) * d:].copy_(L["v"].y)
            kq, vq = L["kv"].k, L["kv"].v
            if L["kv_cache"] is None:
                rope_qk(q, k, T, s.theta, q_bf16=self.q_bf[l])
                kv_append(k, kq.res, kq.ref, kq.scale, kq.zero, self.S, T, b_r, b_f)
                kv_append(v, vq.res, vq.ref, vq.scale, vq.zero, self.S, T, b_r, b_f)
            else:  # RoPE and the append in one launch; the new token's refinement bits go to the
                # host master (and a cached copy), the master's copy on the KV side stream
                rope_kv_append_pair_cached(q, k, v, kq, vq, L["kv_cache"], self.S, T, T, b_r, b_f, theta=s.theta,
                                           q_bf16=self.q_bf[l], stream=main, side=self.side_kv)
                kv_used = True
            if self.record:
                self.k_rot[l].copy_(k)
            attn_decode_refine(self.q_bf[l], L["kv"], Hkv, T + 1, k_tok, workspace=self.ws, out=self.att[l],
                               sel_out=self.sel[l], sel_n=self.sel_n[l])
            if L["kv_cache"] is not None and refine and k_tok > 0:
                # the union's units, the KV cache's step and its fetches all run
                # on their own side stream: nothing later in this step waits
                self.side_kv.wait_stream(main)
                attn_union_units(self.sel[l], self.sel_n[l], Hkv, (Hq // Hkv) * k_tok, self.S, self.units[l],
                                 self.n_units[l], stream=self.side_kv)
                L["kv_cache"].prefetch(self.units[l], self.n_units[l], self.side_kv, self.side_kv)
                kv_used = True
            if self.fused:
                self._produce_linear(l, "attn_out", refine, main, PRODUCE_ROUND, self.att[l].view(-1))
            else:
                round_select(self.att[l].view(-1), self.buf["attn_out"]["x"][l], **self._sel(l, "attn_out", refine))
                self._linear(l, "attn_out", refine, main)
            # lead: the next layer's q/k/v (or the LM head), from the residual after the attention
            last = l + 1 == s.layers
            nxt = self.final_norm if last else self.layers[l + 1]["norm1"]
            self._norm_linear(l, "mlp_in", L["norm2"], L["o"].y, refine, main,
                              predict=(lambda: self._predict(-1 if last else l + 1, "head" if last else "attn_in",
                                                             nxt, main)) if lead else None)
            if self.record:
                self.h_hist[l].copy_(self.x)
            if self.fused:
                self._produce_linear(l, "mlp_mid", refine, main, PRODUCE_SILU_MUL, L["gate"].y, u=L["up"].y)
            else:
                silu_mul_select(L["gate"].y, L["up"].y, self.buf["mlp_mid"]["x"][l],
                                **self._sel(l, "mlp_mid", refine))
                self._linear(l, "mlp_mid", refine, main)
            prev = L["down"].y
        self._norm_linear(-1, "head", self.final_norm, prev, refine, main)
        if self.record:
            self.x_hist[s.layers].copy_(self.x)
        # every fetch of the step (the KV caches' misses for later steps
        # included) completes within the step
        if side_used:
            main.wait_stream(self.side)
        if kv_used:
            main.wait_stream(self.side_kv)

    def union(self, l: int) -> list:
        """Layer l's union token lists of the last step (host lists)."""
        Hkv, grp = self.s.n_kv, self.s.n_q // self.s.n_kv
        cap = max(1, grp * self.k_tok)
        sel = self.sel[l, :Hkv * cap].view(Hkv, cap).cpu().numpy()
        n = self.sel_n[l].cpu().numpy()
        return [sel[g, : (n[g] if n[g] >= 0 else -1 - n[g])] for g in range(Hkv)]

    # ---- bookkeeping ---------------------------------------------------------------------

    def caches(self):
        out = []
        for L in self.layers:
            out += [L[n].cache for n in MATS if L[n].cache is not None]
            if L["kv_cache"] is not None:
                out.append(L["kv_cache"])
        if self.head.cache is not None:
            out.append(self.head.cache)
        return out

    def sync(self) -> None:
        """Host wait for every cache's last step (needed before capturing a
        graph after eager steps, and before reading cache statistics)."""
        for c in self.caches():
            c.stats()

    def cache_totals(self, kind: str) -> dict:
        tot = dict(steps=0, hits=0, misses=0, bypass=0, h2d_bytes=0, late=0)
        cs = []
        for L in self.layers:
            if kind == "weights":
                cs += [L[n].cache for n in MATS if L[n].cache is not None]
            elif L["kv_cache"] is not None:
                cs.append(L["kv_cache"])
        if kind == "weights" and self.head.cache is not None:
            cs.append(self.head.cache)
        for c in cs:
            st = c.stats()
            for key in tot:
                tot[key] += getattr(st, key)
        return tot

    def close(self) -> None:
        for G in self.wgroups + self.pgroups:
            for g in G.values():
                g.close()
        if self.head_pgroup is not None:
            self.head_pgroup.close()
        if self.head_group is not None:
            self.head_group.close()
        for L in self.layers:
            for n in MATS:
                L[n].close()
            if L["kv_cache"] is not None:
                L["kv_cache"].close()
        self.head.close()
