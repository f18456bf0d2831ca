#!/usr/bin/env python
"""Benchmark of StrataFlux refined low-bit decoding on B200.

Headline: one full decode step of a random-init 32-layer Llama-3.1-8B-shaped
model at 131072-token context, batch 1 (the configuration the pages' 128K
measurement names: 3-bit resident + 1-bit refinement weights, 2-bit + 2-bit
KV, RMSNorm, RoPE, SiLU MLP, LM head of 128256).  Per layer: top-3% channel
selection of every GEMV input, one LRU step per weight matrix (10% of its
columns cached in HBM, misses gathered from page-locked host memory on a side
stream before the GEMV that needs them), the refined GEMVs on the tensor
cores, RoPE, the new token quantized and appended, refined attention over
all 131072 tokens (top 1% tokens per query head; refinement bits from a KV
refinement cache of 10% of the token-heads, misses fetched for later steps
within a per-step budget), the MLP; then RMSNorm and the refined LM head.
The whole step is one CUDA graph; the working set (~5.7 GB) is far larger
than L2, so no flush is needed.

Metric: effective HBM GB/s (algorithmic bytes of the step / step time) and
tokens/s.  Extras: the quantization-only step (refinement overhead), the
attention's and the GEMVs' rooflines, host-link GB/s, GPU memory, the
end-to-end step through the public API with host buffers, and the 32K hot
path of round one (2+2-bit weights, independent per-layer inputs).  Prints
one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

MATS = (("q", 4096, 4096, "attn_in"), ("k", 1024, 4096, "attn_in"), ("v", 1024, 4096, "attn_in"),
        ("o", 4096, 4096, "attn_out"), ("gate", 14336, 4096, "mlp_in"), ("up", 14336, 4096, "mlp_in"),
        ("down", 4096, 14336, "mlp_mid"))
SLOTS = (("attn_in", 4096), ("attn_out", 4096), ("mlp_in", 4096), ("mlp_mid", 14336))
G, B_R, B_F = 128, 2, 2
HQ, HKV, D = 32, 8, 128
TOPK_PCT, CACHE_PCT, OUTLIER_PCT, OUTLIER_SCALE = 3, 10, "1/2", 30.0
# the headline metric; both arms (this library, and the oracle as the
# reference) report it under this name
METRIC = "effective HBM GB/s (refined low-bit decode step) and tokens/s at 128K"
TOK_PCT = 1


def workload(T):
    ctx = f"{T // 1024}k" if T % 1024 == 0 else str(T)
    return f"llama31_8b_decode_hotpath_{ctx}"


def workload_step(T):
    ctx = f"{T // 1024}k" if T % 1024 == 0 else str(T)
    return f"llama31_8b_decode_step_{ctx}"


# the full decode step: 3-bit resident + 1-bit refinement weights, LM head 128256
STEP_W_BITS = (3, 1)
VOCAB = 128256


def cluster_attention(T):
    """True where the library runs the attention as one cluster launch per
    layer (up to 32K tokens at <= 4 query heads per KV head), else it runs
    the score / selection / output pipeline."""
    return T <= 32768 and HQ // HKV <= 4
# matrices that read the same activation row share one batch-1 GEMV launch
GEMV_LAUNCHES = (("attn_in", ("q", "k", "v")), ("attn_out", ("o",)), ("mlp_in", ("gate", "up")),
                 ("mlp_mid", ("down",)))


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("sf", "reference"), default="sf")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--context", type=int, default=131072, help="tokens attended by the timed step")
    ap.add_argument("--kv-cache-pct", type=float, default=10.0,
                    help="KV refinement cache, percent of the token-heads (negative: the whole store in HBM)")
    ap.add_argument("--kv-budget", type=int, default=512,
                    help="KV refinement misses fetched per KV head and step at most (negative: no limit)")
    ap.add_argument("--weight-deadline", type=int, default=1,
                    help="1: GEMVs refine the selected columns already cached and misses are fetched for later "
                         "steps; 0: every GEMV waits for the fetch of its own selection")
    ap.add_argument("--fetch-lead", type=int, default=1,
                    help="1: prefetch the next residual-fed inputs' predicted channels a block ahead (with the "
                         "deadline reading)")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-extras", action="store_true", help="skip e2e / resident-only / roofline legs")
    ap.add_argument("--qwen3-batches", type=int, default=1,
                    help="also time Qwen3-8B decode linear layers at batch 1, 4 and 16 (0: skip); part of the extras")
    ap.add_argument("--hotpath-context", type=int, default=32768,
                    help="also time the 2+2-bit hot path at this context (0: skip); part of the extras")
    return ap.parse_args()


# ------------------------------------------------------------------ accounting

# DRAM bytes per launch counted by ncu (dram__bytes_read.sum +
# dram__bytes_write.sum) in a capture of the kernel as it stands, or None when
# the kernel has changed since its last capture.
ATTN_TRAFFIC_32K = 21377792          # attn_fused_kernel<4>, Hq 32, Hkv 8, T 32768, k 1%
GEMV_TRAFFIC_PER_LAUNCH = None       # gemv_mma_kernel (changed since its capture)
# the attention pipeline's four launches of one call (score, listing, ranking,
# output) at Hq 32, Hkv 8, T 131072, k 1%, from the one-layer step's launch
# list; ncu flushes the caches between launches, so each reader of the fp32
# scores counts them from DRAM (in the step they stay in L2)
ATTN_TRAFFIC_128K = 118992128


def gemv_bytes(N, K, k_sel, b_r=B_R, b_f=B_F):
    """Algorithmic HBM bytes of one refined GEMV at batch 1: resident codes,
    fp16 scale and zero per group, the selected columns' refinement bits, x
    in (bf16), y out (fp32)."""
    return N * K * b_r // 8 + 4 * N * K // G + k_sel * N * b_f // 8 + 2 * K + 4 * N


def attn_bytes(T, union_tokens):
    """Resident K and V codes + fp16 scale/zero of every token-head, the
    refinement bits of the refined token-heads, q in, out."""
    return HKV * T * 2 * (D * B_R // 8 + 4) + union_tokens * 2 * D * B_F // 8 + HQ * D * 2 + HQ * D * 4


# ------------------------------------------------------------------ clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # the timed region starts once the sampler has written its first line
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            try:
                if os.path.getsize(self.path) > 0:
                    break
            except OSError:
                pass
            time.sleep(0.02)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ model state

class Model:
    def __init__(self, sf, torch, layers, T, device):
        from workloads import device_synth as ds
        from workloads import count_fraction
        self.sf, self.torch, self.L, self.T, self.dev = sf, torch, layers, T, device
        self.k_tok = count_fraction(TOK_PCT, T)
        self.mats = []
        self.groups = []
        self.jobs = []
        self.jobs0 = []
        self.selects = []
        self.kv = []
        self.ksel = {s: count_fraction(TOPK_PCT, K) for s, K in SLOTS}
        ycount = sum(N for _, N, _, _ in MATS)
        self.y_all = torch.empty((layers, ycount), dtype=torch.float32, device=device)
        self.attn_out = torch.empty((layers, HQ, D), dtype=torch.float32, device=device)
        self.sel_out = torch.empty((layers, HKV, HQ // HKV * self.k_tok), dtype=torch.int32, device=device)
        self.sel_n = torch.empty((layers, HKV), dtype=torch.int32, device=device)
        xcount = sum(K for _, K in SLOTS)
        self.xin = torch.empty((layers, xcount), dtype=torch.bfloat16, device=device)
        self.qin = torch.empty((layers, HQ, D), dtype=torch.bfloat16, device=device)
        self.idx = {s: torch.zeros((layers, self.ksel[s]), dtype=torch.int32, device=device) for s, _ in SLOTS}
        self.nsel = {s: torch.zeros((layers, 1), dtype=torch.int32, device=device) for s, _ in SLOTS}
        self.ws = torch.empty(sf.attn_workspace_size(HQ, HKV, D, T, self.k_tok), dtype=torch.uint8, device=device)
        self.xoff = {}
        off = 0
        for s, K in SLOTS:
            self.xoff[s] = (off, K)
            off += K
        for l in range(layers):
            row = {}
            yo = 0
            for mi, (name, N, K, slot) in enumerate(MATS):
                W = ds.weight(1000 + l * 16 + mi, N, K, device=device)
                qw = sf.quantize_nested(W, G, B_R, B_F)
                del W
                master = qw.ref.cpu().pin_memory()
                qw.ref = None
                cache = sf.RefineCache(K, N * B_F // 8, count_fraction(CACHE_PCT, K), self.ksel[slot], master)
                row[name] = (qw, cache, self.y_all[l, yo:yo + N].view(1, N), slot)
                yo += N
            self.mats.append(row)
            self.groups.append(sf.RefineGroup([(cache, self.idx[slot][l], self.nsel[slot][l])
                                               for qw, cache, y, slot in row.values()]))
            self.jobs.append({slot: sf.Batch1Jobs([(row[n][0], row[n][1], False, row[n][2].view(-1)) for n in names])
                              for slot, names in GEMV_LAUNCHES})
            self.jobs0.append({slot: sf.Batch1Jobs([(row[n][0], None, False, row[n][2].view(-1)) for n in names])
                               for slot, names in GEMV_LAUNCHES})
            self.selects.append(sf.SelectJobs([(self.x(l, s), self.ksel[s], self.idx[s][l], self.nsel[s][l], None)
                                               for s, _ in SLOTS]))
            Kf, Vf = ds.kv(3000 + l, HKV, T, D, device=device)
            self.kv.append(sf.QKV(sf.quantize_nested(Kf, D, B_R, B_F, "by_row"),
                                  sf.quantize_nested(Vf, D, B_R, B_F, "by_row")))
            del Kf, Vf
        torch.cuda.synchronize()
        self.side = torch.cuda.Stream(device=device)
        self.sel_stream = torch.cuda.Stream(device=device)

    def x(self, l, slot):
        o, K = self.xoff[slot]
        return self.xin[l, o:o + K].view(1, K)

    def make_pools(self, n_steps):
        """Per-step synthetic activations and queries, generated on the device."""
        from workloads import device_synth as ds
        from workloads import count_fraction
        torch = self.torch
        xpool = torch.empty((n_steps,) + tuple(self.xin.shape), dtype=torch.bfloat16, device=self.dev)
        qpool = torch.empty((n_steps,) + tuple(self.qin.shape), dtype=torch.bfloat16, device=self.dev)
        outl = {}
        for l in range(self.L):
            for si, (s, K) in enumerate(SLOTS):
                outl[(l, s)] = ds.outlier_channels(5000 + l * 8 + si, K, count_fraction(OUTLIER_PCT, K), self.dev)
        for st in range(n_steps):
            for l in range(self.L):
                for si, (s, K) in enumerate(SLOTS):
                    o, _ = self.xoff[s]
                    xpool[st, l, o:o + K] = ds.activations(2000 + st * 4096 + l * 8 + si, 1, K, outl[(l, s)],
                                                           OUTLIER_SCALE, self.dev)[0]
                qpool[st, l] = ds.query(4000 + st * 64 + l, HQ, D, self.dev)
        return xpool, qpool

    # one decode step of the hot path; refine=False gives the resident-only
    # (quantization-only) baseline with no selection, cache or refinement
    def step(self, refine=True):
        sf, torch = self.sf, self.torch
        main = torch.cuda.current_stream()

        def select_and_prefetch(l):
            # Fetch lead: layer l's selection is computed from inputs available
            # when layer l-1 starts, on its own stream, and its misses are
            # gathered on the side stream; main waits only where the GEMV needs
            # the refinement rows.
            ev = torch.cuda.Event()
            ev.record(main)
            self.sel_stream.wait_event(ev)
            with torch.cuda.stream(self.sel_stream):
                self.selects[l].run()
            self.groups[l].prefetch(self.sel_stream, self.side)


        def gemv(l, slot):
            if refine:
                self.jobs[l][slot].run(self.x(l, slot), self.idx[slot][l], self.nsel[slot][l])
            else:
                self.jobs0[l][slot].run(self.x(l, slot))

        if refine:
            select_and_prefetch(0)
        for l in range(self.L):
            if refine and l + 1 < self.L:
                select_and_prefetch(l + 1)
            gemv(l, "attn_in")
            sf.attn_decode_refine(self.qin[l], self.kv[l], HKV, self.T, self.k_tok if refine else 0,
                                  workspace=self.ws, out=self.attn_out[l], sel_out=self.sel_out[l],
                                  sel_n=self.sel_n[l])
            for slot in ("attn_out", "mlp_in", "mlp_mid"):
                gemv(l, slot)

    def gemvs_only(self):
        for l in range(self.L):
            for slot, _ in GEMV_LAUNCHES:
                self.jobs[l][slot].run(self.x(l, slot), self.idx[slot][l], self.nsel[slot][l])

    def attn_only(self):
        for l in range(self.L):
            self.sf.attn_decode_refine(self.qin[l], self.kv[l], HKV, self.T, self.k_tok, workspace=self.ws,
                                       out=self.attn_out[l], sel_out=self.sel_out[l], sel_n=self.sel_n[l])

    def sync_caches(self):
        for row in self.mats:
            for qw, cache, y, slot in row.values():
                cache.stats()

    def cache_totals(self):
        tot = dict(hits=0, misses=0, bypass=0, h2d_bytes=0, steps=0)
        for row in self.mats:
            for qw, cache, y, slot in row.values():
                st = cache.stats()
                for k in tot:
                    tot[k] += getattr(st, k)
        return tot

    def launches_per_step(self, refine=True):
        """Kernels of the library per step: per layer the four GEMV launches,
        the attention (one cluster launch up to 32K at <= 4 query heads per KV
        head, else the pipeline's score, selection, refinement and output kernels), and
        either the selection, LRU index and miss gather (refined) or four
        activation preparations (resident only)."""
        gemv = len(GEMV_LAUNCHES) * self.L
        if cluster_attention(self.T):
            attn = self.L
        else:
            attn = (5 if (refine and 0 < self.k_tok < self.T) else 2) * self.L
        if not refine:
            return len(SLOTS) * self.L + gemv + attn
        return 3 * self.L + gemv + attn

    def close(self):
        for grp in self.groups:
            grp.close()
        for row in self.mats:
            for qw, cache, y, slot in row.values():
                cache.close()


def capture(torch, fn, stream, keep=False):
    g = torch.cuda.CUDAGraph(keep_graph=True) if keep else torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        g.capture_begin(capture_error_mode="relaxed")
        fn()
        g.capture_end()
    if keep:
        g.instantiate()
    torch.cuda.synchronize()
    return g


def reduce_max(value, dist, device):
    """Max of a per-rank float over all ranks (identity without a group)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step_per_rank, ms_per_step_max, world):
    """Whole-job throughput: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_step_per_rank / (ms_per_step_max * 1e-3) / 1e9


def timed(torch, dist, fn, iters, stream, sync_each=False):
    """Device time (ms) of `iters` calls of fn on `stream`, max over ranks."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(iters):
            fn(i)
            if sync_each:
                stream.synchronize()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1), dist, "cuda")
    if dist is not None:
        dist.barrier()
    return ms


# ------------------------------------------------------------------ CPU oracle

def oracle_sample_step(T, layer_seed=0, which=None):
    """Runs the CPU oracle on a bounded sample of the workload and returns
    (seconds, algorithmic bytes).  ``which`` selects one linear matrix (by
    index) and one KV head; None = one full layer (7 matrices + all heads)."""
    import numpy as np
    from oracle import attn as oattn, gemv as ogemv, quant as oquant, select as oselect, cache as ocache
    from workloads import synth, count_fraction
    mats = MATS if which is None else (MATS[which % len(MATS)],)
    prepared = []
    for mi, (name, N, K, slot) in enumerate(mats):
        W = synth.gen_weight(1000 + layer_seed * 16 + mi, N, K)
        qz = oquant.quantize_nested(W, G, B_R, B_F)
        outl = synth.outlier_channels(5000 + mi, K, count_fraction(OUTLIER_PCT, K))
        x = synth.gen_activations(2000 + mi, 1, K, outl, OUTLIER_SCALE)
        prepared.append((N, K, qz, x))
    hk = HKV if which is None else 1
    hq = HQ if which is None else HQ // HKV
    Kf, Vf, _ = synth.gen_kv(3000 + layer_seed, hk, T, D)
    qk = oquant.quantize_nested(Kf.reshape(-1, D), D, B_R, B_F)
    qv = oquant.quantize_nested(Vf.reshape(-1, D), D, B_R, B_F)
    qb = synth.gen_query(4000 + layer_seed, hq, D)
    k_tok = count_fraction(TOK_PCT, T)
    t0 = time.perf_counter()
    nbytes = 0
    for N, K, qz, x in prepared:
        k = count_fraction(TOPK_PCT, K)
        S = oselect.select_topk(x, k)
        c = ocache.LRUCache(K, count_fraction(CACHE_PCT, K))
        c.step(S.tolist())
        ogemv.gemv_refine(qz, x, S)
        nbytes += gemv_bytes(N, K, len(S))
    r = oattn.attn_decode_refine(qb, qk, qv, hk, T, k_tok)
    dt = time.perf_counter() - t0
    U = sum(len(u) for u in r["union"])
    nbytes += hk * T * 2 * (D * B_R // 8 + 4) + U * 2 * D * B_F // 8 + hq * D * 6
    return dt, nbytes


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ arms

def oracle_sample_step5(T, which, full=False):
    """The CPU oracle on a bounded sample of the full decode step at context T
    (3-bit resident + 1-bit refinement weights, 2+2-bit KV).  Item `which`
    cycles over the seven layer matrices (selection of the top 3% channels,
    one LRU step of a 10% cache, the refined GEMV) and the refined attention
    of one KV head (four query heads) over min(T, 16384) tokens; full=True
    takes all seven matrices and the attention over all T tokens.  Returns
    (seconds, algorithmic bytes, description)."""
    from oracle import attn as oattn, cache as ocache, gemv as ogemv, quant as oquant, select as oselect
    from workloads import synth, count_fraction
    b_r, b_f = STEP_W_BITS
    items = list(range(8)) if full else [which % 8]
    t_tot, nbytes, desc = 0.0, 0, []
    for it in items:
        if it < 7:
            name, N, K, slot = MATS[it]
            W = synth.gen_weight(1000 + it, N, K)
            qz = oquant.quantize_nested(W, G, b_r, b_f)
            outl = synth.outlier_channels(5000 + it, K, count_fraction(OUTLIER_PCT, K))
            x = synth.gen_activations(2000 + it, 1, K, outl, OUTLIER_SCALE)
            k = count_fraction(TOPK_PCT, K)
            t0 = time.perf_counter()
            S = oselect.select_topk(x, k)
            ocache.LRUCache(K, count_fraction(CACHE_PCT, K)).step(S.tolist())
            ogemv.gemv_refine(qz, x, S)
            t_tot += time.perf_counter() - t0
            nbytes += gemv_bytes(N, K, len(S), b_r, b_f)
            desc.append(name)
        else:
            Ts = T if full else min(T, 16384)
            Kf, Vf, _ = synth.gen_kv(3000 + which, 1, Ts, D)
            qk = oquant.quantize_nested(Kf.reshape(-1, D), D, B_R, B_F)
            qv = oquant.quantize_nested(Vf.reshape(-1, D), D, B_R, B_F)
            qb = synth.gen_query(4000 + which, HQ // HKV, D)
            t0 = time.perf_counter()
            r = oattn.attn_decode_refine(qb, qk, qv, 1, Ts, count_fraction(TOK_PCT, Ts))
            t_tot += time.perf_counter() - t0
            U = len(r["union"][0])
            nbytes += Ts * 2 * (D * B_R // 8 + 4) + U * 2 * D * B_F // 8 + (HQ // HKV) * D * 6
            desc.append(f"attention of one KV head over {Ts} tokens")
    return t_tot, nbytes, ", ".join(desc)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def step_config(args) -> dict:
    """The headline workload, as both arms report it in ``config``."""
    return {"workload": workload_step(args.context), "model_shape": "Llama-3.1-8B (32 layers, LM head 128256)",
            "context": args.context, "layers": args.layers, "batch": 1,
            "weights": "3-bit resident + 1-bit refinement, group 128", "kv": "2-bit + 2-bit, per token-head",
            "topk_channels": "3% of each GEMV input",
            "weight_cache": "10% LRU per matrix, " + ("deadline reading (misses fetched for later steps)"
                                                       if args.weight_deadline else "every GEMV waits for its misses")
            + ("; fetch lead: q/k/v, gate/up and LM-head channels predicted from the residual stream "
               "a block ahead and prefetched" if args.fetch_lead and args.weight_deadline else ""),
            "topk_tokens": "1% per query head",
            "kv_cache": (f"{args.kv_cache_pct}% of token-heads, one LRU per KV head, budget {args.kv_budget} per "
                         "head and step" if args.kv_cache_pct >= 0 else "store in HBM"),
            "position": "the step decodes position T = context - 1 every time (rewriting that row)"}


def run_reference(args, rank):
    """The CPU oracle as the reference arm (rank 0 only), on the headline's
    workload: each step one bounded item of the full decode step."""
    if rank != 0:
        return
    T = args.context
    for i in range(args.warmup):
        oracle_sample_step5(T, i)
    t_tot, b_tot = 0.0, 0
    for i in range(args.steps):
        dt, nb, _ = oracle_sample_step5(T, args.warmup + i)
        t_tot += dt
        b_tot += nb
    gbs = b_tot / t_tot / 1e9
    cores = blas_threads()
    sample = (f"per step one item of the full decode step at T={T}, cycled: one of the 7 Llama-3.1-8B-shaped "
              f"linear layers (3+1 bits: selection, LRU step, refined GEMV) or the refined attention of one KV "
              f"head over 16384 tokens; CPU {cpu_model()}")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy draws)",
        "config": step_config(args),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def hotpath_leg(args, sf, torch, dist, dev, world, T, phys):
    """The 2+2-bit hot path of one decode token at context T (round one's
    headline): per layer the four selections, seven cache steps and misses,
    seven refined GEMVs and the refined attention, every layer's inputs drawn
    independently.  Returns its numbers as a dict (an extra of the line)."""
    model = Model(sf, torch, args.layers, T, dev)
    # distinct per-step inputs, cycled: 32 steps apart, a channel's reuse
    # distance exceeds every refinement cache's capacity, so the cycle adds no
    # cache hits (the weights and KV make the working set larger than L2)
    n_total = min(args.warmup + args.steps, 32)
    xpool, qpool = model.make_pools(n_total)
    cap_stream = torch.cuda.Stream(device=dev)

    # warm-up eagerly once (cold caches fill), then capture the step
    model.xin.copy_(xpool[0])
    model.qin.copy_(qpool[0])
    with torch.cuda.stream(cap_stream):
        model.step()
    torch.cuda.synchronize()
    model.sync_caches()
    g = capture(torch, model.step, cap_stream)

    def run_step(i):
        model.xin.copy_(xpool[i % n_total], non_blocking=True)
        model.qin.copy_(qpool[i % n_total], non_blocking=True)
        g.replay()

    for i in range(args.warmup):
        with torch.cuda.stream(cap_stream):
            run_step(i)
    torch.cuda.synchronize()
    before = model.cache_totals()
    with ClockSampler(phys) as clk:
        ms = timed(torch, dist, lambda i: run_step(args.warmup + i), args.steps, cap_stream)
    clocks = clk.summary()
    after = model.cache_totals()
    sel_n = model.sel_n.cpu()
    union_per_layer = float(sel_n.clamp(min=0).sum(dim=1).float().mean())

    step_bytes = 0
    gemv_step_bytes = 0
    for name, N, K, slot in MATS:
        gemv_step_bytes += gemv_bytes(N, K, model.ksel[slot])
    gemv_step_bytes *= args.layers
    attn_step_bytes = attn_bytes(T, union_per_layer) * args.layers
    step_bytes = gemv_step_bytes + attn_step_bytes
    ms_step = ms / args.steps
    value = whole_job_gbs(step_bytes, ms_step, world)
    tok_s = world * 1e3 / ms_step
    h2d_step = (after["h2d_bytes"] - before["h2d_bytes"]) / args.steps
    hits = after["hits"] - before["hits"]
    miss = after["misses"] - before["misses"]

    extras = {}
    roofline = None
    e2e = None
    if not args.skip_extras:
        peaks = {}
        try:
            peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        except OSError:
            pass
        hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
        peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
        # the dominant kernel (largest share of the step's launch list): the
        # cluster attention; its launches of a step run in one graph, timed
        # with events on the launch stream.  traffic: ncu DRAM bytes of one
        # launch of the same kernel (ATTN_TRAFFIC_32K)
        model.sync_caches()
        reps = 5
        g4 = capture(torch, model.attn_only, cap_stream)
        for _ in range(2):
            with torch.cuda.stream(cap_stream):
                g4.replay()
        ms_a = timed(torch, dist, lambda i: g4.replay(), reps, cap_stream)
        t_attn = ms_a / reps / args.layers * 1e-3
        attn_launch_bytes = attn_step_bytes / args.layers
        achieved_a = attn_launch_bytes / t_attn / 1e9
        kname = "attn_fused_kernel" if cluster_attention(T) else "attention pipeline (score, select, refine, out)"
        roofline = {"bound": "hbm", "kernel": kname, "achieved": achieved_a, "peak": hbm_peak,
                    "unit": "GB/s", "frac": achieved_a / hbm_peak,
                    "traffic": ATTN_TRAFFIC_32K if (T == 32768 and HQ == 32 and HKV == 8) else None,
                    "peak_source": peak_src, "launch_us": t_attn * 1e6, "bytes_per_launch": attn_launch_bytes}
        del g4
        # the batch-1 GEMV, the next kernel by share: all its launches of a step
        # in one graph.  traffic: ncu DRAM bytes of the four launches of a
        # layer, per launch (GEMV_TRAFFIC_PER_LAUNCH)
        g2 = capture(torch, model.gemvs_only, cap_stream)
        for _ in range(2):
            with torch.cuda.stream(cap_stream):
                g2.replay()
        ms_g = timed(torch, dist, lambda i: g2.replay(), reps, cap_stream)
        n_launch = len(GEMV_LAUNCHES) * args.layers
        t_launch = ms_g / reps / n_launch * 1e-3
        achieved = gemv_step_bytes / n_launch / t_launch / 1e9
        extras["roofline_gemv"] = {"bound": "hbm", "kernel": "gemv_mma_kernel", "achieved": achieved,
                                   "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                                   "traffic": GEMV_TRAFFIC_PER_LAUNCH, "peak_source": peak_src,
                                   "launch_us": t_launch * 1e6, "bytes_per_launch": gemv_step_bytes / n_launch}
        del g2
        # resident-only (quantization-only) decode step, same kernels without refinement
        g3 = capture(torch, lambda: model.step(refine=False), cap_stream)
        for _ in range(2):
            with torch.cuda.stream(cap_stream):
                g3.replay()

        def run_res(i):
            model.xin.copy_(xpool[i % n_total], non_blocking=True)
            model.qin.copy_(qpool[i % n_total], non_blocking=True)
            g3.replay()
        ms_res = timed(torch, dist, run_res, args.steps, cap_stream) / args.steps
        extras["resident_only_ms_per_step"] = ms_res
        extras["refinement_overhead_pct"] = 100.0 * (ms_step / ms_res - 1.0)
        del g3
        # e2e: host inputs in, host results out, every step, through the same captured API calls
        model.sync_caches()
        hx = xpool.cpu().pin_memory()
        hq = qpool.cpu().pin_memory()
        hy = torch.empty(model.y_all.shape, dtype=torch.float32).pin_memory()
        ho = torch.empty(model.attn_out.shape, dtype=torch.float32).pin_memory()

        def run_e2e(i):
            model.xin.copy_(hx[i % n_total], non_blocking=True)
            model.qin.copy_(hq[i % n_total], non_blocking=True)
            g.replay()
            hy.copy_(model.y_all, non_blocking=True)
            ho.copy_(model.attn_out, non_blocking=True)
        for i in range(2):
            with torch.cuda.stream(cap_stream):
                run_e2e(i)
        ms_e2e = timed(torch, dist, lambda i: run_e2e(args.warmup + i), args.steps, cap_stream, sync_each=True)
        ms_e2e /= args.steps
        bi = model.xin.numel() * 2 + model.qin.numel() * 2
        bo = model.y_all.numel() * 4 + model.attn_out.numel() * 4
        e2e = {"value": whole_job_gbs(step_bytes, ms_e2e, world), "unit": "GB/s", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}

    out = {"workload": workload(T), "value": value, "unit": "GB/s", "ms_per_step": ms_step, "tokens_per_s": tok_s,
           "weights": "2-bit resident + 2-bit refinement, group 128", "bytes_per_step": step_bytes,
           "h2d_miss_bytes_per_step": h2d_step, "cache_hit_rate": hits / max(1, hits + miss),
           "union_tokens_per_layer": union_per_layer, "steps": args.steps, "clocks": clocks}
    if roofline is not None:
        out["roofline"] = roofline
    if e2e is not None:
        out["e2e"] = e2e
    out.update(extras)
    torch.cuda.synchronize()
    del g
    model.close()
    del model
    torch.cuda.empty_cache()
    return out


def qwen3_batch_leg(sf, torch, dist, dev, iters=20):
    """Qwen3-8B-shaped decode linear layers at 3+1 bits, group 128, batch 1,
    4 and 16: top 5% of channels per row, their union refined; one layer's
    seven GEMVs (batch 1: the integer tensor-core batch-1 path; 4 and 16:
    the f16 tensor-core batch path) with the selection of each distinct
    input (q/k/v share one, gate/up another), graph-timed over a pool
    of 8 seeded inputs per batch size.  "store": refinement bits read from
    HBM; "cache": a 25% LRU refinement cache per matrix stepped with the
    selection, its misses fetched from pinned host memory in the step (the
    union of 16 rows' selections misses most of such a cache, so that leg
    measures the host link)."""
    from fractions import Fraction
    from workloads import device_synth as ds
    from quantized_gemv_kv_b200.decode import count_half_up
    shapes = (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
              ("gate", 12288, 4096), ("up", 12288, 4096), ("down", 4096, 12288))
    b_r, b_f, G = 3, 1, 128
    mats = {}
    for i, (name, N, K) in enumerate(shapes):
        W = ds.weight(5000 + i, N, K, device=dev)
        qw = sf.quantize_nested(W, G, b_r, b_f)
        del W
        mats[name] = (qw, sf.pack_batch1(qw))
    torch.cuda.synchronize()
    out = {}
    stream = torch.cuda.Stream()
    for B in (1, 4, 16):
        caches, ys, bufs = {}, {}, {}
        for name, N, K in shapes:
            qw = mats[name][0]
            k = count_half_up(Fraction(5, 100), K)
            master = qw.ref.cpu().contiguous().pin_memory()
            caches[name] = sf.RefineCache(K, N * b_f // 8, count_half_up(Fraction(25, 100), K), min(K, B * k), master)
            ys[name] = torch.empty((B, N), dtype=torch.float32, device=dev)
        for K in (4096, 12288):
            k = count_half_up(Fraction(5, 100), K)
            pool = []
            for j in range(8):
                outl = torch.randperm(K, generator=torch.Generator(device="cpu").manual_seed(60 + j))[:K // 200]
                xf = torch.randn((B, K), generator=torch.Generator(device="cpu").manual_seed(70 + j))
                xf[:, outl] *= 30.0
                pool.append(xf.to(torch.bfloat16).to(dev))
            bufs[K] = (pool, k, torch.empty(B * k, dtype=torch.int32, device=dev),
                       torch.empty(1, dtype=torch.int32, device=dev))
        jobs1 = {name: sf.Batch1Jobs([(mats[name][1], caches[name], False, ys[name][0])]) for name, _, _ in shapes}
        jobs1s = {name: sf.Batch1Jobs([(mats[name][1], None, True, ys[name][0])]) for name, _, _ in shapes}

        def layer(i, cached):
            for name, N, K in shapes:
                pool, k, idx, n = bufs[K]
                x = pool[i % 8]
                if name in ("q", "o", "gate", "down"):  # k/v share q's input, up shares gate's
                    sf.select_topk(x, k, idx, n)
                if cached:
                    caches[name].prefetch(idx, n)
                if B == 1:
                    (jobs1 if cached else jobs1s)[name].run(x, idx, n)
                elif cached:
                    sf.gemv_refine(mats[name][0], x, idx, n, cache=caches[name], y=ys[name])
                else:
                    sf.gemv_refine(mats[name][0], x, idx, n, use_ref_store=True, y=ys[name])

        row = {"path": {1: "integer tensor cores (batch 1)", 4: "f16 tensor cores (batch 2-16)",
                        16: "f16 tensor cores (batch 2-16)"}[B]}
        for cached in (False, True):
            with torch.cuda.stream(stream):
                for i in range(8):
                    layer(i, cached)
            torch.cuda.synchronize()
            graphs = [capture(torch, lambda i=i: layer(i, cached), stream) for i in range(8)]
            for i in range(3):
                graphs[i % 8].replay()
            ms = timed(torch, dist, lambda i: graphs[i % 8].replay(), iters, stream)
            nbytes = 0
            for name, N, K in shapes:
                nbytes += gemv_bytes(N, K, bufs[K][1] * B, b_r, b_f) + 2 * K * (B - 1) + 4 * N * (B - 1)
            us = ms * 1e3 / iters
            row["cache" if cached else "store"] = {"us_per_layer": us, "tokens_per_s_per_layer": B * 1e6 / us,
                                                   "effective_gbs": nbytes / (us * 1e-6) / 1e9}
            del graphs
        out[f"batch_{B}"] = row
        for c in caches.values():
            c.close()
    return {"workload": "Qwen3-8B decode linear layers (q/k/v/o 4096, gate/up/down 12288), 3+1 bits, group 128, "
                        "top 5% per row, union refined; one layer's seven GEMVs with the selection of each input",
            **out}


def graph_kernels(g):
    """Kernel nodes of a captured graph (made with keep_graph=True), counted
    by kernel name: the library's launches read from the graph itself (memset
    and copy nodes are not counted)."""
    import re
    try:
        from cuda.bindings import driver as cd
        graph = cd.CUgraph(g.raw_cuda_graph())
        err, _, n = cd.cuGraphGetNodes(graph, 0)
        err, nodes, n = cd.cuGraphGetNodes(graph, n)
        names = {}
        for nd in nodes[:n]:
            err, t = cd.cuGraphNodeGetType(nd)
            if t != cd.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                continue
            err, prm = cd.cuGraphKernelNodeGetParams(nd)
            err, raw = cd.cuFuncGetName(prm.func)
            raw = raw.decode() if isinstance(raw, bytes) else str(raw)
            m = re.findall(r"[A-Za-z_]\w*kernel\w*", raw)
            key = max(m, key=len) if m else raw
            key = re.sub(r"^\d+", "", key)
            names[key] = names.get(key, 0) + 1
        return names
    except Exception as e:  # reported in the line instead of a count
        return {"error": repr(e)[:200]}


def host_link(torch, dev, nbytes=256 << 20, reps=5):
    """Page-locked host <-> HBM copy bandwidth (GB/s) measured in this run:
    the roofline of the refinement misses."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(device=dev)
    out = {}
    for name, fn in (("h2d_gbs", lambda: d.copy_(h, non_blocking=True)),
                     ("d2h_gbs", lambda: h.copy_(d, non_blocking=True))):
        with torch.cuda.stream(s):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(reps):
                fn()
            e1.record(s)
        torch.cuda.synchronize()
        out[name] = reps * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del h, d
    return out


def phys_gpu(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    return vis.split(",")[local_rank].strip() if vis else str(local_rank)


def step_model(args, sf, torch, dev, layers):
    """The full decode step's model: random-init Llama-3.1-8B shape (RMSNorm
    weights 1), 3+1-bit weights with 10% LRU caches per matrix, the initial
    context of every layer N(0, 1) K/V with 4 outlier key channels per KV head
    x10, 2+2-bit KV behind a KV refinement cache."""
    from fractions import Fraction
    from workloads import device_synth as ds
    from quantized_gemv_kv_b200.decode import DecodeModel, Shape
    T = args.context - 1
    shape = Shape(layers=layers)
    names = ("q", "k", "v", "o", "gate", "up", "down")

    def weight(l, name, N, K):
        seed = 1000 + l * 16 + names.index(name) if l >= 0 else 999
        return ds.weight(seed, N, K, device=dev)

    def norm(l, which):
        return torch.ones(shape.hidden, dtype=torch.float32)

    def kv(l):
        Kf, Vf = ds.kv(3000 + l, shape.n_kv, T, shape.head_dim, device=dev)
        return Kf.view(shape.n_kv, T, shape.head_dim), Vf.view(shape.n_kv, T, shape.head_dim)

    kv_pct = None if args.kv_cache_pct < 0 else args.kv_cache_pct
    budget = None if args.kv_budget < 0 else args.kv_budget
    m = DecodeModel(shape, weight, norm, kv, capacity=args.context, p=Fraction(TOPK_PCT, 100),
                    p_tok=Fraction(TOK_PCT, 100), weight_cache_pct=CACHE_PCT, kv_cache_pct=kv_pct,
                    kv_budget=budget, weight_deadline=bool(args.weight_deadline),
                    fetch_lead=bool(args.fetch_lead), device=dev)
    return m, T


def step_bytes(model, T, refined_tokens_per_layer):
    """Algorithmic HBM bytes of one decode step: every GEMV (resident codes,
    scale/zero, the selected columns' refinement bits from the HBM cache, x,
    y) and the attention of every layer (resident K/V codes and scale/zero of
    the T + 1 tokens, the refined token-heads' K and V refinement bits, q,
    out); the per-token norms, RoPE and append are a few KB and left out."""
    s = model.s
    b_r, b_f = s.w_bits
    gemv = 0
    slot_of = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out", "gate": "mlp_in",
               "up": "mlp_in", "down": "mlp_mid"}
    for name, slot in slot_of.items():
        N, K = s.mat_shape(name)
        gemv += gemv_bytes(N, K, model.k_in[slot], b_r, b_f)
    gemv *= s.layers
    Nh, Kh = s.mat_shape("head")
    gemv += gemv_bytes(Nh, Kh, model.k_in["head"], b_r, b_f)
    attn = s.layers * attn_bytes(T + 1, refined_tokens_per_layer)
    return gemv, attn


def run_sf(args, rank, world, local_rank, dist):
    import torch
    import quantized_gemv_kv_b200 as sf
    from workloads import device_synth as ds
    from workloads import count_fraction
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    phys = phys_gpu(local_rank)
    torch.cuda.synchronize()
    free0, total = torch.cuda.mem_get_info()
    model, T = step_model(args, sf, torch, dev, args.layers)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    free1, _ = torch.cuda.mem_get_info()
    H = model.s.hidden
    n_total = min(args.warmup + args.steps, 32)
    outl = ds.outlier_channels(5000, H, count_fraction(OUTLIER_PCT, H), dev)
    pool = torch.stack([ds.activations(2000 + i, 1, H, outl, OUTLIER_SCALE, dev)[0].float()
                        for i in range(n_total)])
    # the step's own stream above the side streams' priority (theirs is the
    # default, the lowest): when SMs free up, the critical path's blocks go
    # first (measured: 7.39 -> 7.33 ms per step at 128K)
    cap_stream = torch.cuda.Stream(device=dev, priority=-1)
    # one eager step (cold caches fill), then the step as one graph
    model.x_in.copy_(pool[0])
    with torch.cuda.stream(cap_stream):
        model.step(T)
    torch.cuda.synchronize()
    model.sync()
    g = capture(torch, lambda: model.step(T), cap_stream, keep=True)
    kernels = graph_kernels(g)

    def run_step(i):
        model.x_in.copy_(pool[i % n_total], non_blocking=True)
        g.replay()

    for i in range(args.warmup):
        with torch.cuda.stream(cap_stream):
            run_step(i)
    torch.cuda.synchronize()
    model.sync()
    w0, k0 = model.cache_totals("weights"), model.cache_totals("kv")
    with ClockSampler(phys) as clk:
        ms = timed(torch, dist, lambda i: run_step(args.warmup + i), args.steps, cap_stream)
    clocks = clk.summary()
    model.sync()
    w1, k1 = model.cache_totals("weights"), model.cache_totals("kv")
    ms_step = ms / args.steps
    L = args.layers
    union = sum(float(sum(len(u) for u in model.union(l))) for l in range(L)) / L
    if model.kv_cache_pct is not None:
        refined = (k1["hits"] - k0["hits"]) / args.steps / L
    else:
        refined = union
    gemv_b, attn_b = step_bytes(model, T, refined)
    nbytes = gemv_b + attn_b
    value = whole_job_gbs(nbytes, ms_step, world)
    free2, _ = torch.cuda.mem_get_info()
    wmiss = w1["h2d_bytes"] - w0["h2d_bytes"]
    kmiss = k1["h2d_bytes"] - k0["h2d_bytes"]

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        pass
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    extras, roofline, e2e = {}, None, None
    if not args.skip_extras:
        model.sync()
        k_tok = model.k_tok
        # the attention of every layer, in one graph (the step's dominant kernels)
        def attn_only():
            for l, Ly in enumerate(model.layers):
                sf.attn_decode_refine(model.q_bf[l], Ly["kv"], model.s.n_kv, T + 1, k_tok, workspace=model.ws,
                                      out=model.att[l], sel_out=model.sel[l], sel_n=model.sel_n[l])
        ga = capture(torch, attn_only, cap_stream)
        for _ in range(2):
            with torch.cuda.stream(cap_stream):
                ga.replay()
        reps = 5
        t_attn = timed(torch, dist, lambda i: ga.replay(), reps, cap_stream) / reps / L * 1e-3
        achieved = attn_b / L / t_attn / 1e9
        roofline = {"bound": "hbm", "kernel": "attention pipeline (attn_score_mma, attn_compact, attn_select, "
                                              "attn_out)",
                    "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                    "traffic": ATTN_TRAFFIC_128K if (T + 1 == 131072 and model.s.n_q == 32 and model.s.n_kv == 8)
                    else None,
                    "peak_source": peak_src, "launch_us": t_attn * 1e6,
                    "bytes_per_launch": attn_b / L}
        del ga
        # the GEMVs of the step (four launches per layer and the LM head), in one graph
        def gemvs_only():
            for l in range(L):
                for slot in ("attn_in", "attn_out", "mlp_in", "mlp_mid"):
                    b = model.buf[slot]
                    model.jobs0[l][slot].run(b["x"][l:l + 1])
            model.head_job0.run(model.buf["head"]["x"])
        gg = capture(torch, gemvs_only, cap_stream)
        for _ in range(2):
            with torch.cuda.stream(cap_stream):
                gg.replay()
        n_launch = 4 * L + 1
        t_g = timed(torch, dist, lambda i: gg.replay(), reps, cap_stream) / reps / n_launch * 1e-3
        res_b = sum(gemv_bytes(*model.s.mat_shape(n), 0, *model.s.w_bits) for n in
                    ("q", "k", "v", "o", "gate", "up", "down")) * L + gemv_bytes(*model.s.mat_shape("head"), 0,
                                                                                  *model.s.w_bits)
        ach_g = res_b / n_launch / t_g / 1e9
        extras["roofline_gemv"] = {"bound": "hbm", "kernel": "gemv_mma_kernel (3-bit resident, resident-only "
                                                             "launches as in the quantization-only step)",
                                   "achieved": ach_g, "peak": hbm_peak, "unit": "GB/s", "frac": ach_g / hbm_peak,
                                   "traffic": None, "peak_source": peak_src, "launch_us": t_g * 1e6,
                                   "bytes_per_launch": res_b / n_launch}
        del gg
        # the quantization-only step: same kernels, nothing selected, fetched or refined
        g0 = capture(torch, lambda: model.step(T, refine=False), cap_stream)

        def run_res(i):
            model.x_in.copy_(pool[i % n_total], non_blocking=True)
            g0.replay()
        for i in range(3):
            with torch.cuda.stream(cap_stream):
                run_res(i)
        ms_res = timed(torch, dist, run_res, args.steps, cap_stream) / args.steps
        extras["resident_only_ms_per_step"] = ms_res
        extras["refinement_overhead_pct"] = 100.0 * (ms_step / ms_res - 1.0)
        del g0
        # end to end through the public API: the token's embedding from
        # page-locked host memory in, the logits back to host memory, every step
        hx = pool.cpu().pin_memory()
        hl = torch.empty(model.logits.shape, dtype=torch.float32).pin_memory()

        def run_e2e(i):
            model.x_in.copy_(hx[i % n_total], non_blocking=True)
            g.replay()
            hl.copy_(model.logits, non_blocking=True)
        for i in range(2):
            with torch.cuda.stream(cap_stream):
                run_e2e(i)
        ms_e2e = timed(torch, dist, lambda i: run_e2e(args.warmup + i), args.steps, cap_stream,
                       sync_each=True) / args.steps
        e2e = {"value": whole_job_gbs(nbytes, ms_e2e, world), "unit": "GB/s", "ms_per_step": ms_e2e,
               "tokens_per_s": world * 1e3 / ms_e2e, "h2d_bytes_per_step": H * 4,
               "d2h_bytes_per_step": model.logits.numel() * 4}
        link = host_link(torch, dev)
        extras["host_link"] = dict(link, miss_bytes_per_step=(wmiss + kmiss) / args.steps,
                                   weight_miss_bytes_per_step=wmiss / args.steps,
                                   kv_miss_bytes_per_step=kmiss / args.steps,
                                   miss_gbs_over_step=(wmiss + kmiss) / args.steps / (ms_step * 1e-3) / 1e9)
    torch.cuda.synchronize()
    del g
    hot = None
    if not args.skip_extras and args.hotpath_context:
        model.close()
        del model
        torch.cuda.empty_cache()
        hot = hotpath_leg(args, sf, torch, dist, dev, world, args.hotpath_context, phys)
        model = None
    if not args.skip_extras and args.qwen3_batches:
        if model is not None:
            model.close()
            del model
            model = None
        torch.cuda.empty_cache()
        extras["qwen3_batches"] = qwen3_batch_leg(sf, torch, dist, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        try:
            from threadpoolctl import threadpool_limits
        except ImportError:
            threadpool_limits = None
        dt, nb, desc = oracle_sample_step5(T + 1, 0, full=True)
        cpu = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "cpu_model": cpu_model(), "logical_cpus": os.cpu_count(),
               "sample": f"one layer of the step: {desc} ({dt:.1f} s)"}
        if threadpool_limits is not None:
            with threadpool_limits(limits=1):
                dt1, nb1, _ = oracle_sample_step5(T + 1, 0, full=False)
            cpu["one_core"] = {"value": nb1 / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                               "sample": "the q projection's selection, LRU step and refined GEMV"}

    hits, miss = w1["hits"] - w0["hits"], w1["misses"] - w0["misses"]
    khits, kmisses = k1["hits"] - k0["hits"], k1["misses"] - k0["misses"]
    line = {
        "metric": METRIC, "value": value,
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded on-device draws; random-init weights and initial context)",
        "config": dict(step_config(args), **{"l2": "working set > L2, no flush",
                                             "parallelism": f"replicas x{world}", "graph": "CUDA graph per step"}),
        "tokens_per_s": world * 1e3 / ms_step,
        "bytes_per_step": nbytes,
        "gpu_memory_gb": (free0 - free1) / 1e9,
        "gpu_memory_gb_after_run": (free0 - free2) / 1e9,
        "weight_cache_hit_rate": hits / max(1, hits + miss),
        "kv_cache_hit_rate": khits / max(1, khits + kmisses),
        "kv_late_per_layer_step": (k1["late"] - k0["late"]) / args.steps / L,
        "union_tokens_per_layer": union,
        "refined_tokens_per_layer": refined,
        "gpu_launches": (sum(kernels.values()) * args.steps) if kernels and "error" not in kernels else None,
        "kernels_per_step": kernels,
        "clocks": clocks,
    }
    if roofline is not None:
        line["roofline"] = roofline
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    line.update(extras)
    if hot is not None:
        line["hotpath_32k"] = hot
    if model is not None:
        model.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        run_sf(args, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
