#!/usr/bin/env python
"""Benchmark of the StrataFlux refined low-bit decode hot path on B200.

One step = the whole hot path of one decode token of a 32-layer
Llama-3.1-8B-shaped model at 32K context, batch 1:

  per layer: top-3% channel selection of the four linear-layer inputs
  (qkv, o, gate/up, down), one LRU refinement-cache step per weight matrix
  (10% of columns cached, misses gathered from pinned host memory on a side
  stream, issued one layer ahead = fetch lead), the seven refined GEMVs
  (2-bit resident + 2-bit refinement, group 128), and refined decode
  attention over 32768 tokens (2-bit + 2-bit K/V, top-1% tokens per query
  head refined).

The step is captured once in a CUDA graph and replayed.  Weights (1.96 GB),
KV (0.6 GB) and the refinement stores stay resident; per step only the
synthetic activations/queries change (staged device-to-device inside the
timed region).  The working set (> 2.5 GB) is far larger than L2 (126 MB),
so no L2 flush is needed.

Metric: effective HBM GB/s = algorithmic bytes of the step / step time, with
tokens/s (= steps/s) alongside.  Prints one JSON line (rank 0).
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
TOK_PCT = 1


def workload(T):
    ctx = f"{T // 1024}k" if T % 1024 == 0 else str(T)
    return f"llama31_8b_decode_hotpath_{ctx}"


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
    ap.add_argument("--context", type=int, default=32768)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-extras", action="store_true", help="skip e2e / resident-only / roofline legs")
    ap.add_argument("--long-context", type=int, default=131072,
                    help="also time the refined step at this context (0: skip); part of the extras")
    return ap.parse_args()


# ------------------------------------------------------------------ accounting

# DRAM bytes per launch counted by ncu (dram__bytes_read.sum +
# dram__bytes_write.sum) for the kernels as they stand; the commands are in
# profiles/.  They are set back to None whenever the kernel changes.
ATTN_TRAFFIC_32K = 21377792          # attn_fused_kernel<4>, Hq 32, Hkv 8, T 32768, k 1%
GEMV_TRAFFIC_PER_LAUNCH = 15849088   # gemv_mma_kernel, mean of a layer's 4 launches (63.40 MB)


def gemv_bytes(N, K, k_sel):
    """Algorithmic HBM bytes of one refined GEMV at batch 1."""
    return N * K * B_R // 8 + 4 * N * K // G + k_sel * N * B_F // 8 + 2 * K + 4 * N


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
        # prepared activations: with the selection (refined step) and without (resident-only step)
        self.act = {s: torch.zeros((layers, sf.act_bytes(K) // 4), dtype=torch.int32, device=device) for s, K in SLOTS}
        self.act0 = {s: torch.zeros((layers, sf.act_bytes(K) // 4), dtype=torch.int32, device=device)
                     for s, K in SLOTS}
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
            self.selects.append(sf.SelectJobs([(self.x(l, s), self.ksel[s], self.idx[s][l], self.nsel[s][l],
                                                self.act[s][l]) for s, _ in SLOTS]))
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

        def prepare_only(l):
            # the resident-only step prepares its activations the same way,
            # one layer ahead on the selection stream; main waits for them
            ev = torch.cuda.Event()
            ev.record(main)
            self.sel_stream.wait_event(ev)
            with torch.cuda.stream(self.sel_stream):
                for s, _ in SLOTS:
                    sf.act_prepare(self.x(l, s), self.act0[s][l])
                done = torch.cuda.Event()
                done.record(self.sel_stream)
            return done

        def gemv(l, slot):
            if refine:
                self.jobs[l][slot].run(self.x(l, slot), self.act[slot][l])
            else:
                self.jobs0[l][slot].run(self.x(l, slot), self.act0[slot][l])

        ready = {}
        if refine:
            select_and_prefetch(0)
        else:
            ready[0] = prepare_only(0)
        for l in range(self.L):
            if refine and l + 1 < self.L:
                select_and_prefetch(l + 1)
            if not refine:
                if l + 1 < self.L:
                    ready[l + 1] = prepare_only(l + 1)
                main.wait_event(ready.pop(l))
            gemv(l, "attn_in")
            sf.attn_decode_refine(self.qin[l], self.kv[l], HKV, self.T, self.k_tok if refine else 0,
                                  workspace=self.ws, out=self.attn_out[l], sel_out=self.sel_out[l],
                                  sel_n=self.sel_n[l])
            for slot in ("attn_out", "mlp_in", "mlp_mid"):
                gemv(l, slot)

    def gemvs_only(self):
        for l in range(self.L):
            for slot, _ in GEMV_LAUNCHES:
                self.jobs[l][slot].run(self.x(l, slot), self.act[slot][l])

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


def capture(torch, fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        g.capture_begin(capture_error_mode="relaxed")
        fn()
        g.capture_end()
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

def run_reference(args, rank):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    T = args.context
    for i in range(args.warmup):
        oracle_sample_step(T, which=i)
    t_tot, b_tot = 0.0, 0
    for i in range(args.steps):
        dt, nb = oracle_sample_step(T, which=args.warmup + i)
        t_tot += dt
        b_tot += nb
    gbs = b_tot / t_tot / 1e9
    cores = blas_threads()
    sample = (f"per step one of the 7 Llama-3.1-8B-shaped linear layers (cycled) with selection, one LRU step and "
              f"the refined GEMV, plus refined attention of one KV head (4 query heads) at T={T}")
    line = {
        "impl": "reference", "metric": "effective HBM GB/s (refined low-bit decode hot path)", "value": gbs,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy draws)",
        "config": {"workload": workload(T), "context": T, "layers": args.layers, "batch": 1},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_sf(args, rank, world, local_rank, dist):
    import torch
    import quantized_gemv_kv_b200 as sf
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T = args.context
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
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    phys = vis.split(",")[local_rank].strip() if vis else str(local_rank)
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
        # launch of the same kernel (profiles/attn_fused_kernel_32k.md)
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
        # layer, per launch (profiles/gemv_mma_kernel_gateup_llama31_8b.md)
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

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        dt, nb = oracle_sample_step(T)
        cpu = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"one full layer: 7 refined linears (selection, LRU step, GEMV) + refined attention "
                         f"of all 8 KV heads at T={T}; {dt:.1f} s"}

    line = {
        "metric": "effective HBM GB/s (refined low-bit decode hot path)", "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded on-device draws; random-init weights)",
        "config": {"workload": workload(T), "model_shape": "Llama-3.1-8B (32 layers)", "context": T,
                   "layers": args.layers, "batch": 1, "weights": "2-bit resident + 2-bit refinement, group 128",
                   "kv": "2-bit + 2-bit, per token-head", "topk_channels": "3%", "cache": "10% LRU per matrix",
                   "topk_tokens": "1% per query head", "l2": "working set > L2, no flush",
                   "parallelism": f"replicas x{world}", "graph": "CUDA graph per step"},
        "tokens_per_s": tok_s,
        "bytes_per_step": step_bytes,
        "h2d_miss_bytes_per_step": h2d_step,
        "cache_hit_rate": hits / max(1, hits + miss),
        "union_tokens_per_layer": union_per_layer,
        "gpu_launches": model.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    if roofline is not None:
        line["roofline"] = roofline
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    line.update(extras)
    torch.cuda.synchronize()
    del g
    model.close()
    del model
    if not args.skip_extras and args.long_context and args.long_context != T:
        line["long_context"] = long_context_leg(args, sf, torch, dist, dev, world, args.long_context)
    if rank == 0:
        print(json.dumps(line), flush=True)


def long_context_leg(args, sf, torch, dist, dev, world, T):
    """The same refined decode step with every layer's KV at context T
    (128K by default: the context the tokens/s figure is quoted at), timed
    the same way over fewer steps."""
    model = Model(sf, torch, args.layers, T, dev)
    steps, warm = min(args.steps, 20), 3
    n_total = min(warm + steps, 32)
    xpool, qpool = model.make_pools(n_total)
    cap_stream = torch.cuda.Stream(device=dev)
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

    for i in range(warm):
        with torch.cuda.stream(cap_stream):
            run_step(i)
    torch.cuda.synchronize()
    ms = timed(torch, dist, lambda i: run_step(warm + i), steps, cap_stream) / steps
    union = float(model.sel_n.cpu().clamp(min=0).sum(dim=1).float().mean())
    nbytes = attn_bytes(T, union) * args.layers
    for name, N, K, slot in MATS:
        nbytes += gemv_bytes(N, K, model.ksel[slot]) * args.layers
    # the attention alone, all layers in one graph
    g4 = capture(torch, model.attn_only, cap_stream)
    for _ in range(2):
        with torch.cuda.stream(cap_stream):
            g4.replay()
    ms_a = timed(torch, dist, lambda i: g4.replay(), 5, cap_stream) / 5 / args.layers
    del g, g4
    model.close()
    return {"context": T, "steps": steps, "warmup": warm, "ms_per_step": ms, "tokens_per_s": world * 1e3 / ms,
            "value": whole_job_gbs(nbytes, ms, world), "unit": "GB/s", "bytes_per_step": nbytes,
            "union_tokens_per_layer": union,
            "attention": {"kernel": "attn_fused_kernel" if cluster_attention(T)
                          else "attention pipeline (score, select, refine, out)",
                          "launch_us": ms_a * 1e3, "bytes_per_launch": attn_bytes(T, union),
                          "achieved_gbs": attn_bytes(T, union) / (ms_a * 1e-3) / 1e9}}


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
