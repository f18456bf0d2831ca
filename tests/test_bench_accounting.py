"""The bench's algorithmic byte counts (the numerators of every GB/s it
reports) against the sizes of the formats, and its workload naming."""

import bench


def test_gemv_bytes_of_a_llama_layer():
    # 2-bit codes (N K / 4 bytes), fp16 scale and zero per group of 128
    # (4 N K / 128), the selected columns' 2-bit refinement (k N / 4), the
    # bf16 input row and the fp32 output row
    assert bench.gemv_bytes(4096, 4096, 123) == 4096 * 4096 // 4 + 4 * 4096 * 32 + 123 * 4096 // 4 + 2 * 4096 \
        + 4 * 4096
    total = sum(bench.gemv_bytes(N, K, k) for (N, K, k) in
                [(4096, 4096, 123), (1024, 4096, 123), (1024, 4096, 123), (4096, 4096, 123),
                 (14336, 4096, 123), (14336, 4096, 123), (4096, 14336, 430)])
    resident = sum(N * K // 4 + N * K // 32 for (N, K) in
                   [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
                    (4096, 14336)])
    assert 61.0e6 < resident < 61.5e6       # the 61.3 MB of resident codes and scales per layer
    assert total - resident < 2.0e6          # refinement columns and activations: ~1.7 MB


def test_attn_bytes_of_32k_and_128k():
    # per token-head: 32 B of 2-bit K codes + 4 B of fp16 scale/zero, the
    # same for V; per refined token-head 32 B of K and 32 B of V refinement
    assert bench.attn_bytes(32768, 0) == 8 * 32768 * 72 + 32 * 128 * 6
    assert bench.attn_bytes(32768, 9670) - bench.attn_bytes(32768, 0) == 9670 * 64
    assert abs(bench.attn_bytes(131072, 38764.71875) - 78002990.0) < 1.0   # the 128K launch's figure


def test_workload_names_follow_the_context():
    assert bench.workload(32768) == "llama31_8b_decode_hotpath_32k"
    assert bench.workload(131072) == "llama31_8b_decode_hotpath_128k"
    assert bench.workload(1000) == "llama31_8b_decode_hotpath_1000"
    assert bench.cluster_attention(32768) and not bench.cluster_attention(32769)


def test_whole_job_value():
    # every rank's bytes over the slowest rank's time
    assert bench.whole_job_gbs(2e9, 1.0, 4) == 8000.0


def test_step_bytes_of_the_128k_decode_step():
    """The full decode step at 128K: 3-bit codes + scale/zero of 32 layers
    (~2.84 GB) and the LM head (~213 MB), 2-bit K/V of 131072 tokens x 8 KV
    heads x 32 layers (~2.42 GB); about 5.47 GB per token in all."""
    from fractions import Fraction
    from types import SimpleNamespace
    from quantized_gemv_kv_b200.decode import Shape, count_half_up
    s = Shape()
    p = Fraction(3, 100)
    k_in = {"attn_in": count_half_up(p, 4096), "attn_out": count_half_up(p, 4096), "mlp_in": count_half_up(p, 4096),
            "mlp_mid": count_half_up(p, 14336), "head": count_half_up(p, 4096)}
    assert k_in == {"attn_in": 123, "attn_out": 123, "mlp_in": 123, "mlp_mid": 430, "head": 123}
    gemv, attn = bench.step_bytes(SimpleNamespace(s=s, k_in=k_in), 131071, 0)
    layer_res = sum(N * K * 3 // 8 + N * K // 32 for N, K in (s.mat_shape(n) for n in
                    ("q", "k", "v", "o", "gate", "up", "down")))
    head_res = 128256 * 4096 * 3 // 8 + 128256 * 4096 // 32
    assert 2.83e9 < 32 * layer_res < 2.85e9 and 2.1e8 < head_res < 2.15e8
    assert 0 < gemv - 32 * layer_res - head_res < 4.0e7      # refinement columns (~29 MB) and activations
    assert attn == 32 * (8 * 131072 * 72 + 32 * 128 * 6)
    assert 5.4e9 < gemv + attn < 5.55e9


def test_bench_defaults(monkeypatch):
    """No flags: one GPU, a minutes-scale run, W >= 3 warm-up steps, the
    headline at 128K with the 32K hot path as an extra; --impl reference
    selects the oracle arm."""
    monkeypatch.setattr("sys.argv", ["bench.py"])
    a = bench.parse()
    assert (a.gpus, a.impl, a.context, a.hotpath_context) == (1, "sf", 131072, 32768)
    assert a.kv_cache_pct == 10.0 and a.kv_budget > 0
    assert a.warmup >= 3 and 1 <= a.steps <= 1000
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"])
    a = bench.parse()
    assert (a.impl, a.steps, a.warmup) == ("reference", 2, 3)


def test_both_arms_report_one_metric_and_workload(monkeypatch, capsys):
    """The reference arm (the CPU oracle) prints the headline's metric name
    and the same workload config as the library's arm; one step of it runs
    here, on the host."""
    import json
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    a = bench.parse()
    bench.run_reference(a, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["metric"] == bench.METRIC
    assert line["config"] == bench.step_config(a)
    assert line["config"]["workload"] == "llama31_8b_decode_step_128k"
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
