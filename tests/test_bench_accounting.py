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


def test_bench_defaults(monkeypatch):
    """No flags: one GPU, a minutes-scale run, W >= 3 warm-up steps, the
    128K leg on; --impl reference selects the oracle arm."""
    monkeypatch.setattr("sys.argv", ["bench.py"])
    a = bench.parse()
    assert (a.gpus, a.impl, a.context, a.long_context) == (1, "sf", 32768, 131072)
    assert a.warmup >= 3 and 1 <= a.steps <= 1000
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"])
    a = bench.parse()
    assert (a.impl, a.steps, a.warmup) == ("reference", 2, 3)
