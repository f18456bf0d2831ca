"""Seeded synthetic inputs for the selective-precision-streaming hot path.

This package only draws random numbers and rounds them to the storage types
the method consumes (fp32 weights, bf16 activations and queries, fp32 K/V).
It holds none of the method's arithmetic: no quantizer, no selection, no
dequantization.  Both the CPU oracle (through the tests) and the CUDA path
take their inputs from here, so the two sides always see identical bytes.
"""

from .synth import (  # noqa: F401
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    gen_weight,
    gen_activations,
    gen_kv,
    gen_query,
    outlier_channels,
)
from .shapes import (  # noqa: F401
    count_fraction,
    LINEAR_512,
    LLAMA31_8B_LINEAR,
    QWEN3_8B_LINEAR,
    ATTN_32K,
    LLAMA31_8B_DECODE_128K,
    WORKLOADS,
)
