"""CPU oracle for the StrataFlux selective-precision-streaming hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
executes this package.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.

Plain, slow and deliberately unoptimised: numpy and Python loops, fp64 for
every floating-point result except where the method fixes another precision
(the quantizer's fp32 division and fp16 scale, following the quantizer
definition in :mod:`oracle.quant`).  It shares no code with the CUDA path;
the only thing both consume is the seeded input generator package
``workloads``.

Sources.  The pages describing StrataFlux are:

* "StrataFlux: Memory-Hierarchy-Native Low-Bit LLM Inference" (arXiv
  2611.08363, abstract) -- the resident/refinement co-design, reuse of fetched
  precision across decode steps, 2-4-bit weights and 2-3-bit KV.
* The rag-lover.com explainer of StrataFlux, sections TL;DR, 既存手法との違い
  (differences from prior work), 限界と未検証の範囲 (limits) and 解説
  (dialogue): weights are selected by input-activation magnitude, KV by the
  attention weight seen through the low-bit keys; what is fetched is extra
  low-order bits that subdivide between resident levels (nested
  refinement), not an FP16 replacement; a cache miss leaves the resident
  precision; fetched precision is cached and reused.
* The rit.work article on StrataFlux precision streaming, which states that
  the selection rules and the representation cannot be recovered from the
  abstract.

Where the pages are silent (quantizer formula, packing, tie-breaks, cache
policy details) each module states the reading it takes.

Modules
-------
quant   nested quantization, packing, dequantization          (pinned)
select  top-k channel selection by |x|, union over the batch   (pinned)
cache   LRU refinement cache: hits, misses, bypass, slots       (pinned)
gemv    refined decode GEMV                                     (pinned)
attn    refined decode attention (token selection + recompute)  (pinned)
decode  one full decode step of a Llama-shaped model: RMSNorm, RoPE,
        KV append, refined GEMVs and attention, SiLU MLP, LM head (pinned)
"""

from . import quant, select, cache, gemv, attn  # noqa: F401
