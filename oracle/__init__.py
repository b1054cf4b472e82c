"""Oracle: a plain, slow, single-threaded fp64 CPU statement of the routed-expert
HFQ4 MoE layer.

This package is TEST INFRASTRUCTURE.  Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with the CUDA library (``expert_offload_b200``): neither
imports the other; the seeded inputs of ``synth`` are the only thing both
consume.

Modules and what each follows (page title and section; readings where the
pages are silent are stated in each module):
  hfq4       HFQ4 block format, quantise / pack / dequantise
             -- hipfire RDNA engine thread, "HFQ quantisation format and GEMV"
  route      softmax top-k routing, renormalised weights, grouping by expert
             -- hipfire offload explainer, opening section (top-8 of many experts)
  moe        SwiGLU experts, weighted combine, dense cross-check, bf16 model
             of the tensor-core path, residual decode stack
             -- hipfire offload explainer, opening section (backbone vs experts)
  placement  layer split, auto fit-capacity, hot sets, loud refusal
             -- hipfire offload explainer, "placement algorithm"

Pins (all in tests/test_oracle_*.py, run without a GPU): hand-packed blocks
with known bytes (tests/golden), quantiser invariants, brute-force top-k over
all subsets, k = E softmax, a textbook SwiGLU MLP written out separately, a
closed form for constant weights, dense-vs-sparse agreement, and placement
brute force.  The pages print no worked numeric example, so every pin is by
construction; no function here is unpinned.
"""
from . import hfq4, moe, placement, route  # noqa: F401
