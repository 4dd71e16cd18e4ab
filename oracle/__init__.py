"""CPU oracle for the FFN-pool expert layer of attention-FFN disaggregation (AFD).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
this package: only the test suite, the entry point's smoke check and the CPU-baseline
leg of the benchmark use it. It shares no code with the CUDA path.

What it follows (FastAFD, "Methodology / System Design" items 1-3; vLLM AFD plugin,
"FFN service"):
  the FFN GPU receives block-FP8 tokens and top-K routing metadata from M attention
  ranks (the slabs), runs the routed experts as block-FP8 grouped GEMMs with the
  activation between them, and returns each token's combined output.

Modules:
  fp8      e4m3fn decode/encode from the OCP FP8 definition, bf16 round-to-nearest-even
  routing  the canonical routing: stable counting sort of (token, k) pairs by local expert
  ffn      dequantise -> W13 -> SwiGLU -> per-(row,128) FP8 requant -> W2 -> weighted combine,
           in float64; plus a brute-force per-token twin

Pins (tests/test_oracle_*.py): the codec against torch's float8/bfloat16 casts and OCP
values; routing against a sort-based brute force and invariants; the layer against a
dense SwiGLU FFN built from torch.matmul, a closed-form constant case, the
identical-experts case and slab re-splitting. The pages print no worked numeric example
for this layer, so no value is pinned to the pages themselves.
"""
from . import fp8, routing, ffn  # noqa: F401
