"""CPU oracle for the grouped MoE expert MLP with MXFP8 / BF16 operands.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, deliberately
unoptimised restatement of what the layer computes, used to check the CUDA
library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` may import it.  The product path
(``mxfp8_quantize_b200``) never imports, calls or links anything here, and this
package imports nothing from the product path: the two share no code.

Sources (the pages are summaries of NVIDIA's tutorial "efficient MoE training
for biological foundation models" with Transformer Engine / BioNeMo):

* sitech.ge, "Grouped experts instead of a Python loop": one grouped GEMM
  driven by per-expert token counts (``split_sizes``) replaces the per-expert
  loop; the fused path adds MXFP8 quantisation and routing-weight scaling.
* sitech.ge, "Memory and quantization overhead": MXFP8 stores 8-bit values
  with one scaling factor per block of 32 consecutive values; 16-bit master
  weights are quantised every step; GroupedLinear -> ScaledSwiGLU ->
  GroupedLinear is the fused chain, with a matching backward.
* ai4snews, paragraphs 1 and 3: the per-expert loop the grouped call replaces,
  and the Sequential(GroupedLinear(gate_up), ScaledSwiGLU(), GroupedLinear(down))
  chain with SwiGLU and routing-probability scaling folded in.

Modules:
  mx       E4M3 / E8M0 codec (round-up shared exponent, RNE, satfinite)
  fp8      per-tensor FP8 codec (one fp32 scale per tensor, current scaling)
  routing  stable counting-sort permutation, padded expert segments
  moe      per-expert-loop forward and backward (MXFP8, per-tensor FP8 or BF16 operands)

Parity unpinned: Transformer Engine's own numerics (its exact shared-exponent
rule, gradient formats, where it applies the routing probability).  The pages
print no values that fix them; the readings used here are listed in each
module's docstring.
"""
