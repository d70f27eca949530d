"""CPU oracle for the JoLT KV-cache codec (numpy, float64).

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import or run anything in this package. The product library never
imports it, links it or falls back to it.

It is a plain, slow restatement of the method described in "A JoLT for the KV Cache:
Near-Lossless KV Cache Compression via Joint Tucker and JL-Residual Allocation for LLMs"
(arXiv 2607.12550v2, Abstract) and in the aimodeling.com news summary of the same
paper ("JoLT compresses KV cache to one-third with Tucker residuals", English summary):

* partial Tucker decomposition over the token and feature axes only, heads and layers
  left intact (Abstract; news summary, "Two details" paragraph);
* truncated energy restored by a random orthogonal rotation followed by low-bit
  quantisation of the residual (Abstract; "JL rotation whitens the low-bit residual",
  news summary);
* one Lagrangian dual choosing Tucker ranks and residual bit-widths per layer group,
  separately for keys and values, under one byte budget (Abstract);
* FlashJoLT, a randomized-SVD token factor (Abstract).

The pages give no formulas, so every concrete choice (Tucker algorithm, quantiser,
rotation construction, rank grid, error model, stream layout) is a stated reading,
documented next to the code that implements it. The oracle shares no code with the
CUDA path; both are fed from the seeded generators in `synth/`.
"""
from . import numerics, jolt, stream  # noqa: F401
