"""CPU oracle for the NVFP4 weight-only (W4A16) MoE branch.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the GPU path computes.  Only the tests, the graft entry's
smoke check and the benchmark's CPU-baseline leg may import it; the product
library never does, and it shares no code with the CUDA path.

Precision: fp64 throughout, except where the method fixes a narrower
arithmetic (the quantiser's fp32 scale and division steps, which are emulated
exactly with numpy float32 operations, and the bf16 rounding of the output).

Sources (page title, section):
  * "Gemma-4-26B-A4B-NVFP4-mlx" model card, "Quantization recipe" notes:
    NVFP4 = E2M1 x per-16 E4M3 block scale x per-tensor F32 (two levels).
  * "Gemma-4-26B-A4B-it-NVFP4" model page, block-scale formulas:
    S_block = max|w| / V_max with V_max = 6 (E2M1 maximum); q = clip(round(w/S)).
  * "gemma-4-26B-A4B . NVFP4A16" release card, "Quantization details":
    FP4 (E2M1) weights group 16, FP8 E4M3 scale + per-tensor FP32 global scale,
    BF16 activations.
  * "Gemma 4 26B-A4B (MoE) - Core AI" card, "Architecture": hidden 2816,
    128 experts, top-8, moe_intermediate 704; the layer dataflow listing and
    the router description (scale-free RMSNorm, x scale x hidden^-0.5, linear
    to 128, fp32 softmax, top-8, renormalise, x per_expert_scale; GELU-tanh
    gated experts).

  * The same card's layer dataflow listing, for the full block (oracle/block):
    a dense GELU-gated MLP (intermediate 2112) in parallel with the sparse
    branch, five norms, the router on the raw residual, and layer_scalar.

  * The same card's "Compression recipe", for the aff4 codec (oracle/aff4):
    affine int4 with an fp16 scale and bias per (row, K-block of 32).

Parity pins: every function here is pinned by a `-m "not gpu"` test against
closed forms, library routines (torch float8_e4m3fn, torch softmax/gelu/rms_norm,
numpy matmul), exhaustive enumeration or brute force on tiny inputs.  The
pages' own verification numbers need trained weights that are not available,
so the forward pass is pinned by invariants and brute force only.
"""
from . import formats, quantize, moe, block, aff4, w4a4  # noqa: F401
