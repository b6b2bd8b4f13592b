"""The full Gemma-4 MoE block (the feed-forward half of a decoder layer) in
float64.  Test infrastructure only.

Passages followed ("Gemma 4 26B-A4B (MoE) - Core AI" card):
  * "Architecture" table: hidden 2816, dense MLP intermediate_size 2112,
    128 experts / top-8, moe_intermediate_size 704.
  * The layer dataflow listing under it: every layer runs a dense MLP and the
    sparse branch in parallel,
        residual = x
        h  = mlp(pre_feedforward_layernorm(x))            dense branch
        h1 = post_feedforward_layernorm_1(h)
        w, idx = router(residual)                         raw residual
        h2 = experts(pre_feedforward_layernorm_2(residual), idx)
        h2 = post_feedforward_layernorm_2(sum_k w_k h2_k)
        x  = residual + post_feedforward_layernorm(h1 + h2)
        x  = x * layer_scalar
    and the MLPs are GELU-gated with the tanh form of GELU.
  * "Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe", and the NVFP4A16
    card, "Quantization details": the dense MLP, the router and all norms stay
    BF16; activations are BF16.

Readings where the pages are silent:
  * Each of the five norms is an RMSNorm multiplied by its learned weight,
    x / sqrt(mean(x^2) + eps) * w, eps = 1e-6.
  * BF16 activations: the inputs of the two MLPs (the outputs of
    pre_feedforward_layernorm and pre_feedforward_layernorm_2) are rounded to
    bf16, as the block's bf16 modules receive them; everything else is kept
    exact (float64), and the block's output is rounded once to bf16.
  * layer_scalar is one bf16 scalar per layer.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .formats import bf16_to_f64, f64_to_bf16_rne
from . import moe as M


@dataclasses.dataclass
class BlockParams:
    """bf16 tensors as uint16 bit patterns."""
    experts: object                 # NVFP4 experts (oracle/moe layout)
    router: object                  # router parameters
    dense_gate: np.ndarray          # [Id, H]
    dense_up: np.ndarray            # [Id, H]
    dense_down: np.ndarray          # [H, Id]
    pre_ff_norm: np.ndarray         # [H]  pre_feedforward_layernorm
    post_ff_norm_1: np.ndarray      # [H]  post_feedforward_layernorm_1
    pre_ff_norm_2: np.ndarray       # [H]  pre_feedforward_layernorm_2
    post_ff_norm_2: np.ndarray      # [H]  post_feedforward_layernorm_2
    post_ff_norm: np.ndarray        # [H]  post_feedforward_layernorm
    layer_scalar: np.ndarray        # [1]
    eps: float = 1e-6


def rmsnorm(x: np.ndarray, w_bits, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w along the last axis, float64."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * bf16_to_f64(w_bits)


def dense_mlp(x: np.ndarray, gate_bits, up_bits, down_bits) -> np.ndarray:
    """The dense GELU-gated MLP: down(gelu_tanh(gate x) * up x), float64."""
    g = x @ bf16_to_f64(gate_bits).T
    u = x @ bf16_to_f64(up_bits).T
    return (M.gelu_tanh(g) * u) @ bf16_to_f64(down_bits).T


def forward(x_bits, p: BlockParams, ids_override=None, return_parts=False):
    """The block on x (bf16 bits [T, H], the post-attention hidden).  Returns
    the output in float64 (before its bf16 rounding) or, with return_parts, a
    dict with the intermediates as well."""
    res = bf16_to_f64(x_bits)
    x1 = f64_to_bf16_rne(rmsnorm(res, p.pre_ff_norm, p.eps))          # dense MLP input (bf16)
    h = dense_mlp(bf16_to_f64(x1), p.dense_gate, p.dense_up, p.dense_down)
    h1 = rmsnorm(h, p.post_ff_norm_1, p.eps)
    x2 = f64_to_bf16_rne(rmsnorm(res, p.pre_ff_norm_2, p.eps))        # experts' input (bf16)
    parts = M.forward(x2, p.experts, p.router, ids_override=ids_override, return_parts=True,
                      route_bits=x_bits)                              # router on the raw residual
    h2 = rmsnorm(parts["y64"], p.post_ff_norm_2, p.eps)
    out = (res + rmsnorm(h1 + h2, p.post_ff_norm, p.eps)) * bf16_to_f64(p.layer_scalar)[0]
    if not return_parts:
        return out
    return {"out64": out, "out_bf16": f64_to_bf16_rne(out), "x1": x1, "x2": x2, "h": h, "h1": h1,
            "y_moe": parts["y64"], "h2": h2, "ids": parts["ids"], "w": parts["w"], "logits": parts["logits"]}
