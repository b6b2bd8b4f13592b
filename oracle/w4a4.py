"""W4A4 form of the MoE branch: the activations are quantised to NVFP4 as
well, so each expert GEMM multiplies two FP4 operands.  Test infrastructure
only: the product path never imports this module.

Passages followed:
  * "Gemma-4-26B-A4B-NVFP4-mlx", opening description: the NVFP4 checkpoint
    carries, per expert projection, the packed codes, the block scales, the
    FP32 global (weight_scale_2) and an `input_scale` sidecar, the static
    per-tensor global of the projection's input activations.
  * "Gemma-4-26B-A4B-it-NVFP4", model README: built for native FP4 tensor-core
    execution; block-scale formulas (blocks of 16 along the inner dimension,
    V_max = 6), read in the two-level E2M1 x E4M3 x FP32 form as for weights.
  * "gemma-4-26B-A4B . NVFP4A16", Korean summary: W4A16 keeps BF16
    activations and gives up only the Blackwell activation speed-up that the
    W4A4 form takes.
  * Expert wiring, GELU-tanh gate and weighted combine as in oracle/moe.py.

Readings (the pages leave these open):
  * an activation row is quantised exactly as a weight row (oracle/quantize.py
    quantize_blocks), with the projection's static input global in place of
    amax / 2688: Gx for the experts' input x, Gh for the hidden h;
  * one Gx and one Gh per layer, shared by all experts, so a token's x is
    quantised once for its 8 slots;
  * the gated hidden h is formed in float64 and rounded once to float32, the
    precision in which the GPU path forms it, before its quantisation;
  * the GEMMs multiply the dequantised operands exactly (float64), the
    globals applied as written: gate_up = Gx * G_gu[e] * sum_k
    (E2M1*E4M3)_x (E2M1*E4M3)_w, likewise down with Gh * G_d[e].
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f32, f64_to_bf16_rne
from .moe import expert_dense, gelu_tanh, permute, route
from .quantize import dequantize, quantize_blocks


def quantize_act(v32: np.ndarray, G) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4 codes and E4M3 block scales of float32 activation rows [R, K]
    under the static global G: (packed uint8 [R, K/2], scales uint8 [R, K/16])."""
    return quantize_blocks(np.asarray(v32, np.float32), G)


def forward(x_bits, experts, router, gx, gh, ids_override=None, return_parts=False):
    """y = sum_j w_j * expert_{ids_j}(x) with both expert GEMMs on NVFP4
    operands, float64.  x_bits [T, H] bf16; gx, gh the input globals.
    With return_parts also returns the quantised x, the float32 hidden and
    its quantisation per slot (slot t*k + j)."""
    x32 = bf16_to_f32(x_bits)
    T, H = x32.shape
    ids, w, logits = route(x_bits, router, ids_override)
    k = ids.shape[1]
    xq, xs = quantize_act(x32, gx)
    xhat = dequantize(xq, xs, gx)                       # [T, H] float64, exact
    counts, offsets, sorted_slot, _ = permute(ids, experts.E)
    I = experts.I
    y = np.zeros((T, H), np.float64)
    h32_all = np.zeros((T * k, I), np.float32)
    hq_all = np.zeros((T * k, I // 2), np.uint8)
    hs_all = np.zeros((T * k, I // 16), np.uint8)
    for e in range(experts.E):
        if counts[e] == 0:
            continue
        slots = sorted_slot[offsets[e]:offsets[e + 1]]
        tok = slots // k
        wgu, wd = expert_dense(experts, e)
        gu = xhat[tok] @ wgu.T
        h32 = (gelu_tanh(gu[:, :I]) * gu[:, I:]).astype(np.float32)
        hq, hs = quantize_act(h32, gh)
        out = dequantize(hq, hs, gh) @ wd.T
        np.add.at(y, tok, w.ravel()[slots][:, None] * out)
        h32_all[slots], hq_all[slots], hs_all[slots] = h32, hq, hs
    if not return_parts:
        return y
    return {"y64": y, "y_bf16": f64_to_bf16_rne(y), "ids": ids, "w": w, "logits": logits,
            "xq": xq, "xs": xs, "h32": h32_all, "hq": hq_all, "hs": hs_all}


def down_from_codes(hq, hs, gh, ids, w, experts, T):
    """The down GEMM and combine alone, from given hidden codes per slot
    (slot t*k + j): y = sum_j w_j * G_d W_d deq(hq, hs, gh).  Lets a check
    start from the hidden codes another implementation produced."""
    k = ids.shape[1]
    y = np.zeros((T, experts.H), np.float64)
    hhat = dequantize(hq, hs, gh)
    for e in np.unique(ids):
        slots = np.nonzero(ids.ravel() == e)[0]
        _, wd = expert_dense(experts, int(e))
        np.add.at(y, slots // k, w.ravel()[slots][:, None] * (hhat[slots] @ wd.T))
    return y
