"""NVFP4 quantise / dequantise, step by step.  Test infrastructure only.

Passages followed:
  * "Gemma-4-26B-A4B-it-NVFP4" model page, block-scale formulas: contiguous
    blocks of 16 along the inner (K) dimension; S_block = max|w_i| / V_max,
    V_max = 6; q_i = clip(round(w_i / S_block), -6, 6); w_hat = q_i * S_block.
    The page prints this one-level form and an integer rounding; read with
    the two-level scheme of the other cards, "round" is round-to-nearest-even
    onto the E2M1 grid, and S_block is stored as E4M3 relative to a global.
  * "gemma-4-26B-A4B . NVFP4A16", "Quantization details" and
    "Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe": E2M1 codes, E4M3
    per-16 block scale, per-tensor FP32 global scale; dequantised weight is
    E2M1 x E4M3 x F32.
  * The global scale maps the tensor's amax onto the largest block-scale
    value times the largest code: G = amax / (6 * 448).

Exact fp32 arithmetic (each step one correctly rounded float32 operation,
emulated with numpy float32, which is IEEE-correct):
  G    = f32(amax) / 2688
  t_b  = (amax_b / 6) / G
  s_b  = E4M3_rn_satfinite(t_b)
  d_b  = f32(s_b) * G
  x_i  = w_i / d_b
  q_i  = E2M1_rn(x_i), saturating at 6, sign bit = sign bit of w_i
Degenerate blocks (d_b == 0, including an all-zero tensor where G == 0) give
scale 0 and codes that carry only the sign bit.
"""
from __future__ import annotations

import numpy as np

from .formats import (bf16_to_f32, e2m1_decode, e2m1_encode, e4m3_decode,
                      e4m3_encode_satfinite, pack_nibbles, unpack_nibbles)

BLOCK = 16
E2M1_MAX = np.float32(6.0)
GLOBAL_DENOM = np.float32(6.0 * 448.0)   # 2688, exact in float32


def global_scale(w32: np.ndarray) -> np.float32:
    """Per-tensor FP32 global scale G = amax / 2688 of one tensor (float32)."""
    amax = np.max(np.abs(w32)) if w32.size else np.float32(0.0)
    return np.float32(np.float32(amax) / GLOBAL_DENOM)


def quantize_blocks(w: np.ndarray, G) -> tuple[np.ndarray, np.ndarray]:
    """The block and element steps for float32 values w [N, K] under a given
    FP32 global scale G: returns (packed uint8 [N, K/2], scales uint8 [N, K/16]).
    Weights take G from their own amax (quantize_tensor); activations of the
    W4A4 form take a static per-projection G (oracle/w4a4.py)."""
    w = np.asarray(w, np.float32)
    G = np.float32(G)
    n, k = w.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 16")
    blocks = w.reshape(n, k // BLOCK, BLOCK)
    amax_b = np.max(np.abs(blocks), axis=-1)                      # float32, exact
    if G > 0:
        with np.errstate(over="ignore"):
            t = (amax_b / np.float32(6.0)) / G                    # two fp32 divides
        s = e4m3_encode_satfinite(t.astype(np.float64))
    else:
        s = np.zeros(amax_b.shape, np.uint8)
    s_val = e4m3_decode(s).astype(np.float32)                     # exact
    d = (s_val * G).astype(np.float32)                            # one fp32 multiply
    with np.errstate(divide="ignore", invalid="ignore"):
        x = blocks / d[..., None]                                 # fp32 divide
    codes = e2m1_encode(x)
    degenerate = (d == 0)[..., None] & np.ones_like(codes, dtype=bool)
    sign_only = (np.signbit(blocks).astype(np.uint8) << 3)
    codes = np.where(degenerate, sign_only, codes)
    return pack_nibbles(codes.reshape(n, k)), s


def quantize_tensor(w_bits: np.ndarray):
    """Quantise one bf16 tensor [N, K] (bf16 bit patterns) with its own
    global scale.  Returns (packed uint8 [N, K/2], scales uint8 [N, K/16],
    G float32)."""
    w = bf16_to_f32(w_bits)
    if w.shape[1] % BLOCK:
        raise ValueError("K must be a multiple of 16")
    G = global_scale(w)
    q, s = quantize_blocks(w, G)
    return q, s, np.float32(G)


def quantize(w_bits: np.ndarray):
    """Quantise stacked expert weights [E, N, K] (bf16 bits), one global scale
    per expert.  Returns (q uint8 [E, N, K/2], s uint8 [E, N, K/16],
    g float32 [E])."""
    e, n, k = w_bits.shape
    q = np.empty((e, n, k // 2), np.uint8)
    s = np.empty((e, n, k // BLOCK), np.uint8)
    g = np.empty(e, np.float32)
    for j in range(e):
        q[j], s[j], g[j] = quantize_tensor(w_bits[j])
    return q, s, g


def dequantize(q: np.ndarray, s: np.ndarray, g) -> np.ndarray:
    """w_hat = E2M1 x E4M3 x G in float64 (exact).  q [..., N, K/2],
    s [..., N, K/16], g broadcastable to the leading dims (scalar for one
    tensor, [E] for a stack)."""
    codes = unpack_nibbles(q)
    v = e2m1_decode(codes)
    sv = e4m3_decode(s)
    k = codes.shape[-1]
    v = v.reshape(v.shape[:-1] + (k // BLOCK, BLOCK)) * sv[..., None]
    v = v.reshape(v.shape[:-2] + (k,))
    g = np.asarray(g, np.float64)
    return v * g.reshape(g.shape + (1,) * (v.ndim - g.ndim))


def dequantize_f32(q: np.ndarray, s: np.ndarray, g) -> np.ndarray:
    """The dequantised weight rounded once to float32 (the exact product
    E2M1 x E4M3 x G has at most 30 significant bits, so float64 holds it
    exactly and a single float32 rounding follows)."""
    return dequantize(q, s, g).astype(np.float32)
