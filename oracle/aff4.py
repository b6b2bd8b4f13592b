"""The aff4 expert codec (affine int4) in float64.  Test infrastructure only.

Passage followed: "Gemma 4 26B-A4B (MoE) - Core AI" card, "Compression
recipe": routed experts in affine int4, one fp16 scale and one fp16 bias per
(output row, K-block of 32); a q4_0 grid w = (q - 8) d is represented exactly
by scale = d, bias = -8 d.  So the dequantised weight is
    w = q * scale + bias,   q in 0..15 (unsigned 4-bit code).

Readings where the page is silent: codes are packed two per byte with element
2j in the low nibble of byte j (the NVFP4 layout of this library); gate_up
keeps the fused [gate; up] row order.  The page's quantiser ("MSE-optimal clip
over 6 candidates") is not restated: the experts are generated directly in
packed form, like the NVFP4 ones.
"""
from __future__ import annotations

import dataclasses

import numpy as np

BLOCK = 32


@dataclasses.dataclass
class Aff4Experts:
    """uint8 codes and fp16 scales / biases as uint16 bit patterns."""
    gate_up_q: np.ndarray  # uint8 [E, 2I, H/2]
    gate_up_s: np.ndarray  # uint16 (f16) [E, 2I, H/32]
    gate_up_b: np.ndarray  # uint16 (f16) [E, 2I, H/32]
    down_q: np.ndarray     # uint8 [E, H, I/2]
    down_s: np.ndarray     # uint16 (f16) [E, H, I/32]
    down_b: np.ndarray     # uint16 (f16) [E, H, I/32]
    codec: str = "aff4"

    @property
    def E(self) -> int:
        return self.gate_up_q.shape[0]

    @property
    def H(self) -> int:
        return self.gate_up_q.shape[2] * 2

    @property
    def I(self) -> int:
        return self.down_q.shape[2] * 2


def f16_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def unpack_u4(q: np.ndarray) -> np.ndarray:
    """uint8 [..., K/2] -> codes 0..15 [..., K], element 2j from the low nibble."""
    q = np.asarray(q, np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = q & 0xF
    out[..., 1::2] = q >> 4
    return out


def dequantize(q: np.ndarray, s_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """w = q * scale + bias per K-block of 32, float64 (exact: a 4-bit code
    times an fp16 value plus an fp16 value is exact in float64)."""
    codes = unpack_u4(q).astype(np.float64)
    k = codes.shape[-1]
    codes = codes.reshape(codes.shape[:-1] + (k // BLOCK, BLOCK))
    w = codes * f16_to_f64(s_bits)[..., None] + f16_to_f64(b_bits)[..., None]
    return w.reshape(w.shape[:-2] + (k,))


def expert_dense(experts: Aff4Experts, e: int):
    """Float64 dequantised weights of expert e: (W_gate_up [2I, H], W_down [H, I])."""
    return (dequantize(experts.gate_up_q[e], experts.gate_up_s[e], experts.gate_up_b[e]),
            dequantize(experts.down_q[e], experts.down_s[e], experts.down_b[e]))
