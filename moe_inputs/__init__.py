"""Seeded synthetic inputs for the NVFP4 weight-only MoE branch.

This module is shared by the tests, the benchmark and the CPU oracle.  It draws
random numbers and lays them out in the storage formats; it performs none of
the method's arithmetic (no quantisation, no routing, no expert maths).

Shapes follow the Gemma-4-26B-A4B MoE layer (Core AI port card, "Architecture"
table): hidden 2816, 128 experts, top-8, moe_intermediate 704.  The expert
storage follows the NVFP4 scheme of the NVFP4A16 release card ("Quantization
details"): packed E2M1 codes, one E4M3 block scale per 16 elements along K, one
FP32 global scale per expert projection.

Every array is a numpy array on the host.  bf16 tensors are carried as their
raw uint16 bit patterns so that both sides see identical bytes.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch

H = 2816        # hidden size
E = 128         # routed experts per layer
TOP_K = 8       # experts per token
I = 704         # moe_intermediate_size; gate_up has 2*I rows
BLOCK = 16      # elements per E4M3 block scale
DENSE_I = 2112  # the block's dense MLP intermediate size

__all__ = [
    "H", "E", "TOP_K", "I", "BLOCK", "Router", "Experts",
    "bf16_bits", "make_x", "make_router", "make_expert", "make_experts",
    "make_quant_expert", "make_quant_weights",
    "zipf_bias", "layer_seed_plan", "DENSE_I", "Block", "make_block", "make_aff4_experts",
]


def bf16_bits(a) -> np.ndarray:
    """Round a float array to bf16 with torch (round-to-nearest-even) and
    return the raw uint16 bit patterns."""
    t = torch.as_tensor(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@dataclasses.dataclass
class Router:
    proj: np.ndarray              # uint16 (bf16 bits) [E, H]
    scale: np.ndarray             # uint16 (bf16 bits) [H]
    per_expert_scale: np.ndarray  # uint16 (bf16 bits) [E]
    logit_bias: np.ndarray | None = None  # float32 [E] or None
    eps: float = 1e-6
    top_k: int = TOP_K

    @property
    def E(self) -> int:
        return self.proj.shape[0]

    @property
    def H(self) -> int:
        return self.proj.shape[1]


@dataclasses.dataclass
class Experts:
    gate_up_q: np.ndarray  # uint8 [E, 2I, H/2]   two E2M1 codes per byte
    gate_up_s: np.ndarray  # uint8 [E, 2I, H/16]  E4M3 block scales
    gate_up_g: np.ndarray  # float32 [E]          global scale
    down_q: np.ndarray     # uint8 [E, H, I/2]
    down_s: np.ndarray     # uint8 [E, H, I/16]
    down_g: np.ndarray     # float32 [E]

    @property
    def E(self) -> int:
        return self.gate_up_q.shape[0]

    @property
    def H(self) -> int:
        return self.gate_up_q.shape[2] * 2

    @property
    def I(self) -> int:
        return self.down_q.shape[2] * 2

    def nbytes_per_expert(self) -> int:
        return sum(a[0].nbytes for a in (self.gate_up_q, self.gate_up_s, self.down_q,
                                         self.down_s)) + 8


def make_x(seed: int, T: int, h: int = H) -> np.ndarray:
    """Activations x ~ N(0, 1), stored as bf16 bits [T, h]."""
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal((T, h), dtype=np.float32))


def zipf_bias(seed: int, e: int = E, beta: float = 0.015, s: float = 1.1) -> np.ndarray:
    """Zipf-shaped per-expert logit bias: b_e = -beta * s * ln(rank_e), with the
    ranks 1..e assigned by a seeded permutation.  Skews the per-expert token
    counts of a prefill batch (hot experts get >1000 of 4096 tokens)."""
    rng = np.random.default_rng(seed)
    rank = rng.permutation(e) + 1
    return (-beta * s * np.log(rank.astype(np.float64))).astype(np.float32)


def make_router(seed: int, e: int = E, h: int = H, bias: np.ndarray | None = None,
                top_k: int = TOP_K) -> Router:
    """proj ~ N(0, 0.02) [e, h]; scale ~ 1 + N(0, 0.05) [h];
    per_expert_scale ~ U(0.5, 1.5) [e]; all bf16."""
    rng = np.random.default_rng(seed)
    proj = rng.standard_normal((e, h), dtype=np.float32) * np.float32(0.02)
    scale = np.float32(1.0) + rng.standard_normal(h, dtype=np.float32) * np.float32(0.05)
    pes = rng.uniform(0.5, 1.5, size=e).astype(np.float32)
    return Router(bf16_bits(proj), bf16_bits(scale), bf16_bits(pes),
                  None if bias is None else np.asarray(bias, np.float32), 1e-6, top_k)


def _random_scale_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """E4M3 block-scale bytes whose values lie in [2^-3, 2^0): the exponent
    field is drawn uniformly over the three binades (fields 4, 5, 6) and the
    3-bit mantissa uniformly; the sign is positive.  This is a code-level
    stand-in for scales distributed as 2^U(-3, 0)."""
    exp_field = rng.integers(4, 7, size=shape, dtype=np.uint8)
    mant = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return (exp_field << 3) | mant


def make_expert(seed: int, j: int, h: int = H, i: int = I):
    """Expert j of a layer, generated from its own stream default_rng([seed, j])
    so that any single expert can be regenerated alone.  Returns
    (gate_up_q, gate_up_s, gate_up_g, down_q, down_s, down_g) for that expert."""
    rng = np.random.default_rng([seed, j])
    gu_g = np.float32(rng.uniform(1e-3, 4e-3))
    d_g = np.float32(rng.uniform(1e-3, 4e-3))
    gu_q = np.frombuffer(rng.bytes(2 * i * h // 2), np.uint8).reshape(2 * i, h // 2)
    gu_s = _random_scale_codes(rng, (2 * i, h // BLOCK))
    d_q = np.frombuffer(rng.bytes(h * i // 2), np.uint8).reshape(h, i // 2)
    d_s = _random_scale_codes(rng, (h, i // BLOCK))
    return gu_q, gu_s, gu_g, d_q, d_s, d_g


def make_experts(seed: int, e: int = E, h: int = H, i: int = I) -> Experts:
    """A layer's experts generated directly in packed form: uniformly random
    code bytes (two independent uniform E2M1 nibbles per byte, -0 included),
    E4M3 block scales per `_random_scale_codes`, FP32 global scales
    ~ U(1e-3, 4e-3) per expert per projection.  Expert j comes from
    `make_expert(seed, j)`."""
    gu_q = np.empty((e, 2 * i, h // 2), np.uint8)
    gu_s = np.empty((e, 2 * i, h // BLOCK), np.uint8)
    d_q = np.empty((e, h, i // 2), np.uint8)
    d_s = np.empty((e, h, i // BLOCK), np.uint8)
    gu_g = np.empty(e, np.float32)
    d_g = np.empty(e, np.float32)
    for j in range(e):
        gu_q[j], gu_s[j], gu_g[j], d_q[j], d_s[j], d_g[j] = make_expert(seed, j, h, i)
    return Experts(gu_q, gu_s, gu_g, d_q, d_s, d_g)


def make_quant_expert(seed: int, j: int, n: int, k: int, outlier_frac: float = 0.005,
                      outlier_mult: float = 20.0, std: float = 0.02) -> np.ndarray:
    """bf16 bits of expert j's weight [n, k] ~ N(0, std), with a seeded
    fraction `outlier_frac` of the entries multiplied by `outlier_mult`.
    Drawn from its own stream default_rng([seed, j])."""
    rng = np.random.default_rng([seed, j])
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(std)
    mask = rng.random((n, k), dtype=np.float32) < outlier_frac
    w[mask] *= np.float32(outlier_mult)
    return bf16_bits(w)


def make_quant_weights(seed: int, e: int, n: int, k: int, outlier_frac: float = 0.005,
                       outlier_mult: float = 20.0, std: float = 0.02) -> np.ndarray:
    """bf16 bits of expert weights [e, n, k]; expert j is
    `make_quant_expert(seed, j, ...)`."""
    out = np.empty((e, n, k), np.uint16)
    for j in range(e):
        out[j] = make_quant_expert(seed, j, n, k, outlier_frac, outlier_mult, std)
    return out


# Static input globals of the W4A4 form (the checkpoint's per-projection
# `input_scale`): amax / (6 * 448) for an activation range of 8 for the
# experts' input x ~ N(0, 1) and 2 for the gated hidden of these synthetic
# experts (|h| stays below 0.7 on seeded draws).  Inputs, not results.
W4A4_GX = np.float32(8.0 / 2688.0)
W4A4_GH = np.float32(2.0 / 2688.0)


def layer_seed_plan(n_layers: int = 30, base: int = 100) -> list[int]:
    """Seeds of an independently seeded layer stack (layer l uses base + l)."""
    return [base + l for l in range(n_layers)]


@dataclasses.dataclass
class Block:
    """The full MoE block's parameters besides the experts and the router
    (bf16 bit patterns): the dense GELU-gated MLP and the five norm weights,
    and the layer scalar."""
    dense_gate: np.ndarray      # [Id, H]
    dense_up: np.ndarray        # [Id, H]
    dense_down: np.ndarray      # [H, Id]
    pre_ff_norm: np.ndarray     # [H]
    post_ff_norm_1: np.ndarray  # [H]
    pre_ff_norm_2: np.ndarray   # [H]
    post_ff_norm_2: np.ndarray  # [H]
    post_ff_norm: np.ndarray    # [H]
    layer_scalar: np.ndarray    # [1]


def make_block(seed: int, h: int = H, di: int = DENSE_I) -> Block:
    """Dense MLP weights ~ N(0, 0.02); norm weights ~ 1 + N(0, 0.05);
    layer scalar ~ U(0.5, 1.0); all bf16."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((di, h), dtype=np.float32) * np.float32(0.02)
    u = rng.standard_normal((di, h), dtype=np.float32) * np.float32(0.02)
    d = rng.standard_normal((h, di), dtype=np.float32) * np.float32(0.02)
    norms = [np.float32(1.0) + rng.standard_normal(h, dtype=np.float32) * np.float32(0.05) for _ in range(5)]
    ls = np.array([rng.uniform(0.5, 1.0)], np.float32)
    return Block(bf16_bits(g), bf16_bits(u), bf16_bits(d), *[bf16_bits(n) for n in norms], bf16_bits(ls))


def make_aff4_experts(seed: int, e: int = E, h: int = H, i: int = I):
    """A layer's experts in the aff4 codec, generated directly in packed form
    (no quantiser): uniformly random 4-bit codes; per (row, K-block of 32) an
    fp16 scale ~ U(2e-4, 8e-4) and an fp16 bias = -scale * U(6, 9) (a grid
    centred near zero, as the q4_0 form w = (q - 8) d gives).  Expert j is
    drawn from default_rng([seed, 1000 + j]).  Returns oracle-shaped arrays:
    (gate_up_q, gate_up_s, gate_up_b, down_q, down_s, down_b) with the scales
    and biases as fp16 bit patterns."""
    def f16(a):
        return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)
    gq = np.empty((e, 2 * i, h // 2), np.uint8)
    gs = np.empty((e, 2 * i, h // 32), np.uint16)
    gb = np.empty_like(gs)
    dq = np.empty((e, h, i // 2), np.uint8)
    ds = np.empty((e, h, i // 32), np.uint16)
    db = np.empty_like(ds)
    for j in range(e):
        rng = np.random.default_rng([seed, 1000 + j])
        gq[j] = np.frombuffer(rng.bytes(2 * i * h // 2), np.uint8).reshape(2 * i, h // 2)
        s = rng.uniform(2e-4, 8e-4, size=(2 * i, h // 32)).astype(np.float32)
        gs[j], gb[j] = f16(s), f16(-s * rng.uniform(6, 9, size=s.shape).astype(np.float32))
        dq[j] = np.frombuffer(rng.bytes(h * i // 2), np.uint8).reshape(h, i // 2)
        s = rng.uniform(2e-4, 8e-4, size=(h, i // 32)).astype(np.float32)
        ds[j], db[j] = f16(s), f16(-s * rng.uniform(6, 9, size=s.shape).astype(np.float32))
    return gq, gs, gb, dq, ds, db
