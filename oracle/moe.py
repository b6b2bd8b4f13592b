"""The sparse MoE branch in float64.  Test infrastructure only.

Passages followed ("Gemma 4 26B-A4B (MoE) - Core AI" card):
  * "Architecture" table: hidden 2816, 128 experts, top-8, moe_intermediate 704.
  * The layer dataflow listing under "Architecture": the router reads the raw
    residual; the experts produce per-slot outputs h2_k that are combined as
    sum_k w_k * h2_k.
  * The router description under the same listing: scale-free RMSNorm, times
    a learned scale, times hidden^-0.5, linear to the number of experts,
    softmax in fp32 over all experts, top-8, renormalise the eight
    probabilities to sum 1, multiply by a learned per_expert_scale gathered
    at the selected ids.  Experts are GELU-gated with the tanh form of GELU.
  * "New source modules": the fused gate_up_proj [E, 2*704, 2816] splits into
    separate gate and up stacks, gate first ("Gemma-4-26B-A4B-NVFP4-mlx",
    "How it was made": "fuse gate||up").
  * "Decode only ...": the batched variant sorts tokens by expert and runs a
    grouped GEMM per expert; the oracle groups slots by expert the same way
    and uses numpy matmul for each expert's GEMM.

Readings where the pages are silent:
  * RMSNorm epsilon 1e-6, added to mean(x^2) inside the square root.
  * Top-k order: descending probability, equal probabilities broken by the
    lower expert id; ids are returned in that order.
  * The logit bias (zero unless given) is added to the router linear's output.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, f64_to_bf16_rne
from .quantize import dequantize


# ------------------------------------------------------------------ router (a1)
def rmsnorm_scale_free(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) along the last axis, float64."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def router_logits(x_bits, router) -> np.ndarray:
    """Router logits [T, E]: rmsnorm(x) * scale * H^-0.5, then the linear map
    to E experts (plus the optional per-expert logit bias)."""
    x = bf16_to_f64(x_bits)
    H = x.shape[-1]
    r = rmsnorm_scale_free(x, router.eps) * bf16_to_f64(router.scale) * (H ** -0.5)
    logits = r @ bf16_to_f64(router.proj).T
    if router.logit_bias is not None:
        logits = logits + np.asarray(router.logit_bias, np.float64)
    return logits


def softmax(logits: np.ndarray) -> np.ndarray:
    """Softmax over the last axis in float64."""
    z = logits - np.max(logits, axis=-1, keepdims=True)
    e = np.exp(z)
    return e / np.sum(e, axis=-1, keepdims=True)


def top_k(p: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of each row, in descending order;
    ties broken by the lower index."""
    T, E = p.shape
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -p), axis=-1)
    return order[:, :k].astype(np.int32)


def route(x_bits, router, ids_override: np.ndarray | None = None):
    """The router: returns (ids int32 [T, k], weights float64 [T, k],
    logits float64 [T, E]).  With `ids_override` the given ids are used in
    place of the top-k selection (for comparing outputs where a near-tie
    makes several selections correct) and their weights are computed the
    same way."""
    logits = router_logits(x_bits, router)
    p = softmax(logits)
    ids = top_k(p, router.top_k) if ids_override is None else np.asarray(ids_override, np.int32)
    p_sel = np.take_along_axis(p, ids.astype(np.int64), axis=-1)
    w = p_sel / np.sum(p_sel, axis=-1, keepdims=True)
    w = w * bf16_to_f64(router.per_expert_scale)[ids]
    return ids, w, logits


# ---------------------------------------------------------------- permute (a2)
def permute(ids: np.ndarray, n_experts: int):
    """Group the T*k routing slots by expert.  Slot s = t*k + j.  Returns
    (counts [E], offsets [E+1], sorted_slot [T*k], slot_pos [T*k]) with slots
    of one expert in increasing slot order (a stable sort by expert id)."""
    flat = np.asarray(ids, np.int64).ravel()
    counts = np.bincount(flat, minlength=n_experts).astype(np.int32)
    offsets = np.zeros(n_experts + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    sorted_slot = np.argsort(flat, kind="stable").astype(np.int32)
    slot_pos = np.empty_like(sorted_slot)
    slot_pos[sorted_slot] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, sorted_slot, slot_pos


# ------------------------------------------------------------ experts (a3-a5)
def gelu_tanh(g: np.ndarray) -> np.ndarray:
    """GELU, tanh form: 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))."""
    g = np.asarray(g, np.float64)
    return 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))


def expert_dense(experts, e: int):
    """Float64 dequantised weights of expert e: (W_gate_up [2I, H], W_down [H, I]).
    NVFP4 experts here; experts of the aff4 codec dequantise through
    oracle/aff4.py."""
    if getattr(experts, "codec", "nvfp4") == "aff4":
        from . import aff4
        return aff4.expert_dense(experts, e)
    wgu = dequantize(experts.gate_up_q[e], experts.gate_up_s[e], experts.gate_up_g[e])
    wd = dequantize(experts.down_q[e], experts.down_s[e], experts.down_g[e])
    return wgu, wd


def expert_mlp(xe: np.ndarray, wgu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """One expert on the rows of xe [n, H]: gate||up = xe W_gu^T (gate rows
    first), h = gelu_tanh(gate) * up, out = h W_d^T.  Returns [n, H]."""
    I = wgu.shape[0] // 2
    gu = xe @ wgu.T
    h = gelu_tanh(gu[:, :I]) * gu[:, I:]
    return h @ wd.T


def expert_hidden(xe: np.ndarray, wgu: np.ndarray) -> np.ndarray:
    """The gated hidden h [n, I] of one expert (for checking the first GEMM
    and the GELU gate on their own)."""
    I = wgu.shape[0] // 2
    gu = xe @ wgu.T
    return gelu_tanh(gu[:, :I]) * gu[:, I:]


# --------------------------------------------------------------- forward (a6)
def forward(x_bits, experts, router, ids_override=None, return_parts=False, route_bits=None):
    """The MoE branch y = sum_j w_j * expert_{ids_j}(x), float64.

    By default the router and the experts read the same x (the branch on its
    own).  In the full block the router reads the raw residual while the
    experts read its pre-feedforward norm (the layer dataflow listing):
    `route_bits` is then the router's input and `x_bits` the experts'.
    Returns y64 [T, H] (float64) or, with return_parts, a dict that also holds
    ids, weights, logits and the bf16-rounded output."""
    x = bf16_to_f64(x_bits)
    T, H = x.shape
    ids, w, logits = route(x_bits if route_bits is None else route_bits, router, ids_override)
    counts, offsets, sorted_slot, _ = permute(ids, experts.E)
    k = ids.shape[1]
    y = np.zeros((T, H), np.float64)
    for e in range(experts.E):
        if counts[e] == 0:
            continue
        slots = sorted_slot[offsets[e]:offsets[e + 1]]
        tok = slots // k
        wgu, wd = expert_dense(experts, e)
        out = expert_mlp(x[tok], wgu, wd)
        wt = w.ravel()[slots]
        np.add.at(y, tok, wt[:, None] * out)
    if not return_parts:
        return y
    return {"y64": y, "y_bf16": f64_to_bf16_rne(y), "ids": ids, "w": w, "logits": logits}


def residual_rmsnorm(res: np.ndarray, y_bits, eps: float = 1e-6):
    """One link of a chained layer stack: res' = res + y, x' = bf16(rmsnorm(res')).
    `res` is float64 here (the oracle carries the residual in float64);
    returns (res', x' bf16 bits)."""
    res2 = np.asarray(res, np.float64) + bf16_to_f64(y_bits)
    return res2, f64_to_bf16_rne(rmsnorm_scale_free(res2, eps))
