"""torch conveniences over the C ABI: allocate outputs and workspaces with
torch (device memory plumbing) and pass their pointers to the library calls
on torch's current CUDA stream."""
from __future__ import annotations

import ctypes
import dataclasses

import numpy as np
import torch

from . import capi
from .capi import check

E, H, I, TOP_K = 128, 2816, 704, 8


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


@dataclasses.dataclass
class Router:
    """Router parameters on the device: proj bf16 [E, H], scale bf16 [H],
    per_expert_scale bf16 [E], optional logit_bias f32 [E]."""
    proj: torch.Tensor
    scale: torch.Tensor
    per_expert_scale: torch.Tensor
    logit_bias: torch.Tensor | None = None
    eps: float = 1e-6
    top_k: int = TOP_K

    def c_struct(self) -> capi.moe_router:
        return capi.moe_router(_ptr(self.proj), _ptr(self.scale), _ptr(self.per_expert_scale),
                               _ptr(self.logit_bias), self.proj.shape[0], self.proj.shape[1],
                               self.top_k, self.eps)

    @staticmethod
    def from_host(r, device="cuda") -> "Router":
        """From a host router of bf16 bit patterns (numpy uint16 arrays)."""
        def bf(a):
            return torch.from_numpy(a.view("int16")).view(torch.bfloat16).to(device)
        bias = None if r.logit_bias is None else torch.from_numpy(r.logit_bias).to(device)
        return Router(bf(r.proj), bf(r.scale), bf(r.per_expert_scale), bias, float(r.eps), int(r.top_k))


@dataclasses.dataclass
class Experts:
    """NVFP4 expert stacks on the device (layouts of include/nvfp4moe.h), with
    the optional packed copy of the codes (see packed())."""
    gate_up_q: torch.Tensor
    gate_up_s: torch.Tensor
    gate_up_g: torch.Tensor
    down_q: torch.Tensor
    down_s: torch.Tensor
    down_g: torch.Tensor
    gate_up_pk: torch.Tensor | None = None
    down_pk: torch.Tensor | None = None

    def c_struct(self) -> capi.moe_experts:
        return capi.moe_experts(_ptr(self.gate_up_q), _ptr(self.gate_up_s), _ptr(self.gate_up_g),
                                _ptr(self.down_q), _ptr(self.down_s), _ptr(self.down_g),
                                self.gate_up_q.shape[0], self.gate_up_q.shape[2] * 2,
                                self.down_q.shape[2] * 2, _ptr(self.gate_up_pk), _ptr(self.down_pk))

    def packed(self, stream=None) -> "Experts":
        """The same experts with the packed code tiles (moe_nvfp4_pack_codes)
        that the decode kernels stream as whole blocks; shares the other
        tensors."""
        if self.gate_up_pk is not None:
            return self
        E_ = self.gate_up_q.shape[0]
        dev = self.gate_up_q.device
        gu = torch.empty(capi.moe_pack_bytes(E_, 0), dtype=torch.uint8, device=dev)
        dn = torch.empty(capi.moe_pack_bytes(E_, 1), dtype=torch.uint8, device=dev)
        plain = dataclasses.replace(self, gate_up_pk=None, down_pk=None)
        check(capi.moe_nvfp4_pack_codes(ctypes.byref(plain.c_struct()), _ptr(gu), _ptr(dn), _stream(stream)),
              "moe_nvfp4_pack_codes")
        return dataclasses.replace(self, gate_up_pk=gu, down_pk=dn)

    @staticmethod
    def from_host(x, device="cuda") -> "Experts":
        t = lambda a: torch.from_numpy(a).to(device)  # noqa: E731
        return Experts(t(x.gate_up_q), t(x.gate_up_s), t(x.gate_up_g), t(x.down_q), t(x.down_s),
                       t(x.down_g))

    def nbytes_per_expert(self) -> int:
        return sum(a[0].numel() * a.element_size() for a in
                   (self.gate_up_q, self.gate_up_s, self.down_q, self.down_s)) + 8


# ------------------------------------------------------------------ quantise
def quantize(w: torch.Tensor, stream=None):
    """bf16 [E, N, K] -> (q uint8 [E, N, K/2], s uint8 [E, N, K/16], g f32 [E])."""
    if w.dtype != torch.bfloat16 or w.dim() != 3:
        raise ValueError("w must be a bf16 tensor [E, N, K]")
    Ee, N, K = w.shape
    dev = w.device
    q = torch.empty((Ee, N, K // 2), dtype=torch.uint8, device=dev)
    s = torch.empty((Ee, N, K // 16), dtype=torch.uint8, device=dev)
    g = torch.empty((Ee,), dtype=torch.float32, device=dev)
    nbytes = capi.nvfp4_quantize_workspace_bytes(Ee, N, K)
    ws = _workspace(nbytes, dev)
    check(capi.nvfp4_quantize(_ptr(w), Ee, N, K, _ptr(q), _ptr(s), _ptr(g), _ptr(ws), ws.numel(),
                              _stream(stream)), "nvfp4_quantize")
    return q, s, g


def dequantize(q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, stream=None) -> torch.Tensor:
    Ee, N, K2 = q.shape
    out = torch.empty((Ee, N, K2 * 2), dtype=torch.float32, device=q.device)
    check(capi.nvfp4_dequantize(_ptr(q), _ptr(s), _ptr(g), Ee, N, K2 * 2, _ptr(out), _stream(stream)),
          "nvfp4_dequantize")
    return out


# --------------------------------------------------------------------- route
def route(x: torch.Tensor, router: Router, stream=None):
    """bf16 [T, H] -> (ids int32 [T, 8], weights f32 [T, 8])."""
    T = x.shape[0]
    rs = router.c_struct()
    ids = torch.empty((T, router.top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, router.top_k), dtype=torch.float32, device=x.device)
    nbytes = capi.moe_route_workspace_bytes(T, ctypes.byref(rs))
    ws = _workspace(nbytes, x.device)
    check(capi.moe_route(_ptr(x), T, ctypes.byref(rs), _ptr(ids), _ptr(w), _ptr(ws), ws.numel(),
                         _stream(stream)), "moe_route")
    return ids, w


def permute(ids: torch.Tensor, stream=None):
    """int32 [T, 8] expert ids -> (counts int32 [E], offsets int32 [E+1],
    sorted_slot int32 [T*8], slot_pos int32 [T*8])."""
    if ids.dtype != torch.int32 or ids.dim() != 2 or ids.shape[1] != TOP_K:
        raise ValueError("ids must be an int32 tensor [T, 8]")
    T = ids.shape[0]
    dev = ids.device
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    sorted_slot = torch.empty((T * TOP_K,), dtype=torch.int32, device=dev)
    slot_pos = torch.empty((T * TOP_K,), dtype=torch.int32, device=dev)
    ws = _workspace(capi.moe_permute_workspace_bytes(T), dev)
    check(capi.moe_permute(_ptr(ids), T, _ptr(counts), _ptr(offsets), _ptr(sorted_slot), _ptr(slot_pos),
                           _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return counts, offsets, sorted_slot, slot_pos


# ------------------------------------------------------------------- forward
class MoeLayer:
    """One NVFP4 MoE branch: holds the device parameters and a workspace sized
    for up to `max_tokens` tokens.  Calls of one layer must not overlap on the
    GPU (they share the workspace)."""

    def __init__(self, experts: Experts, router: Router, max_tokens: int):
        self.experts, self.router = experts, router
        self._xs, self._rs = experts.c_struct(), router.c_struct()
        self.max_tokens = int(max_tokens)
        nbytes = capi.moe_forward_workspace_bytes(self.max_tokens, ctypes.byref(self._xs),
                                                  ctypes.byref(self._rs))
        if nbytes == 0:
            raise ValueError("unsupported experts/router configuration")
        self.workspace = _workspace(nbytes, experts.gate_up_q.device)

    def workspace_bytes(self, T: int) -> int:
        return capi.moe_forward_workspace_bytes(T, ctypes.byref(self._xs), ctypes.byref(self._rs))

    def forward_into(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        check(capi.moe_nvfp4_forward(_ptr(x), T, ctypes.byref(self._xs), ctypes.byref(self._rs),
                                     _ptr(y), _ptr(self.workspace), self.workspace.numel(),
                                     _stream(stream)), "moe_nvfp4_forward")
        return y

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        y = torch.empty_like(x)
        return self.forward_into(x, y, stream)

    def forward_dense_into(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
        """The dense over-read (every token through all 128 experts, weighted
        by its routing weights): the same y, for measuring the gather's
        advantage.  Uses its own workspace, sized on first use."""
        T = x.shape[0]
        nbytes = capi.moe_forward_dense_workspace_bytes(T, ctypes.byref(self._xs), ctypes.byref(self._rs))
        if nbytes == 0:
            raise ValueError(f"T={T} is outside the dense variant's range")
        if getattr(self, "_dense_ws", None) is None or self._dense_ws.numel() < nbytes:
            self._dense_ws = _workspace(nbytes, x.device)
        check(capi.moe_nvfp4_forward_dense(_ptr(x), T, ctypes.byref(self._xs), ctypes.byref(self._rs),
                                           _ptr(y), _ptr(self._dense_ws), self._dense_ws.numel(),
                                           _stream(stream)), "moe_nvfp4_forward_dense")
        return y

    def views(self, T: int) -> dict:
        """Intermediate results of the last forward of T tokens, as torch views
        of the workspace (see moe_forward_views in the header)."""
        return forward_views(self, T)


@dataclasses.dataclass
class Aff4Experts:
    """Expert stacks in the aff4 codec on the device: u8 codes, fp16 scales
    and biases per (row, K-block of 32) (layouts of moe_experts_aff4)."""
    gate_up_q: torch.Tensor
    gate_up_s: torch.Tensor
    gate_up_b: torch.Tensor
    down_q: torch.Tensor
    down_s: torch.Tensor
    down_b: torch.Tensor

    def c_struct(self) -> capi.moe_experts_aff4:
        return capi.moe_experts_aff4(_ptr(self.gate_up_q), _ptr(self.gate_up_s), _ptr(self.gate_up_b),
                                     _ptr(self.down_q), _ptr(self.down_s), _ptr(self.down_b),
                                     self.gate_up_q.shape[0], self.gate_up_q.shape[2] * 2,
                                     self.down_q.shape[2] * 2)

    @staticmethod
    def from_host(arrays, device="cuda") -> "Aff4Experts":
        """From host arrays (gate_up_q, gate_up_s, gate_up_b, down_q, down_s,
        down_b): u8 codes and fp16 bit patterns (uint16)."""
        def t(a):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).view(torch.float16).to(device)
            return torch.from_numpy(a).to(device)
        return Aff4Experts(*(t(a) for a in arrays))


class Aff4Layer:
    """One sparse MoE branch with aff4 experts and a workspace for up to
    `max_tokens` tokens (moe_aff4_forward)."""

    def __init__(self, experts: Aff4Experts, router: Router, max_tokens: int):
        self.experts, self.router = experts, router
        self._xs, self._rs = experts.c_struct(), router.c_struct()
        self.max_tokens = int(max_tokens)
        nbytes = capi.moe_aff4_forward_workspace_bytes(self.max_tokens, ctypes.byref(self._xs),
                                                       ctypes.byref(self._rs))
        if nbytes == 0:
            raise ValueError("unsupported experts/router configuration")
        self.workspace = _workspace(nbytes, experts.gate_up_q.device)

    def forward_into(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        check(capi.moe_aff4_forward(_ptr(x), T, ctypes.byref(self._xs), ctypes.byref(self._rs), _ptr(y),
                                    _ptr(self.workspace), self.workspace.numel(), _stream(stream)),
              "moe_aff4_forward")
        return y

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        return self.forward_into(x, torch.empty_like(x), stream)

    def ids(self, T: int) -> torch.Tensor:
        """The routed ids of the last forward of T tokens.  The workspace
        layout is the NVFP4 forward's (it depends on T only), so the view
        offsets come from moe_forward_workspace_views with the same pointers
        standing in for an NVFP4 stack."""
        e = self._xs
        stand_in = capi.moe_experts(e.gate_up_q, e.gate_up_s, e.gate_up_s, e.down_q, e.down_s, e.down_s,
                                    e.E, e.H, e.I)
        v = capi.moe_forward_views()
        check(capi.moe_forward_workspace_views(T, ctypes.byref(stand_in), ctypes.byref(self._rs), ctypes.byref(v)),
              "moe_forward_workspace_views")
        return self.workspace[v.ids:v.ids + T * TOP_K * 4].view(torch.int32).view(T, TOP_K)


class W4A4Layer:
    """One sparse MoE branch in the W4A4 form (moe_w4a4_forward): NVFP4
    experts, their block scales packed once into the tensor core's order, the
    static input globals gx (experts' input) and gh (hidden), and a workspace
    for up to `max_tokens` tokens."""

    def __init__(self, experts: Experts, router: Router, gx: float, gh: float, max_tokens: int, stream=None):
        experts = experts.packed(stream)
        self.experts, self.router = experts, router
        dev = experts.gate_up_q.device
        ex = experts.c_struct()
        E_ = experts.gate_up_q.shape[0]
        self.gate_up_sf, self.down_sf = (torch.empty(capi.moe_pack_bytes(E_, w), dtype=torch.uint8, device=dev)
                                         for w in (2, 3))
        check(capi.moe_w4a4_pack_scales(ctypes.byref(ex), _ptr(self.gate_up_sf), _ptr(self.down_sf), _stream(stream)),
              "moe_w4a4_pack_scales")
        self._xs = capi.moe_experts_w4a4(ex, _ptr(self.gate_up_sf), _ptr(self.down_sf), float(gx), float(gh))
        self._rs = router.c_struct()
        self.max_tokens = int(max_tokens)
        nbytes = capi.moe_w4a4_workspace_bytes(self.max_tokens, ctypes.byref(self._xs), ctypes.byref(self._rs))
        if nbytes == 0:
            raise ValueError("unsupported experts/router configuration")
        self.workspace = _workspace(nbytes, dev)

    def forward_into(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        check(capi.moe_w4a4_forward(_ptr(x), T, ctypes.byref(self._xs), ctypes.byref(self._rs), _ptr(y),
                                    _ptr(self.workspace), self.workspace.numel(), _stream(stream)),
              "moe_w4a4_forward")
        return y

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        return self.forward_into(x, torch.empty_like(x), stream)

    def views(self, T: int) -> dict:
        """What the last forward of T tokens left in the workspace, as device
        tensors (layouts of moe_w4a4_workspace_views)."""
        v = capi.moe_w4a4_views()
        check(capi.moe_w4a4_workspace_views(T, ctypes.byref(self._xs), ctypes.byref(self._rs), ctypes.byref(v)),
              "moe_w4a4_workspace_views")
        ws, S = self.workspace, T * TOP_K
        nt, mt = v.tile_tokens, v.max_tiles

        def i32(off, n):
            return ws[off:off + 4 * n].view(torch.int32)
        return {
            "ids": i32(v.ids, S).view(T, TOP_K),
            "weights": ws[v.weights:v.weights + 4 * S].view(torch.float32).view(T, TOP_K),
            "counts": i32(v.counts, E), "offsets": i32(v.offsets, E + 1),
            "sorted_slot": i32(v.sorted_slot, S), "slot_pos": i32(v.slot_pos, S),
            "x_codes": ws[v.x_codes:v.x_codes + mt * 11 * nt * 128],
            "x_scales": ws[v.x_scales:v.x_scales + mt * (H // 64) * 512],
            "h_codes": ws[v.h_codes:v.h_codes + mt * 3 * nt * 128],
            "h_scales": ws[v.h_scales:v.h_scales + mt * (I // 64) * 512],
            "tile_tokens": nt, "max_tiles": mt,
        }


@dataclasses.dataclass
class DenseParts:
    """The full block's bf16 tensors besides the experts and the router: the
    dense GELU-gated MLP, the five norm weights and the layer scalar."""
    dense_gate: torch.Tensor       # [2112, H]
    dense_up: torch.Tensor         # [2112, H]
    dense_down: torch.Tensor       # [H, 2112]
    pre_ff_norm: torch.Tensor      # [H]
    post_ff_norm_1: torch.Tensor   # [H]
    pre_ff_norm_2: torch.Tensor    # [H]
    post_ff_norm_2: torch.Tensor   # [H]
    post_ff_norm: torch.Tensor     # [H]
    layer_scalar: torch.Tensor     # [1]

    @staticmethod
    def from_host(b, device="cuda") -> "DenseParts":
        """From host bf16 bit patterns (numpy uint16 arrays)."""
        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view("int16")).view(torch.bfloat16).to(device)
        return DenseParts(*(bf(getattr(b, f.name)) for f in dataclasses.fields(DenseParts)))


class MoeBlock:
    """The full feed-forward block of a Gemma-4-26B-A4B layer (dense MLP in
    parallel with the NVFP4 sparse branch, norms, residual, layer scalar) with
    a workspace for up to `max_tokens` tokens."""

    def __init__(self, experts: Experts, router: Router, parts: DenseParts, max_tokens: int, eps: float = 1e-6):
        self.experts, self.router, self.parts = experts, router, parts
        self._c = capi.moe_block(experts.c_struct(), router.c_struct(), _ptr(parts.dense_gate),
                                 _ptr(parts.dense_up), _ptr(parts.dense_down), _ptr(parts.pre_ff_norm),
                                 _ptr(parts.post_ff_norm_1), _ptr(parts.pre_ff_norm_2),
                                 _ptr(parts.post_ff_norm_2), _ptr(parts.post_ff_norm), _ptr(parts.layer_scalar),
                                 parts.dense_gate.shape[0], eps)
        self.max_tokens = int(max_tokens)
        nbytes = capi.moe_block_workspace_bytes(self.max_tokens, ctypes.byref(self._c))
        if nbytes == 0:
            raise ValueError("unsupported block configuration")
        self.workspace = _workspace(nbytes, experts.gate_up_q.device)

    def forward_into(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        check(capi.moe_block_forward(_ptr(x), T, ctypes.byref(self._c), _ptr(y), _ptr(self.workspace),
                                     self.workspace.numel(), _stream(stream)), "moe_block_forward")
        return y

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        return self.forward_into(x, torch.empty_like(x), stream)

    def ids(self, T: int) -> torch.Tensor:
        """The routed ids of the last forward of T tokens."""
        v = capi.moe_forward_views()
        check(capi.moe_forward_workspace_views(T, ctypes.byref(self._c.experts), ctypes.byref(self._c.router),
                                               ctypes.byref(v)), "moe_forward_workspace_views")
        return self.workspace[v.ids:v.ids + T * TOP_K * 4].view(torch.int32).view(T, TOP_K)


def forward_views(layer: MoeLayer, T: int) -> dict:
    v = capi.moe_forward_views()
    check(capi.moe_forward_workspace_views(T, ctypes.byref(layer._xs), ctypes.byref(layer._rs),
                                           ctypes.byref(v)), "moe_forward_workspace_views")
    ws = layer.workspace
    S = T * TOP_K

    def view(off, n, dtype):
        item = torch.empty((), dtype=dtype).element_size()
        return ws[off:off + n * item].view(dtype)

    return {
        "ids": view(v.ids, S, torch.int32).view(T, TOP_K),
        "weights": view(v.weights, S, torch.float32).view(T, TOP_K),
        "counts": view(v.counts, E, torch.int32),
        "offsets": view(v.offsets, E + 1, torch.int32),
        "sorted_slot": view(v.sorted_slot, S, torch.int32),
        "slot_pos": view(v.slot_pos, S, torch.int32),
        "xexp": view(v.xexp, S, torch.int32),
        "h": view(v.h, S * I, torch.float16).view(S, I),
    }


def unscaled_hidden(views: dict) -> torch.Tensor:
    """The gated hidden h of forward_views in fp32 and at its true scale: row
    p of the stored h carries the factor 2^(-2 e), e = xexp[p] clamped to
    [-63, 63]."""
    e = views["xexp"].clamp(-63, 63).to(torch.float64)
    return (views["h"].to(torch.float64) * torch.pow(2.0, 2.0 * e)[:, None])


def residual_rmsnorm(res: torch.Tensor, y: torch.Tensor | None, x_out: torch.Tensor, eps: float = 1e-6,
                     stream=None) -> None:
    T, Hh = res.shape
    check(capi.moe_residual_rmsnorm(_ptr(res), _ptr(y), _ptr(x_out), T, Hh, eps, _stream(stream)),
          "moe_residual_rmsnorm")


def device_status(stream=None) -> int:
    return capi.nvfp4_get_device_status(_stream(stream))
