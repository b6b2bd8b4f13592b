"""Python binding of libnvfp4moe.so, the NVFP4 weight-only MoE library for
B200 (sm_100a).

Two layers:
  * the C ABI under its own names (`nvfp4_quantize`, `moe_route`,
    `moe_nvfp4_forward`, ... in `nvfp4_weight_only_router_b200.capi`): raw
    device pointers and sizes, returning the status code;
  * torch conveniences (`quantize`, `dequantize`, `route`, `permute`,
    `MoeLayer`, `residual_rmsnorm`): they allocate outputs and workspaces with torch and
    pass pointers to the same C calls on torch's current stream.

Every computation runs in the library's CUDA kernels; there is no fallback.
The shared library is loaded on first use of anything but `build`; that use
raises ImportError if it has not been built
(`python -m nvfp4_weight_only_router_b200.build`).
"""
from __future__ import annotations

import importlib

_API = {"MoeLayer", "MoeBlock", "DenseParts", "Aff4Experts", "Aff4Layer", "W4A4Layer", "Router", "Experts", "quantize", "dequantize", "route", "permute", "residual_rmsnorm",
        "device_status", "forward_views", "unscaled_hidden"}
_CAPI = {"NVFP4Error", "check", "status_string"}

__all__ = sorted(_API | _CAPI | {"capi", "build"})


def __getattr__(name):
    if name == "capi":
        return importlib.import_module(".capi", __name__)
    if name in _CAPI:
        return getattr(importlib.import_module(".capi", __name__), name)
    if name in _API:
        return getattr(importlib.import_module(".api", __name__), name)
    raise AttributeError(name)
