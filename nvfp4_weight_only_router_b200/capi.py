"""ctypes declarations of the C ABI in include/nvfp4moe.h (argument
marshalling only).  The functions keep the C names and signatures: pointers
are Python ints (device addresses), `stream` is a cudaStream_t as an int
(0 = legacy default stream), and each returns the nvfp4_status code."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m nvfp4_weight_only_router_b200.build` "
        "(the package has no fallback path)")
lib = ctypes.CDLL(LIB_PATH)

c_void_p, c_int32, c_int64, c_size_t, c_float = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                                   ctypes.c_size_t, ctypes.c_float)

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_ALIGNMENT", 3: "NVFP4_ERR_WORKSPACE",
    4: "NVFP4_ERR_CUDA", 5: "NVFP4_ERR_TIMEOUT", 6: "NVFP4_ERR_UNSUPPORTED", 7: "NVFP4_ERR_DEVICE",
    8: "NVFP4_ERR_RANGE",
}
NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_ALIGNMENT = 2
NVFP4_ERR_WORKSPACE = 3
NVFP4_ERR_CUDA = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_ERR_UNSUPPORTED = 6
NVFP4_ERR_DEVICE = 7
NVFP4_ERR_RANGE = 8


class moe_router(ctypes.Structure):
    _fields_ = [("proj", c_void_p), ("scale", c_void_p), ("per_expert_scale", c_void_p),
                ("logit_bias", c_void_p), ("E", c_int32), ("H", c_int32), ("top_k", c_int32),
                ("eps", c_float)]


class moe_experts(ctypes.Structure):
    _fields_ = [("gate_up_q", c_void_p), ("gate_up_s", c_void_p), ("gate_up_g", c_void_p),
                ("down_q", c_void_p), ("down_s", c_void_p), ("down_g", c_void_p),
                ("E", c_int32), ("H", c_int32), ("I", c_int32),
                ("gate_up_pk", c_void_p), ("down_pk", c_void_p)]


class moe_forward_views(ctypes.Structure):
    _fields_ = [("ids", c_size_t), ("weights", c_size_t), ("counts", c_size_t),
                ("offsets", c_size_t), ("sorted_slot", c_size_t), ("slot_pos", c_size_t),
                ("xexp", c_size_t), ("h", c_size_t)]


class moe_experts_aff4(ctypes.Structure):
    _fields_ = [("gate_up_q", c_void_p), ("gate_up_s", c_void_p), ("gate_up_b", c_void_p),
                ("down_q", c_void_p), ("down_s", c_void_p), ("down_b", c_void_p),
                ("E", c_int32), ("H", c_int32), ("I", c_int32)]


class moe_block(ctypes.Structure):
    _fields_ = [("experts", moe_experts), ("router", moe_router), ("dense_gate", c_void_p),
                ("dense_up", c_void_p), ("dense_down", c_void_p), ("pre_ff_norm", c_void_p),
                ("post_ff_norm_1", c_void_p), ("pre_ff_norm_2", c_void_p), ("post_ff_norm_2", c_void_p),
                ("post_ff_norm", c_void_p), ("layer_scalar", c_void_p), ("dense_I", c_int32), ("eps", c_float)]


class moe_experts_w4a4(ctypes.Structure):
    _fields_ = [("experts", moe_experts), ("gate_up_sf", c_void_p), ("down_sf", c_void_p),
                ("input_scale_gate_up", c_float), ("input_scale_down", c_float)]


class moe_w4a4_views(ctypes.Structure):
    _fields_ = [("ids", c_size_t), ("weights", c_size_t), ("counts", c_size_t), ("offsets", c_size_t),
                ("sorted_slot", c_size_t), ("slot_pos", c_size_t), ("x_codes", c_size_t),
                ("x_scales", c_size_t), ("h_codes", c_size_t), ("h_scales", c_size_t),
                ("tile_tokens", c_int32), ("max_tiles", c_int32)]


_R = ctypes.POINTER(moe_router)
_X = ctypes.POINTER(moe_experts)
_B = ctypes.POINTER(moe_block)
_A = ctypes.POINTER(moe_experts_aff4)
_W = ctypes.POINTER(moe_experts_w4a4)

# name -> (restype, argtypes), in the order of the header
SIGNATURES = {
    "nvfp4_quantize_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64]),
    "nvfp4_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_size_t, c_void_p]),
    "nvfp4_quantize_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p,
                                         c_void_p, c_void_p]),
    "nvfp4_dequantize": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64,
                                   c_void_p, c_void_p]),
    "moe_route_workspace_bytes": (c_size_t, [c_int32, _R]),
    "moe_route": (c_int32, [c_void_p, c_int32, _R, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward_workspace_bytes": (c_size_t, [c_int32, _X, _R]),
    "moe_nvfp4_forward": (c_int32, [c_void_p, c_int32, _X, _R, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_aff4_forward_workspace_bytes": (c_size_t, [c_int32, _A, _R]),
    "moe_aff4_forward": (c_int32, [c_void_p, c_int32, _A, _R, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward_dense_workspace_bytes": (c_size_t, [c_int32, _X, _R]),
    "moe_nvfp4_forward_dense": (c_int32, [c_void_p, c_int32, _X, _R, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_nvfp4_forward_profiled": (c_int32, [c_void_p, c_int32, _X, _R, c_void_p, c_void_p, c_size_t,
                                             c_void_p, ctypes.POINTER(c_void_p)]),
    "moe_forward_workspace_views": (c_int32, [c_int32, _X, _R, ctypes.POINTER(moe_forward_views)]),
    "moe_block_workspace_bytes": (c_size_t, [c_int32, _B]),
    "moe_block_forward": (c_int32, [c_void_p, c_int32, _B, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_pack_bytes": (c_size_t, [c_int32, c_int32]),
    "moe_nvfp4_pack_codes": (c_int32, [_X, c_void_p, c_void_p, c_void_p]),
    "moe_w4a4_pack_scales": (c_int32, [_X, c_void_p, c_void_p, c_void_p]),
    "moe_w4a4_workspace_bytes": (c_size_t, [c_int32, _W, _R]),
    "moe_w4a4_forward": (c_int32, [c_void_p, c_int32, _W, _R, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_w4a4_forward_profiled": (c_int32, [c_void_p, c_int32, _W, _R, c_void_p, c_void_p, c_size_t, c_void_p,
                                            ctypes.POINTER(c_void_p)]),
    "moe_w4a4_workspace_views": (c_int32, [c_int32, _W, _R, ctypes.POINTER(moe_w4a4_views)]),
    "moe_permute_workspace_bytes": (c_size_t, [c_int32]),
    "moe_permute": (c_int32, [c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                              c_void_p]),
    "moe_residual_rmsnorm": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_float, c_void_p]),
    "nvfp4_get_device_status": (c_int32, [c_void_p]),
    "nvfp4_selftest_wait_timeout": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_size_t, ctypes.c_uint32, c_void_p]),
    "nvfp4_status_string": (ctypes.c_char_p, [c_int32]),
    "nvfp4_abi_version": (ctypes.c_int, []),
    "nvfp4_last_cuda_error": (ctypes.c_char_p, []),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
    globals()[_name] = _fn


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = f"{what}: {STATUS.get(status, status)} ({status_string(status)})"
        if status == NVFP4_ERR_CUDA:
            msg += f": {lib.nvfp4_last_cuda_error().decode()}"
        super().__init__(msg)


def status_string(status: int) -> str:
    return lib.nvfp4_status_string(status).decode()


def check(status: int, what: str = "nvfp4moe") -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(status, what)
