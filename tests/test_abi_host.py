"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects invalid arguments with the documented status
codes before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def capi():
    from nvfp4_weight_only_router_b200 import build
    build.build()
    from nvfp4_weight_only_router_b200 import capi
    return capi


def header_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4moe.h")).read()
    return re.findall(r"NVFP4MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_every_declared_symbol_is_exported(capi):
    names = header_functions()
    assert len(names) == 31
    for n in names:
        assert hasattr(capi.lib, n), n
        assert n in capi.SIGNATURES, n


def test_only_declared_symbols_are_exported(capi):
    out = os.popen(f"nm -D --defined-only {capi.LIB_PATH}").read().split("\n")
    exported = {l.split()[-1] for l in out if " T " in l}
    assert exported == set(header_functions())


def test_abi_version_and_status_strings(capi):
    assert capi.nvfp4_abi_version() == 3
    for code in range(9):
        assert capi.status_string(code)
    assert capi.status_string(0) == "ok"


def _router(capi, E=128, H=2816, k=8, eps=1e-6, ptr=4096):
    return capi.moe_router(ptr, ptr, ptr, None, E, H, k, eps)


def _experts(capi, E=128, H=2816, I=704, ptr=4096):
    return capi.moe_experts(ptr, ptr, ptr, ptr, ptr, ptr, E, H, I)


def test_quantize_validation(capi):
    c = capi
    assert c.nvfp4_quantize_workspace_bytes(128, 1408, 2816) == 768
    assert c.nvfp4_quantize_workspace_bytes(0, 1, 32) == 0
    P = 4096
    assert c.nvfp4_quantize(None, 1, 16, 32, P, P, P, P, 256, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.nvfp4_quantize(P, 1, 16, 24, P, P, P, P, 256, None) == c.NVFP4_ERR_UNSUPPORTED
    assert c.nvfp4_quantize(P, 0, 16, 32, P, P, P, P, 256, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.nvfp4_quantize(P + 8, 1, 16, 32, P, P, P, P, 256, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.nvfp4_quantize(P, 1, 16, 32, P, P, P, None, 256, None) == c.NVFP4_ERR_WORKSPACE
    assert c.nvfp4_quantize(P, 1, 16, 32, P, P, P, P, 0, None) == c.NVFP4_ERR_WORKSPACE
    assert c.nvfp4_quantize(P, 1, 16, 32, P, P, P, P + 16, 4096, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.nvfp4_quantize(P, 1, 1 << 20, 4096, P, P, P, P, 4096, None) == c.NVFP4_ERR_UNSUPPORTED
    # E amax words plus the single-pass kernel's three arrival counters
    assert c.nvfp4_quantize_workspace_bytes(1, 16, 32) == 256
    assert c.nvfp4_quantize_workspace_bytes(61, 16, 32) == 256
    assert c.nvfp4_quantize_workspace_bytes(62, 16, 32) == 512
    assert c.nvfp4_quantize(P, 128, 1408, 2816, P, P, P, P, 512, None) == c.NVFP4_ERR_WORKSPACE


def test_route_validation(capi):
    c = capi
    r = _router(c)
    assert c.moe_route_workspace_bytes(1, ctypes.byref(r)) > 0
    assert c.moe_route_workspace_bytes(0, ctypes.byref(r)) == 0
    assert c.moe_route_workspace_bytes(65537, ctypes.byref(r)) == 0
    P = 4096
    assert c.moe_route(P, 1, ctypes.byref(r), P, P, None, 0, None) == c.NVFP4_ERR_WORKSPACE
    assert c.moe_route(None, 1, ctypes.byref(r), P, P, P, 1 << 20, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_route(P, 0, ctypes.byref(r), P, P, P, 1 << 20, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_route(P, 1, None, P, P, P, 1 << 20, None) == c.NVFP4_ERR_INVALID_ARG
    for bad, code in [(_router(c, E=64), c.NVFP4_ERR_UNSUPPORTED), (_router(c, k=4), c.NVFP4_ERR_UNSUPPORTED),
                      (_router(c, H=100), c.NVFP4_ERR_UNSUPPORTED), (_router(c, H=1792), c.NVFP4_ERR_UNSUPPORTED),
                      (_router(c, H=4352), c.NVFP4_ERR_UNSUPPORTED), (_router(c, H=2880), c.NVFP4_ERR_UNSUPPORTED),
                      (_router(c, eps=-1.0), c.NVFP4_ERR_INVALID_ARG),
                      (_router(c, ptr=4097), c.NVFP4_ERR_ALIGNMENT)]:
        assert c.moe_route(P, 1, ctypes.byref(bad), P, P, P, 1 << 20, None) == code
    assert c.moe_route(P + 2, 1, ctypes.byref(r), P, P, P, 1 << 20, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.moe_route(P, 1, ctypes.byref(r), P, P, P + 16, 1 << 20, None) == c.NVFP4_ERR_ALIGNMENT


def test_forward_validation_and_workspace_sizes(capi):
    c = capi
    r, x = _router(c), _experts(c)
    sizes = [c.moe_forward_workspace_bytes(T, ctypes.byref(x), ctypes.byref(r)) for T in (1, 64, 4096)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    assert sizes[2] < 1 << 31
    assert c.moe_forward_workspace_bytes(1, ctypes.byref(_experts(c, I=512)), ctypes.byref(r)) == 0
    P = 4096
    ws = sizes[0]
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(x), ctypes.byref(r), P, P, ws - 1, None) == c.NVFP4_ERR_WORKSPACE
    assert c.moe_nvfp4_forward(None, 1, ctypes.byref(x), ctypes.byref(r), P, P, ws, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(x), ctypes.byref(r), None, P, ws, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(_experts(c, H=2048)), ctypes.byref(r), P, P, ws, None) == c.NVFP4_ERR_UNSUPPORTED
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(x), ctypes.byref(_router(c, H=2048)), P, P, ws, None) == c.NVFP4_ERR_UNSUPPORTED
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(_experts(c, ptr=4100)), ctypes.byref(r), P, P, ws, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(x), ctypes.byref(r), P, P + 128, ws, None) == c.NVFP4_ERR_ALIGNMENT
    v = c.moe_forward_views()
    assert c.moe_forward_workspace_views(64, ctypes.byref(x), ctypes.byref(r), ctypes.byref(v)) == 0
    offs = [v.ids, v.weights, v.counts, v.offsets, v.sorted_slot, v.slot_pos, v.xexp, v.h]
    assert all(o % 4 == 0 for o in offs) and max(offs) < sizes[1]


def test_residual_validation(capi):
    c = capi
    P = 4096
    assert c.moe_residual_rmsnorm(None, None, P, 1, 2816, 1e-6, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_residual_rmsnorm(P, None, P, 1, 2817, 1e-6, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_residual_rmsnorm(P + 4, None, P, 1, 2816, 1e-6, None) == c.NVFP4_ERR_ALIGNMENT


def test_last_cuda_error_is_a_string_before_any_failure(capi):
    # no call of this thread has failed yet: the runtime's text for success
    assert capi.lib.nvfp4_last_cuda_error().decode() == "no error"


def test_permute_validation(capi):
    c = capi
    assert c.moe_permute_workspace_bytes(0) == 0
    assert c.moe_permute_workspace_bytes(65537) == 0
    small, big = c.moe_permute_workspace_bytes(1), c.moe_permute_workspace_bytes(65536)
    assert 0 < small < big
    P = 4096
    assert c.moe_permute(None, 1, P, P, P, P, P, small, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_permute(P, 0, P, P, P, P, P, small, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_permute(P, 1, P, P + 4, P, P, P, small, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.moe_permute(P, 1, P, P, P, P, P, small - 1, None) == c.NVFP4_ERR_WORKSPACE
    assert c.moe_permute(P, 1, P, P, P, P, P + 16, small, None) == c.NVFP4_ERR_ALIGNMENT


def test_selftest_validation(capi):
    c = capi
    P = 4096
    ws = c.nvfp4_quantize_workspace_bytes(2, 1408, 2816)
    assert c.nvfp4_selftest_wait_timeout(P, 2, 1408, 2816, P, P, P, P, ws, 0, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.nvfp4_selftest_wait_timeout(P, 2, 1408, 2816, P, P, P, P, ws, 1000001, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.nvfp4_selftest_wait_timeout(P, 2, 1408, 2816, P, P, P, None, ws, 1000, None) == c.NVFP4_ERR_WORKSPACE
    assert c.nvfp4_selftest_wait_timeout(P + 2, 2, 1408, 2816, P, P, P, P, ws, 1000, None) == c.NVFP4_ERR_ALIGNMENT


def test_last_cuda_error_after_a_failed_call_without_a_device(capi):
    """With no CUDA device, a valid no-allocation quantise fails in its first
    runtime call (before any launch): the status is NVFP4_ERR_CUDA and
    nvfp4_last_cuda_error names the runtime's error, not "no error"."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a host without a CUDA device (the call would launch on fake pointers)")
    P = 4096
    assert capi.nvfp4_quantize_noalloc(P, 1, 16, 32, P, P, P, None) == capi.NVFP4_ERR_CUDA
    assert capi.lib.nvfp4_last_cuda_error().decode() != "no error"


def test_dense_variant_validation(capi):
    c = capi
    r, x = _router(c), _experts(c)
    assert c.moe_forward_dense_workspace_bytes(0, ctypes.byref(x), ctypes.byref(r)) == 0
    assert c.moe_forward_dense_workspace_bytes(257, ctypes.byref(x), ctypes.byref(r)) == 0
    small = c.moe_forward_dense_workspace_bytes(1, ctypes.byref(x), ctypes.byref(r))
    # 128 slots per token instead of 8: far more workspace than the routed forward
    assert small > 8 * c.moe_forward_workspace_bytes(1, ctypes.byref(x), ctypes.byref(r))
    P = 4096
    assert c.moe_nvfp4_forward_dense(P, 257, ctypes.byref(x), ctypes.byref(r), P, P, small, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_nvfp4_forward_dense(P, 1, ctypes.byref(x), ctypes.byref(r), P, P, small - 1, None) == c.NVFP4_ERR_WORKSPACE


def _block(c, dense_I=2112, ptr=4096, eps=1e-6):
    P = ptr
    return c.moe_block(_experts(c), _router(c), P, P, P, P, P, P, P, P, P, dense_I, eps)


def test_block_validation(capi):
    c = capi
    b = _block(c)
    sizes = [c.moe_block_workspace_bytes(T, ctypes.byref(b)) for T in (1, 64, 4096)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    assert c.moe_block_workspace_bytes(8193, ctypes.byref(b)) == 0
    assert c.moe_block_workspace_bytes(1, ctypes.byref(_block(c, dense_I=2048))) == 0
    P = 4096
    ws = sizes[0]
    assert c.moe_block_forward(P, 1, ctypes.byref(b), P, P, ws - 1, None) == c.NVFP4_ERR_WORKSPACE
    assert c.moe_block_forward(None, 1, ctypes.byref(b), P, P, ws, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_block_forward(P, 1, ctypes.byref(_block(c, dense_I=2048)), P, P, ws, None) == c.NVFP4_ERR_UNSUPPORTED
    assert c.moe_block_forward(P, 1, ctypes.byref(_block(c, eps=-1.0)), P, P, ws, None) == c.NVFP4_ERR_INVALID_ARG
    bad = _block(c)
    bad.post_ff_norm = 4096 + 8
    assert c.moe_block_forward(P, 1, ctypes.byref(bad), P, P, ws, None) == c.NVFP4_ERR_ALIGNMENT
    bad.post_ff_norm = None
    assert c.moe_block_forward(P, 1, ctypes.byref(bad), P, P, ws, None) == c.NVFP4_ERR_INVALID_ARG


def test_aff4_validation(capi):
    c = capi
    r = _router(c)
    a = c.moe_experts_aff4(4096, 4096, 4096, 4096, 4096, 4096, 128, 2816, 704)
    x = _experts(c)
    n = c.moe_aff4_forward_workspace_bytes(64, ctypes.byref(a), ctypes.byref(r))
    assert n == c.moe_forward_workspace_bytes(64, ctypes.byref(x), ctypes.byref(r))   # the same layout
    P = 4096
    bad = c.moe_experts_aff4(4096, 4096, None, 4096, 4096, 4096, 128, 2816, 704)
    assert c.moe_aff4_forward(P, 1, ctypes.byref(bad), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_INVALID_ARG
    bad = c.moe_experts_aff4(4096, 4096, 4096, 4096, 4096, 4096, 128, 2816, 512)
    assert c.moe_aff4_forward(P, 1, ctypes.byref(bad), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_UNSUPPORTED
    bad = c.moe_experts_aff4(4096, 4096 + 2, 4096, 4096, 4096, 4096, 128, 2816, 704)
    assert c.moe_aff4_forward(P, 1, ctypes.byref(bad), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.moe_aff4_forward(P, 1, ctypes.byref(a), ctypes.byref(r), P, P, 0, None) == c.NVFP4_ERR_WORKSPACE


def _w4a4(c, gx=0.003, gh=0.0007, sf=4096, pk=4096):
    x = _experts(c)
    x.gate_up_pk, x.down_pk = pk, pk
    return c.moe_experts_w4a4(x, sf, sf, gx, gh)


def test_packing_validation(capi):
    c = capi
    assert c.moe_pack_bytes(128, 0) == 128 * 11 * 11 * 128 * 128      # 128-row tiles x 256-element chunks
    assert c.moe_pack_bytes(128, 1) == 128 * 22 * 3 * 128 * 128
    assert c.moe_pack_bytes(128, 2) == 128 * 1408 * 176
    assert c.moe_pack_bytes(128, 3) == 128 * 2816 * 44
    assert c.moe_pack_bytes(0, 0) == 0 and c.moe_pack_bytes(128, 4) == 0
    P = 4096
    x = _experts(c, I=512)
    assert c.moe_nvfp4_pack_codes(ctypes.byref(x), P, P, None) == c.NVFP4_ERR_UNSUPPORTED
    assert c.moe_nvfp4_pack_codes(ctypes.byref(_experts(c)), None, P, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_nvfp4_pack_codes(ctypes.byref(_experts(c)), P, P + 4, None) == c.NVFP4_ERR_ALIGNMENT
    assert c.moe_w4a4_pack_scales(ctypes.byref(_experts(c)), P, None, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_w4a4_pack_scales(ctypes.byref(_experts(c)), P + 8, P, None) == c.NVFP4_ERR_ALIGNMENT
    # the packed codes of a forward: both or neither, aligned
    r = _router(c)
    one = _experts(c)
    one.gate_up_pk = P
    n = c.moe_forward_workspace_bytes(1, ctypes.byref(_experts(c)), ctypes.byref(r))
    assert c.moe_forward_workspace_bytes(1, ctypes.byref(one), ctypes.byref(r)) == 0
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(one), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_INVALID_ARG
    one.down_pk = P + 4
    assert c.moe_nvfp4_forward(P, 1, ctypes.byref(one), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_ALIGNMENT


def test_w4a4_validation(capi):
    c = capi
    r, w = _router(c), _w4a4(c)
    sizes = [c.moe_w4a4_workspace_bytes(T, ctypes.byref(w), ctypes.byref(r)) for T in (1, 64, 4096)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    assert c.moe_w4a4_workspace_bytes(65537, ctypes.byref(w), ctypes.byref(r)) == 0
    v = c.moe_w4a4_views()
    assert c.moe_w4a4_workspace_views(64, ctypes.byref(w), ctypes.byref(r), ctypes.byref(v)) == c.NVFP4_OK
    assert v.tile_tokens == 16 and v.max_tiles == 512 // 16 + 128
    assert c.moe_w4a4_workspace_views(4096, ctypes.byref(w), ctypes.byref(r), ctypes.byref(v)) == c.NVFP4_OK
    assert v.tile_tokens == 128 and v.max_tiles == 32768 // 128 + 128
    P, n = 4096, sizes[0]
    assert c.moe_w4a4_forward(P, 1, ctypes.byref(w), ctypes.byref(r), P, P, n - 1, None) == c.NVFP4_ERR_WORKSPACE
    assert c.moe_w4a4_forward(None, 1, ctypes.byref(w), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_INVALID_ARG
    for bad in (_w4a4(c, gx=0.0), _w4a4(c, gh=float("inf")), _w4a4(c, gx=float("nan")), _w4a4(c, sf=None),
                _w4a4(c, pk=None)):
        assert c.moe_w4a4_forward(P, 1, ctypes.byref(bad), ctypes.byref(r), P, P, n, None) == c.NVFP4_ERR_INVALID_ARG
    assert c.moe_w4a4_forward(P, 1, ctypes.byref(_w4a4(c, sf=4096 + 8)), ctypes.byref(r), P, P, n,
                              None) == c.NVFP4_ERR_ALIGNMENT
