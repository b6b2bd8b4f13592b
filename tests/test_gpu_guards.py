"""Out-of-bounds writes: every output buffer and the workspace of a call sit
between two 4 KB guard regions filled with a fixed byte pattern, which the
call must leave unchanged (the forwards on both expert paths and in the W4A4
form, the full block, the router and both quantiser paths)."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from nvfp4_weight_only_router_b200 import capi
from tests.gpu_common import bf16_to_dev

pytestmark = pytest.mark.gpu

G = 4096          # guard bytes on each side (keeps 256-byte alignment)
PATTERN = 0xA5


class Guarded:
    """A device buffer of n bytes at .ptr with guards before and after."""

    def __init__(self, n, dev):
        self.n = int(n)
        self.buf = torch.full((self.n + 2 * G,), PATTERN, dtype=torch.uint8, device=dev)
        self.ptr = self.buf.data_ptr() + G

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:G].cpu().numpy()
        tail = self.buf[G + self.n:].cpu().numpy()
        assert np.all(head == PATTERN), f"{what}: write before the buffer"
        assert np.all(tail == PATTERN), f"{what}: write past the buffer"


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("T", [5, 300])
def test_forward_writes_stay_in_bounds(layer0, dev, T):
    ex, rt = layer0["dex"].packed(), layer0["drt"]
    xs, rs = ex.c_struct(), rt.c_struct()
    x = bf16_to_dev(gen.make_x(70 + T, T), dev)
    y = Guarded(T * 2816 * 2, dev)
    n = capi.moe_forward_workspace_bytes(T, ctypes.byref(xs), ctypes.byref(rs))
    ws = Guarded(n, dev)
    capi.check(capi.moe_nvfp4_forward(x.data_ptr(), T, ctypes.byref(xs), ctypes.byref(rs), y.ptr, ws.ptr, n,
                                      _stream()))
    assert lib.device_status() == 0
    y.check("y")
    ws.check("workspace")


@pytest.mark.parametrize("T", [5, 300])
def test_w4a4_writes_stay_in_bounds(layer0, dev, T):
    layer = lib.W4A4Layer(layer0["dex"], layer0["drt"], gen.W4A4_GX, gen.W4A4_GH, max_tokens=T)
    x = bf16_to_dev(gen.make_x(80 + T, T), dev)
    y = Guarded(T * 2816 * 2, dev)
    n = capi.moe_w4a4_workspace_bytes(T, ctypes.byref(layer._xs), ctypes.byref(layer._rs))
    ws = Guarded(n, dev)
    capi.check(capi.moe_w4a4_forward(x.data_ptr(), T, ctypes.byref(layer._xs), ctypes.byref(layer._rs), y.ptr,
                                     ws.ptr, n, _stream()))
    assert lib.device_status() == 0
    y.check("y")
    ws.check("workspace")


def test_block_writes_stay_in_bounds(layer0, dev):
    T = 5
    parts = lib.DenseParts.from_host(gen.make_block(201), dev)
    block = lib.MoeBlock(layer0["dex"], layer0["drt"], parts, max_tokens=T)
    x = bf16_to_dev(gen.make_x(90, T), dev)
    y = Guarded(T * 2816 * 2, dev)
    n = capi.moe_block_workspace_bytes(T, ctypes.byref(block._c))
    ws = Guarded(n, dev)
    capi.check(capi.moe_block_forward(x.data_ptr(), T, ctypes.byref(block._c), y.ptr, ws.ptr, n, _stream()))
    assert lib.device_status() == 0
    y.check("y")
    ws.check("workspace")


@pytest.mark.parametrize("T", [5, 300])
def test_route_writes_stay_in_bounds(layer0, dev, T):
    rs = layer0["drt"].c_struct()
    x = bf16_to_dev(gen.make_x(100 + T, T), dev)
    ids, w = Guarded(T * 8 * 4, dev), Guarded(T * 8 * 4, dev)
    n = capi.moe_route_workspace_bytes(T, ctypes.byref(rs))
    ws = Guarded(n, dev)
    capi.check(capi.moe_route(x.data_ptr(), T, ctypes.byref(rs), ids.ptr, w.ptr, ws.ptr, n, _stream()))
    assert lib.device_status() == 0
    for b, what in ((ids, "ids"), (w, "weights"), (ws, "workspace")):
        b.check(what)


@pytest.mark.parametrize("K", [256, 2816])
def test_quantize_writes_stay_in_bounds(dev, K):
    E, N = 2, 64
    wq = gen.make_quant_weights(3, E, N, K)
    w = torch.from_numpy(wq.view(np.int16)).view(torch.bfloat16).to(dev)
    q, s, g = Guarded(E * N * K // 2, dev), Guarded(E * N * K // 16, dev), Guarded(E * 4, dev)
    n = capi.nvfp4_quantize_workspace_bytes(E, N, K)
    ws = Guarded(n, dev)
    capi.check(capi.nvfp4_quantize(w.data_ptr(), E, N, K, q.ptr, s.ptr, g.ptr, ws.ptr, n, _stream()))
    assert lib.device_status() == 0
    for b, what in ((q, "codes"), (s, "scales"), (g, "globals"), (ws, "workspace")):
        b.check(what)
