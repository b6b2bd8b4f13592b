"""nvfp4_quantize_noalloc, the entry point for callers that cannot allocate
device memory when they quantise (a framework plugin that may not allocate in
its execute callback, a path that must not enter an allocator): its scratch is
a fixed array inside the library instead of a caller workspace.

The test calls it through the C ABI twice in a row, on two different inputs,
and checks each result against the ordinary nvfp4_quantize entry point,
bit-exactly (the quantiser's parity bar).  It is collected last so that a run
stopping at the first failure has run every other test first; it passes alone
in a fresh process as well."""
import numpy as np
import pytest
import torch

import moe_inputs as gen

pytestmark = pytest.mark.gpu


def _quantize_both(capi, w_bits, dev):
    E, N, K = w_bits.shape
    w = torch.from_numpy(np.ascontiguousarray(w_bits).view(np.int16)).view(torch.bfloat16).to(dev)
    outs = []
    for _ in range(2):
        outs.append((torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev),
                     torch.empty((E, N, K // 16), dtype=torch.uint8, device=dev),
                     torch.empty((E,), dtype=torch.float32, device=dev)))
    (q0, s0, g0), (q1, s1, g1) = outs
    stream = torch.cuda.current_stream().cuda_stream
    nbytes = capi.nvfp4_quantize_workspace_bytes(E, N, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    capi.check(capi.nvfp4_quantize(w.data_ptr(), E, N, K, q0.data_ptr(), s0.data_ptr(), g0.data_ptr(),
                                   ws.data_ptr(), nbytes, stream))
    capi.check(capi.nvfp4_quantize_noalloc(w.data_ptr(), E, N, K, q1.data_ptr(), s1.data_ptr(),
                                           g1.data_ptr(), stream))
    torch.cuda.synchronize()
    return (q0, s0, g0), (q1, s1, g1)


def test_noalloc_matches_workspace_entry_point_twice(dev):
    from nvfp4_weight_only_router_b200 import capi
    from oracle import quantize as Q
    # two calls in a row with different inputs (and a different tensor count,
    # so stale scratch from the first call would show up in the second); each
    # result also against the oracle directly
    for seed, shape in ((21, (6, 96, 512)), (22, (3, 1408, 2816))):
        bits = gen.make_quant_weights(seed, *shape)
        ref, got = _quantize_both(capi, bits, dev)
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        q0, s0, g0 = Q.quantize(bits)
        assert np.array_equal(got[0].cpu().numpy(), q0) and np.array_equal(got[1].cpu().numpy(), s0)
        assert np.array_equal(got[2].cpu().numpy().view(np.uint32), g0.view(np.uint32))
    assert capi.nvfp4_get_device_status(None) == 0


def test_noalloc_rejects_too_many_tensors(dev):
    from nvfp4_weight_only_router_b200 import capi
    P = 1 << 12
    assert capi.nvfp4_quantize_noalloc(P, 4097, 1, 32, P, P, P, None) == capi.NVFP4_ERR_UNSUPPORTED
