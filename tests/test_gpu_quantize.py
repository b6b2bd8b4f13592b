"""nvfp4_quantize / nvfp4_dequantize on the GPU against the oracle:
bit-exact codes, scales and global scales; bit-exact fp32 dequantisation."""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import quantize as Q
from tests.conftest import golden_lines
from tests.gpu_common import bf16_to_dev

pytestmark = pytest.mark.gpu


def _run(bits, dev):
    q, s, g = lib.quantize(bf16_to_dev(bits, dev))
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), g.cpu().numpy()


def _assert_equal_quant(got, want):
    q, s, g = got
    q0, s0, g0 = want
    assert np.array_equal(g.view(np.uint32), np.asarray(g0, np.float32).view(np.uint32))
    assert np.array_equal(s, s0), f"{np.count_nonzero(s != s0)} scale bytes differ"
    assert np.array_equal(q, q0), f"{np.count_nonzero(q != q0)} code bytes differ"


def test_worked_example_row(dev):
    rows = golden_lines("nvfp4_worked_example.txt")
    w = np.array([float.fromhex(r[0]) for r in rows if r[0] not in ("G", "block")], np.float32)
    bits = np.tile(gen.bf16_bits(w)[None, None, :], (2, 3, 1))   # E=2, N=3, K=80 -> pad K to 96
    bits = np.concatenate([bits, np.zeros((2, 3, 16), np.uint16)], axis=2)
    _assert_equal_quant(_run(bits, dev), Q.quantize(bits))


@pytest.mark.parametrize("shape", [(1, 1, 32), (3, 17, 64), (5, 64, 2816), (2, 300, 704)])
def test_random_shapes(dev, shape):
    bits = gen.make_quant_weights(11, *shape)
    _assert_equal_quant(_run(bits, dev), Q.quantize(bits))


def test_worked_example_rows_single_pass(dev):
    """The worked example's blocks (ties at every E2M1 threshold, saturation,
    zero and subnormal-scale blocks) repeated over enough rows that the
    single-pass kernel (pieces of every tensor split over all CTAs) runs."""
    rows = golden_lines("nvfp4_worked_example.txt")
    w = np.array([float.fromhex(r[0]) for r in rows if r[0] not in ("G", "block")], np.float32)
    row = np.concatenate([gen.bf16_bits(w), np.zeros(16, np.uint16)])
    bits = np.tile(row[None, None, :], (2, 600, 1))
    bits[1, 7] = 0x8000                      # one negative-zero row in the second tensor
    _assert_equal_quant(_run(bits, dev), Q.quantize(bits))


@pytest.mark.parametrize("N,K", [(8, 64), (16, 2816)])
def test_edge_values(dev, N, K):
    """Edge values through the two-pass kernels ([4, 8, 64]) and through the
    single-pass kernel ([4, 16, 2816])."""
    rng = np.random.default_rng(12)
    w = rng.standard_normal((4, N, K)).astype(np.float32)
    w[0] = 0.0                              # all-zero tensor -> G = 0
    w[1, 0, :16] = 0.0                      # zero block
    w[1, 1, :16] = -0.0                     # negative-zero block
    w[1, 2, 16:32] = 1e-30                  # tiny block (subnormal scale range)
    w[2] *= 1e4                             # large values
    w[3, :, ::7] *= 1000                    # outliers inside blocks
    bits = gen.bf16_bits(w)
    bits[1, 1, :16] = 0x8000
    _assert_equal_quant(_run(bits, dev), Q.quantize(bits))


def test_full_size_workload_all_tensors(dev):
    """The quantise workload itself: bf16 [128, 1408, 2816] ~ N(0, 0.02) with
    0.5% x20 outliers (expert j from its own seeded stream), every one of the
    128 tensors bit-exact against the oracle (run in a process pool), and the
    fp32 dequantisation of four of them round-tripping bit-exactly."""
    from tests.oracle_pool import pool, quant_expert_and_oracle
    E, N, K = 128, 1408, 2816
    with pool() as ex:
        res = list(ex.map(quant_expert_and_oracle, [(4, j, N, K) for j in range(E)]))
    w = np.stack([r[0] for r in res])
    q, s, g = _run(w, dev)
    assert lib.device_status() == 0
    for j, (_, q0, s0, g0) in enumerate(res):
        assert g[j].view(np.uint32) == np.float32(g0).view(np.uint32), j
        assert np.array_equal(s[j], s0), f"tensor {j}: {np.count_nonzero(s[j] != s0)} scale bytes differ"
        assert np.array_equal(q[j], q0), f"tensor {j}: {np.count_nonzero(q[j] != q0)} code bytes differ"
    qd, sd, gd = (torch.from_numpy(a).to(dev) for a in (q, s, g))
    deq = lib.dequantize(qd, sd, gd)
    torch.cuda.synchronize()
    for j in (0, 5, 63, 127):
        d0 = Q.dequantize_f32(res[j][1], res[j][2], res[j][3])
        assert np.array_equal(deq[j].cpu().numpy().view(np.uint32), d0.view(np.uint32))


def test_more_tensors_than_a_grid_dimension(dev):
    """65,600 tiny tensors [1, 32] (the two-pass kernels, whose amax pass puts
    tensors on the grid's y dimension, at most 65,535): the tensors past that
    limit are quantised too; bit-exact on every tensor of a sample that covers
    both sides of the limit."""
    E = 65600
    bits = gen.make_quant_weights(9, E, 1, 32)
    q, s, g = _run(bits, dev)
    assert lib.device_status() == 0
    sample = np.r_[0:64, 65500:65600, np.random.default_rng(1).choice(E, 200, replace=False)]
    for j in sample:
        q0, s0, g0 = Q.quantize_tensor(bits[j])
        assert g[j].view(np.uint32) == np.float32(g0).view(np.uint32), j
        assert np.array_equal(s[j], s0) and np.array_equal(q[j], q0), j


def test_timeout_selftest_then_gpu_still_answers(dev):
    """A bounded wait that cannot complete: the single-pass quantiser's
    cross-CTA arrival count raised past what the grid can reach, every wait
    limited to 20 ms.  The call returns, the device status reads
    NVFP4_ERR_TIMEOUT, and the GPU still answers: a quantise right after is
    bit-exact against the oracle."""
    import time
    from nvfp4_weight_only_router_b200 import capi
    bits = gen.make_quant_weights(13, 2, 1408, 2816)
    w = bf16_to_dev(bits, dev)
    q = torch.empty((2, 1408, 1408), dtype=torch.uint8, device=dev)
    s = torch.empty((2, 1408, 176), dtype=torch.uint8, device=dev)
    g = torch.empty((2,), dtype=torch.float32, device=dev)
    nbytes = capi.nvfp4_quantize_workspace_bytes(2, 1408, 2816)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    assert lib.device_status() == 0
    t0 = time.perf_counter()
    capi.check(capi.nvfp4_selftest_wait_timeout(w.data_ptr(), 2, 1408, 2816, q.data_ptr(), s.data_ptr(),
                                                g.data_ptr(), ws.data_ptr(), ws.numel(), 20000,
                                                torch.cuda.current_stream().cuda_stream))
    assert capi.nvfp4_get_device_status(None) == capi.NVFP4_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert capi.nvfp4_get_device_status(None) == capi.NVFP4_OK   # read and cleared
    _assert_equal_quant(_run(bits, dev), Q.quantize(bits))
    assert lib.device_status() == 0
