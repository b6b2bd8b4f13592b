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


def test_full_size_sampled_and_roundtrip(dev):
    """[128, 1408, 2816] bf16 (the expert gate_up stack shape), built from 8
    independently drawn experts repeated 16 times; experts from each copy
    group are compared with the oracle, and the fp32 dequantisation of them
    round-trips bit-exactly."""
    base = gen.make_quant_weights(4, 8, 1408, 2816)
    bits = np.tile(base, (16, 1, 1))
    wd = bf16_to_dev(bits, dev)
    q, s, g = lib.quantize(wd)
    deq = lib.dequantize(q, s, g)
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    for e in (0, 5, 63, 127):
        want = Q.quantize_tensor(bits[e])
        got = (q[e].cpu().numpy(), s[e].cpu().numpy(), g[e:e + 1].cpu().numpy())
        _assert_equal_quant(got, (want[0], want[1], np.array([want[2]])))
        d0 = Q.dequantize_f32(want[0], want[1], want[2])
        assert np.array_equal(deq[e].cpu().numpy().view(np.uint32), d0.view(np.uint32))
    # identical copies quantise identically
    assert torch.equal(q[0], q[8]) and torch.equal(s[3], s[3 + 64])
