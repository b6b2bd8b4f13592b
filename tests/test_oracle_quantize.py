"""Pins of the oracle's NVFP4 quantiser and dequantiser: a hand-derived worked
example, exact round trips on representable tensors, the rounding error bound
on general inputs, library routines for the scale step, degenerate cases."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import quantize as Q
from moe_inputs import bf16_bits
from tests.conftest import golden_lines


def _worked_example():
    rows = golden_lines("nvfp4_worked_example.txt")
    G = None
    scales, ws, codes = [], [], []
    for r in rows:
        if r[0] == "G":
            G = float.fromhex(r[1])
        elif r[0] == "block":
            scales.append(int(r[2], 16))
        else:
            ws.append(float.fromhex(r[0]))
            codes.append(int(r[2], 16))
    return G, np.array(scales, np.uint8), np.array(ws), np.array(codes, np.uint8)


def test_worked_example():
    G, scales, w, codes = _worked_example()
    bits = bf16_bits(w.astype(np.float32))[None, :]
    assert np.array_equal(F.bf16_to_f64(bits)[0], w), "fixture values are bf16-exact"
    assert np.array_equal(np.signbit(F.bf16_to_f64(bits)[0]), np.signbit(w))
    q, s, g = Q.quantize_tensor(bits)
    assert float(g) == G
    assert s[0].tolist() == scales.tolist()
    assert F.unpack_nibbles(q)[0].tolist() == codes.tolist()


def test_worked_example_dequant_closed_form():
    """Dequantised value = E2M1 value of the code x the hand-derived step d of
    its block (E2M1 values from the grid fixture)."""
    G, scales, w, codes = _worked_example()
    grid = {int(c, 16): float(v) for c, v in golden_lines("e2m1_grid.txt")}
    d = {0: 0.875, 1: 0.21875, 2: 0.21875, 3: 0.0, 4: 3 * 2.0 ** -18}
    what = Q.dequantize(F.pack_nibbles(codes[None, :]), scales[None, :], G)[0]
    want = np.array([grid[int(c)] * d[i // 16] for i, c in enumerate(codes)])
    assert np.array_equal(what, want)


def _representable_tensor(rng, n, k, gexp):
    """codes, scales and a power-of-two G such that every block holds a +-6
    code and one block has scale 448: the dequantised tensor is then an exact
    fixed point of the quantiser."""
    codes = rng.integers(0, 16, size=(n, k), dtype=np.uint8)
    nb = k // 16
    pos6 = rng.integers(0, 16, size=(n, nb))
    for i in range(n):
        for b in range(nb):
            codes[i, 16 * b + pos6[i, b]] = rng.choice([0x7, 0xF])
    # scales: any positive normal/subnormal E4M3 value, one block forced to 448
    s = rng.integers(0x01, 0x7F, size=(n, nb), dtype=np.uint8)
    s[rng.integers(n), rng.integers(nb)] = 0x7E
    G = 2.0 ** gexp
    w = Q.dequantize(F.pack_nibbles(codes), s, G)
    return codes, s, G, w


@pytest.mark.parametrize("gexp", [-9, -14, 0, 3])
def test_round_trip_exact_on_representable(gexp):
    rng = np.random.default_rng(100 + gexp)
    codes, s, G, w = _representable_tensor(rng, 24, 256, gexp)
    bits = bf16_bits(w.astype(np.float32))
    assert np.array_equal(F.bf16_to_f64(bits), w)  # exactly representable in bf16
    q, s2, g2 = Q.quantize_tensor(bits)
    assert float(g2) == G
    assert np.array_equal(s2, s)
    assert np.array_equal(F.unpack_nibbles(q), codes)


def test_scale_step_matches_torch_float8_and_global_matches_torch_division():
    w = F.bf16_to_f32(bf16_bits(np.random.default_rng(3).standard_normal((64, 512)).astype(np.float32) * 0.02))
    bits = bf16_bits(w)
    q, s, g = Q.quantize_tensor(bits)
    amax = torch.from_numpy(w).abs().max()
    g_ref = (amax / torch.tensor(2688.0, dtype=torch.float32)).item()
    assert np.float32(g) == np.float32(g_ref)
    amax_b = torch.from_numpy(w).abs().reshape(64, 32, 16).amax(-1)
    t = (amax_b / 6.0) / torch.tensor(g_ref, dtype=torch.float32)
    s_ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, s_ref)


def _grid_gap(mag):
    """Spacing of the E2M1 grid around a magnitude in [0, 6]."""
    return np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0))


def test_error_bound_general_inputs():
    rng = np.random.default_rng(4)
    w = rng.standard_normal((128, 1024)).astype(np.float32) * np.float32(0.02)
    mask = rng.random((128, 1024)) < 0.005
    w[mask] *= 20
    bits = bf16_bits(w)
    w64 = F.bf16_to_f64(bits)
    q, s, g = Q.quantize_tensor(bits)
    what = Q.dequantize(q, s, g)
    d = np.repeat(F.e4m3_decode(s) * float(g), 16, axis=1)   # exact real step size
    x = np.abs(w64) / d
    bound = d * np.where(x <= 6, _grid_gap(np.minimum(x, 6)) / 2, x - 6) + d * 6 * 2.0 ** -22
    assert np.all(np.abs(w64 - what) <= bound)
    # the quantiser is much better than the bound on average
    rel = np.linalg.norm(w64 - what) / np.linalg.norm(w64)
    assert rel < 0.2


def test_codes_are_nearest_of_all_16():
    """Brute force on small blocks: every code is the nearest of the 16 E2M1
    values to w/d (with d from the stored scale), ties to even."""
    rng = np.random.default_rng(5)
    w = rng.standard_normal((8, 64)).astype(np.float32)
    bits = bf16_bits(w)
    q, s, g = Q.quantize_tensor(bits)
    codes = F.unpack_nibbles(q)
    vals = F.e2m1_decode(np.arange(16))
    w32 = F.bf16_to_f32(bits)
    dd = np.repeat((F.e4m3_decode(s).astype(np.float32) * np.float32(g)).astype(np.float32), 16, axis=1)
    x = (w32 / dd).astype(np.float64)
    for i in range(8):
        for j in range(64):
            dist = np.abs(np.abs(x[i, j]) - np.abs(vals))
            same_sign = np.signbit(vals) == np.signbit(w32[i, j])
            dist[~same_sign] = np.inf
            best = np.flatnonzero(dist == dist.min())
            pick = [c for c in best if c % 2 == 0] or list(best)
            assert codes[i, j] == pick[0]


def test_all_zero_tensor_is_degenerate():
    bits = np.zeros((4, 32), np.uint16)
    bits[1, 3] = 0x8000  # -0.0
    q, s, g = Q.quantize_tensor(bits)
    assert float(g) == 0.0 and not s.any()
    codes = F.unpack_nibbles(q)
    assert codes[1, 3] == 0x8 and codes.sum() == 0x8


def test_zero_block_in_nonzero_tensor():
    w = np.zeros((1, 32), np.float32)
    w[0, 20] = 1.0
    q, s, g = Q.quantize_tensor(bf16_bits(w))
    assert s[0, 0] == 0 and s[0, 1] == 0x7E
    assert F.unpack_nibbles(q)[0, :16].sum() == 0


def test_stacked_quantize_uses_one_global_per_expert():
    rng = np.random.default_rng(6)
    w = rng.standard_normal((3, 16, 64)).astype(np.float32)
    w[1] *= 100
    bits = bf16_bits(w)
    q, s, g = Q.quantize(bits)
    for e in range(3):
        q1, s1, g1 = Q.quantize_tensor(bits[e])
        assert np.array_equal(q[e], q1) and np.array_equal(s[e], s1) and g[e] == g1
    assert g[1] > 50 * g[0]


def test_dequantize_closed_form_small():
    # one block, codes 0..15 with scale 1.5 (0x3C) and G = 0.25
    codes = np.arange(16, dtype=np.uint8)[None, :]
    w = Q.dequantize(F.pack_nibbles(codes), np.array([[0x3C]], np.uint8), 0.25)
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    want = np.array(grid + [-v for v in grid]) * 1.5 * 0.25
    assert np.array_equal(w[0], want)
