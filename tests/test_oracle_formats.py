"""Pins of the oracle's number formats against the format definitions, golden
tables and library routines (torch float8_e4m3fn, torch bf16 conversion)."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats as F
from tests.conftest import golden_lines


def test_e2m1_decode_matches_grid_table():
    rows = golden_lines("e2m1_grid.txt")
    codes = np.array([int(r[0], 16) for r in rows])
    want = np.array([float(r[1]) for r in rows])
    got = F.e2m1_decode(codes)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))  # -0.0 for code 0x8


def test_e2m1_ties_and_saturation_table():
    for x, code in golden_lines("e2m1_ties.txt"):
        got = int(F.e2m1_encode(np.float32(float(x))))
        assert got == int(code, 16), (x, hex(got), code)


def _brute_force_e2m1(x: float) -> int:
    """Nearest of all 16 codes by exhaustive search; among equally near codes
    of the right sign, the even one; the sign bit follows the sign of x."""
    vals = [Fraction(F.e2m1_decode(c).item()) for c in range(16)]
    neg = math.copysign(1.0, x) < 0
    cands = [c for c in range(16) if bool(c & 8) == neg]
    dist = [abs(abs(Fraction(x)) - abs(vals[c])) for c in cands]  # exact rationals
    best = min(dist)
    tied = [c for c, d in zip(cands, dist) if d == best]
    even = [c for c in tied if c % 2 == 0]
    return (even or tied)[0]


def test_e2m1_encode_brute_force_sweep():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.uniform(-8, 8, 3000).astype(np.float32),
        np.float32([0.0, -0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 1e30, -1e30]),
        np.nextafter(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]), np.float32(0)),
        np.nextafter(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]), np.float32(10)),
    ])
    got = F.e2m1_encode(xs)
    want = np.array([_brute_force_e2m1(float(v)) for v in xs], np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert F.E4M3_MAX == 448.0


def test_e4m3_points_table():
    for code, val in golden_lines("e4m3_points.txt"):
        got = F.e4m3_decode(int(code, 16)).item()
        want = float("nan") if val == "nan" else float.fromhex(val) if "0x" in val else float(val)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got)


def test_e4m3_encode_vs_torch_rne():
    # every finite value, every midpoint (ties) and one ulp either side of it
    pos = F.E4M3_POSITIVE
    mids = (pos[:-1] + pos[1:]) / 2
    base = np.concatenate([pos, mids]).astype(np.float32)
    xs = np.concatenate([base, np.nextafter(base, np.float32(0)), np.nextafter(base, np.float32(1e9)),
                         np.random.default_rng(1).uniform(0, 448, 5000).astype(np.float32)])
    xs = xs[(xs >= 0) & (xs <= 448)]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode_satfinite(xs)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    xs = np.float32([448.0, 460.0, 464.0, 500.0, 1e6, 3e38])
    assert np.all(F.e4m3_encode_satfinite(xs) == 0x7E)


def test_bf16_roundtrip_and_fp32_rne_vs_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
                        np.float32([0.0, -0.0, 1.0, -2.5, 1e-40, -1e-39, 3e38])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = F.f64_to_bf16_rne(x.astype(np.float64))
    assert np.array_equal(got, ref)
    assert np.array_equal(F.bf16_to_f64(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_single_rounding_from_f64():
    # 1 + 2^-8 + 2^-40 lies above the bf16 midpoint 1 + 2^-8 and must round up;
    # rounding through float32 first would land on the midpoint and round to 1.0.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert F.f64_to_bf16_rne(np.float64(x)) == 0x3F81
    assert F.f64_to_bf16_rne(np.float64(1.0 + 2.0 ** -8)) == 0x3F80  # exact tie -> even
    assert F.f64_to_bf16_rne(np.float64(1.0 + 3 * 2.0 ** -8)) == 0x3F82


def test_nibble_packing_order():
    # element 2j -> low nibble, element 2j+1 -> high nibble of byte j
    codes = np.array([[0x1, 0x2, 0xF, 0x0, 0x8, 0x7]], np.uint8)
    packed = F.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x0F, 0x78]]
    assert np.array_equal(F.unpack_nibbles(packed), codes)
