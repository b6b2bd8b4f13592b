"""Number formats of the NVFP4 scheme, from their definitions.  Test
infrastructure only (see the package docstring).

E2M1 ("Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe"; "gemma-4-26B-A4B .
NVFP4A16", "Quantization details"): 1 sign bit, 2 exponent bits (bias 1),
1 mantissa bit.  Exponent field 0 is subnormal (value = m * 0.5).  The
magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}; the largest is the V_max = 6 of
the "Gemma-4-26B-A4B-it-NVFP4" block-scale formula.

E4M3 (the FP8 block-scale type of the same cards): 1 sign bit, 4 exponent bits
(bias 7), 3 mantissa bits; field 0 is subnormal (m * 2^-9); the all-ones
exponent with mantissa 7 is NaN and there is no infinity, so the largest
finite value is 1.75 * 2^8 = 448.

bf16: the top 16 bits of an IEEE binary32.
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------- E2M1
def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit E2M1 code (low 4 bits of `codes`), as float64."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e - 1.0))
    return sign * mag


# The eight magnitudes in code order, derived from the definition above.
E2M1_MAGNITUDES = e2m1_decode(np.arange(8))


def _round_to_grid_rne(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into an increasing grid of the nearest grid value to each `mag`
    (>= 0), ties to the even index.  Values above the last grid point go to
    the last index.  All arithmetic is on float64 values that are exact for
    the inputs used here (fp32 inputs, short grid values), and the two
    differences compared are between a value and its two bracketing grid
    points, so they are exact."""
    mag = np.asarray(mag, np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi-1] < mag <= grid[hi]
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[-1], len(grid) - 1, idx)   # saturate
    idx = np.where(mag <= grid[0], 0, idx)
    return idx


def e2m1_encode(x) -> np.ndarray:
    """Round each value of `x` (float32 or float64) to the E2M1 grid,
    round-to-nearest with ties to the even code, saturating at +-6, and
    return the 4-bit code.  The sign bit is the sign bit of x (so -0.0 and
    small negatives that round to zero give code 0x8)."""
    x = np.asarray(x)
    mag_idx = _round_to_grid_rne(np.abs(x.astype(np.float64)), E2M1_MAGNITUDES)
    sign = np.signbit(x).astype(np.int64)
    return ((sign << 3) | mag_idx).astype(np.uint8)


# --------------------------------------------------------------------------- E4M3
def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte, as float64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# Non-negative finite E4M3 values in code order 0x00..0x7E (increasing).
E4M3_POSITIVE = e4m3_decode(np.arange(0x7F))
E4M3_MAX = float(E4M3_POSITIVE[-1])  # 448


def e4m3_encode_satfinite(t) -> np.ndarray:
    """Round non-negative values to E4M3, round-to-nearest-even, saturating to
    the largest finite value 448 (never producing NaN).  Returns the byte."""
    t = np.asarray(t, np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("e4m3_encode_satfinite expects non-negative, non-NaN values")
    return _round_to_grid_rne(t, E4M3_POSITIVE).astype(np.uint8)


# --------------------------------------------------------------------------- bf16
def bf16_to_f64(bits) -> np.ndarray:
    """Value of bf16 bit patterns (uint16) as float64 (exact)."""
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_to_f32(bits) -> np.ndarray:
    """Value of bf16 bit patterns (uint16) as float32 (exact)."""
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def f64_to_bf16_rne(x) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits, binary32 exponent
    range, round-to-nearest-even, subnormals kept, overflow to inf) and return
    the bit patterns.  One rounding directly from float64."""
    x = np.asarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    flat = x.ravel()
    res = out.ravel()
    finite = np.isfinite(flat)
    mag = np.abs(flat)
    # Quantum of the bf16 grid at each magnitude: 2^(exponent - 7) for normals,
    # 2^-133 for the subnormal range (below 2^-126).
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    # log2 can be off by one near powers of two; fix with exact comparisons.
    ex = np.where(np.exp2(ex) > mag, ex - 1, ex)
    ex = np.where(np.exp2(ex + 1) <= mag, ex + 1, ex)
    ex = np.maximum(ex, -126.0)
    q = np.exp2(ex - 7.0)
    r = np.rint(mag / q) * q            # mag/q is exact (power-of-two scaling); rint is RNE
    r = np.where(finite, r, mag)
    signed = np.copysign(r, flat)
    f32 = signed.astype(np.float32)     # exact: r has <= 8 significant bits (inf if too big)
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    nan = np.isnan(flat)
    bits[nan] = 0x7FC0
    res[:] = bits
    return out


# ------------------------------------------------------------------ nibble packing
def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Pack 4-bit codes along the last axis: element 2j goes to the low nibble
    and element 2j+1 to the high nibble of byte j."""
    c = np.asarray(codes, np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of `pack_nibbles`."""
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
