// NVFP4 block encoder shared by the weight quantiser and the W4A4
// activation quantisation ("Gemma-4-26B-A4B-it-NVFP4" page, block-scale
// formulas, in the two-level form of the "gemma-4-26B-A4B . NVFP4A16" card):
// for a block of 16 values under the FP32 global G, the scale code
// s = E4M3_rne_satfinite((amax_b / 6) / G), d = s * G, and per element the E2M1
// code nearest to x / d (ties to the even code, saturating at 6, sign of x),
// each step one correctly rounded fp32 operation.
#pragma once

#include "common.cuh"

namespace nvfp4moe {

// E4M3 round-to-nearest-even with saturation to 448, for t >= 0.
__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(t));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2 = e4m3x2_to_f16x2((uint16_t)(code | (code << 8)));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Two fp32 values -> two E2M1 codes (4-bit: sign, 2 exponent bits, 1 mantissa
// bit) in one byte, `hi` in the high nibble: the hardware conversion rounds to
// nearest with ties to the even code and saturates at 6, which is the grid
// rounding of the method; the sign bit follows the value (-0 and negatives
// that round to 0 give 0x8).
__device__ __forceinline__ uint32_t e2m1x2_rne(float hi, float lo) {
  uint16_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u16.u8 %0, b;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// Eight fp32 values -> eight E2M1 codes (same rounding as e2m1x2_rne), element
// i in nibble i of the result (element 2j in the low nibble of byte j).
__device__ __forceinline__ uint32_t e2m1x8_rne(const float (&x)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
  return r;
}

// Approximate reciprocal (relative error at most 2^-23; normal inputs).
__device__ __forceinline__ float rcp_approx(float d) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  return r;
}

// Per-tensor constants of the block encoder for the FP32 global G: G itself
// and k ~ 1 / (6 G) for the bracketed scale step.
struct TensorScale {
  float G, k_lo, k_hi;
  bool fast;  // k finite: the bracketed scale step applies
};

__device__ __forceinline__ TensorScale scale_consts(float G) {
  TensorScale t;
  t.G = G;
  const float g6 = __fmul_rn(6.0f, t.G);
  t.fast = g6 >= 1.17549435e-38f;
  const float k = t.fast ? __fdiv_rn(1.0f, g6) : 0.0f;  // 1 / (6 G), relative error <= 2^-23
  t.k_lo = __fmul_rn(k, 0.99999904632568359375f);      // 1 - 2^-20
  t.k_hi = __fmul_rn(k, 1.00000095367431640625f);      // 1 + 2^-20
  return t;
}

// A weight tensor's constants: G = amax / 2688 (one correctly rounded division).
__device__ __forceinline__ TensorScale tensor_scale(float amax) { return scale_consts(__fdiv_rn(amax, 2688.0f)); }

// two fp32 products a * r of a pair in one packed instruction (each lane
// correctly rounded, as two separate multiplies)
__device__ __forceinline__ void mul_f32x2(float a0, float a1, float r, float& p0, float& p1) {
  uint64_t x, rr, out;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(out) : "l"(x), "l"(rr));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(p0), "=f"(p1) : "l"(out));
}

// The defined steps are t = (amax_b / 6) / G and x = w / d, each a correctly
// rounded division, then monotone roundings (E4M3 RNE-satfinite of t, E2M1
// RNE of x).  Each quotient is bracketed instead: the product with an
// approximate reciprocal scaled by 1 -+ 2^-20 lies strictly below / above the
// correctly rounded quotient (the approximations err by at most ~2^-22), so
// when both ends round to the same code, so does the exact quotient.  Where
// they differ (a quotient within ~2^-20 of a rounding threshold) the block
// takes the correctly rounded divisions.
//
// One block of 16 fp32 values x with amax_b = max |x_i|: returns the e4m3
// scale code and the 16 E2M1 codes packed two per byte (element 2j in the low
// nibble).
__device__ __forceinline__ uint32_t encode_block16f(const float (&x)[16], float amax_b, const TensorScale& ts,
                                                    uint2& codes) {
  const float G = ts.G;
  uint32_t sc = 0;
  if (G > 0.0f) {
    bool done = false;
    if (ts.fast) {
      uint16_t two;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
          : "=h"(two)
          : "f"(__fmul_rn(amax_b, ts.k_hi)), "f"(__fmul_rn(amax_b, ts.k_lo)));
      sc = two & 0xFFu;
      done = (uint32_t)(two >> 8) == sc;
    }
    if (!done) sc = f32_to_e4m3_satfinite(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), G));
  }
  const float d = __fmul_rn(e4m3_to_f32(sc), G);

  uint32_t packed[2] = {0u, 0u};
  if (d > 0.0f) {
    bool exact = false;
    if (d >= 1.17549435e-38f) {  // normal d: 1/d is finite
      const float r = rcp_approx(d);
      const float rl = __fmul_rn(r, 0.99999904632568359375f);  // 1 - 2^-20
      const float rh = __fmul_rn(r, 1.00000095367431640625f);  // 1 + 2^-20
      uint32_t hi[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          mul_f32x2(x[8 * h + i], x[8 * h + i + 1], rl, a[i], a[i + 1]);
          mul_f32x2(x[8 * h + i], x[8 * h + i + 1], rh, b[i], b[i + 1]);
        }
        packed[h] = e2m1x8_rne(a);
        hi[h] = e2m1x8_rne(b);
      }
      exact = packed[0] == hi[0] && packed[1] == hi[1];
    }
    if (!exact) {
      // a quotient close to a rounding threshold (or a subnormal d): the
      // correctly rounded division decides
      packed[0] = packed[1] = 0u;
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const uint32_t byte = e2m1x2_rne(__fdiv_rn(x[i + 1], d), __fdiv_rn(x[i], d));
        packed[i >> 3] |= byte << ((i & 7) * 4);
      }
    }
  } else {
    // zero block (d = 0): only the sign bits
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i >> 3] |= ((__float_as_uint(x[i]) >> 31) << 3) << ((i & 7) * 4);
  }
  codes = make_uint2(packed[0], packed[1]);
  return sc;
}

}  // namespace nvfp4moe
