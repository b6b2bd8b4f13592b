// NVFP4 quantise / dequantise kernels.
//
// Method ("Gemma-4-26B-A4B-it-NVFP4" page, block-scale formulas, in the
// two-level form of the "gemma-4-26B-A4B . NVFP4A16" card, "Quantization
// details"): per tensor G = amax / (6 * 448); per block of 16 along K
// s = E4M3_rne_satfinite((amax_b / 6) / G), d = s * G; per element the code is
// the E2M1 value nearest to w / d, ties to the even code, saturating at 6, with
// the sign bit of w.  Each step is one correctly rounded fp32 operation.
//
// Pass 1 (amax_kernel) reduces |w| per tensor; pass 2 (encode_kernel) encodes
// one 16-element block per thread with 32-byte loads and 8-byte stores.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

// |w| of a bf16 pattern as a monotone integer key (non-NaN inputs).
__device__ __forceinline__ uint32_t bf16_abs_key(uint32_t b) { return b & 0x7FFFu; }

__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ w, int64_t per_expert,
                                                   uint32_t* __restrict__ amax_bits) {
  const int e = blockIdx.y;
  const uint4* base = reinterpret_cast<const uint4*>(w + (size_t)e * per_expert);
  const int64_t n16 = per_expert / 8;  // 8 bf16 per 16-byte load
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 v = ldg_nc_v4(base + i);
    uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, bf16_abs_key(a[j] & 0xFFFFu));
      m = max(m, bf16_abs_key(a[j] >> 16));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = 1; j < (int)(blockDim.x >> 5); ++j) m = max(m, red[j]);
    atomicMax(amax_bits + e, m << 16);  // fp32 bit pattern of the bf16 amax
  }
}

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

__global__ void __launch_bounds__(256) encode_kernel(const uint16_t* __restrict__ w,
                                                     int64_t blocks_per_expert, int64_t n_blocks,
                                                     const uint32_t* __restrict__ amax_bits,
                                                     uint8_t* __restrict__ q, uint8_t* __restrict__ s,
                                                     float* __restrict__ g) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= n_blocks) return;
  const int64_t e = blk / blocks_per_expert;
  const float amax = __uint_as_float(amax_bits[e]);
  const float G = __fdiv_rn(amax, 2688.0f);
  if (blk == e * blocks_per_expert) g[e] = G;

  const uint4* src = reinterpret_cast<const uint4*>(w) + blk * 2;
  uint4 v0 = ldg_nc_v4(src), v1 = ldg_nc_v4(src + 1);
  uint32_t pair[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float x[16];
  uint32_t key = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    x[2 * j] = bf16_bits_to_f32(pair[j] & 0xFFFFu);
    x[2 * j + 1] = bf16_bits_to_f32(pair[j] >> 16);
    key = max(key, bf16_abs_key(pair[j] & 0xFFFFu));
    key = max(key, bf16_abs_key(pair[j] >> 16));
  }
  const float amax_b = __uint_as_float(key << 16);
  uint32_t sc = 0;
  if (G > 0.0f) sc = f32_to_e4m3_satfinite(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), G));
  const float d = __fmul_rn(e4m3_to_f32(sc), G);

  uint32_t packed[2] = {0u, 0u};
  if (d > 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      // element 2j in the low nibble of byte j
      const uint32_t byte = e2m1x2_rne(__fdiv_rn(x[i + 1], d), __fdiv_rn(x[i], d));
      packed[i >> 3] |= byte << ((i & 7) * 4);
    }
  } else {
    // zero block (d = 0): only the sign bits
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i >> 3] |= ((__float_as_uint(x[i]) >> 31) << 3) << ((i & 7) * 4);
  }
  *reinterpret_cast<uint2*>(q + blk * 8) = make_uint2(packed[0], packed[1]);
  s[blk] = (uint8_t)sc;
}

// w = e2m1 * e4m3 * G rounded once to fp32: e2m1 * e4m3 is exact in f16/f32,
// so the only rounding is the final multiply by G.  One thread per 8 codes.
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ q,
                                                      const uint8_t* __restrict__ s,
                                                      const float* __restrict__ g,
                                                      int64_t groups_per_expert, int64_t n_groups,
                                                      float* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // group of 8 codes
  if (i >= n_groups) return;
  const int64_t e = i / groups_per_expert;
  const uint32_t w = *reinterpret_cast<const uint32_t*>(q + i * 4);
  const uint32_t sc = s[i >> 1];  // 16 codes per scale, 8 per group
  const float sv = e4m3_to_f32(sc);
  const float G = g[e];
  uint32_t h[4];
  e2m1x8_to_f16x2(w, h);
  float4 o0, o1;
  float v[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[j] & 0xFFFFu))) * sv, G);
    v[2 * j + 1] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[j] >> 16))) * sv, G);
  }
  o0 = make_float4(v[0], v[1], v[2], v[3]);
  o1 = make_float4(v[4], v[5], v[6], v[7]);
  float4* dst = reinterpret_cast<float4*>(out + i * 8);
  dst[0] = o0;
  dst[1] = o1;
}

cudaError_t launch_quantize(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* q,
                            uint8_t* s, float* g, uint32_t* amax_ws, cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(amax_ws, 0, sizeof(uint32_t) * E, st);
  if (err != cudaSuccess) return err;
  const int64_t per = N * K;
  int gx = (int)((per / 8 + 255) / 256);
  if (gx > 64) gx = 64;
  amax_kernel<<<dim3(gx, (unsigned)E), 256, 0, st>>>(w, per, amax_ws);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t bpe = per / 16, nb = E * bpe;
  encode_kernel<<<(unsigned)((nb + 255) / 256), 256, 0, st>>>(w, bpe, nb, amax_ws, q, s, g);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* q, const uint8_t* s, const float* g, int64_t E,
                              int64_t N, int64_t K, float* out, cudaStream_t st) {
  const int64_t gpe = N * K / 8, ng = E * gpe;
  dequant_kernel<<<(unsigned)((ng + 255) / 256), 256, 0, st>>>(q, s, g, gpe, ng, out);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
