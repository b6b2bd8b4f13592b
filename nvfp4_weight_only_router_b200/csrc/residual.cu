// One link of a chained layer stack: res += y; x = bf16(rmsnorm(res)), with the
// scale-free RMSNorm of the router description ("Gemma 4 26B-A4B (MoE) - Core
// AI"): x / sqrt(mean(x^2) + eps).  One CTA per token; fp32 throughout.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

__global__ void __launch_bounds__(256) residual_rmsnorm_kernel(float* __restrict__ res,
                                                               const uint16_t* __restrict__ y,
                                                               uint16_t* __restrict__ x_out, int H,
                                                               float eps) {
  const int t = blockIdx.x;
  float* r = res + (size_t)t * H;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < H; c += blockDim.x * 4) {
    float4 v = *reinterpret_cast<float4*>(r + c);
    if (y) {
      const uint2 yy = *reinterpret_cast<const uint2*>(y + (size_t)t * H + c);
      v.x += bf16_bits_to_f32(yy.x & 0xFFFFu);
      v.y += bf16_bits_to_f32(yy.x >> 16);
      v.z += bf16_bits_to_f32(yy.y & 0xFFFFu);
      v.w += bf16_bits_to_f32(yy.y >> 16);
      *reinterpret_cast<float4*>(r + c) = v;
    }
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  __shared__ float red[8];
  __shared__ float s_inv;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
    s_inv = 1.0f / sqrtf(tot / (float)H + eps);
  }
  __syncthreads();
  const float inv = s_inv;
  for (int c = threadIdx.x * 4; c < H; c += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(r + c);
    const uint2 o = make_uint2(pack_bf16x2(__float2bfloat16_rn(v.x * inv), __float2bfloat16_rn(v.y * inv)),
                               pack_bf16x2(__float2bfloat16_rn(v.z * inv), __float2bfloat16_rn(v.w * inv)));
    *reinterpret_cast<uint2*>(x_out + (size_t)t * H + c) = o;
  }
}

}  // namespace

cudaError_t launch_residual_rmsnorm(float* res, const uint16_t* y, uint16_t* x_out, int T, int H,
                                    float eps, cudaStream_t st) {
  residual_rmsnorm_kernel<<<T, 256, 0, st>>>(res, y, x_out, H, eps);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
