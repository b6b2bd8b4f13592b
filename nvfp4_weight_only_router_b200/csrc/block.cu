// Per-token kernels of the full MoE block ("Gemma 4 26B-A4B (MoE) - Core
// AI", the layer dataflow listing):
//   x1 = pre_feedforward_layernorm(x), x2 = pre_feedforward_layernorm_2(x)
//        (the two MLP inputs, rounded to bf16 as the block's bf16 modules
//        receive them);
//   hd = gelu_tanh(gate) * up of the dense MLP, split exactly into bf16 high
//        and low parts for the down GEMM;
//   out = (x + post_feedforward_layernorm(post_feedforward_layernorm_1(h)
//          + post_feedforward_layernorm_2(sum_k w_k h2_k))) * layer_scalar.
// Every norm is x / sqrt(mean(x^2) + eps) * weight, in fp32.  One CTA of
// 352 threads per token, each thread holding 8 consecutive elements of the
// 2816-element row.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kBT = kH / 8;  // 352 threads, 8 elements each

// Sum of v over the CTA (352 threads = 11 warps), returned to every thread;
// red[] holds 11 floats of scratch.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();  // red[] free from any earlier use
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kBT / 32; ++w) t += red[w];
  return t;
}

__device__ __forceinline__ void load_bf16x8(const uint16_t* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = bf16_bits_to_f32(w[k] & 0xFFFFu);
    v[2 * k + 1] = bf16_bits_to_f32(w[k] >> 16);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = pack_bf16x2(__float2bfloat16_rn(v[2 * k]), __float2bfloat16_rn(v[2 * k + 1]));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kBT) block_prenorm_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ g1,
                                                            const uint16_t* __restrict__ g2, float eps,
                                                            uint16_t* __restrict__ x1, uint16_t* __restrict__ x2) {
  __shared__ float red[kBT / 32];
  const size_t row = (size_t)blockIdx.x * kH;
  const int c = threadIdx.x * 8;
  float v[8], w1[8], w2[8];
  load_bf16x8(x + row + c, v);
  load_bf16x8(g1 + c, w1);
  load_bf16x8(g2 + c, w2);
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) ss = __fmaf_rn(v[k], v[k], ss);
  const float inv = 1.0f / sqrtf(block_sum(ss, red) / (float)kH + eps);
  float a[8], b[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    a[k] = v[k] * inv * w1[k];
    b[k] = v[k] * inv * w2[k];
  }
  *reinterpret_cast<uint4*>(x1 + row + c) = pack_bf16x8(a);
  *reinterpret_cast<uint4*>(x2 + row + c) = pack_bf16x8(b);
}

// hd[t, n] = gelu_tanh(g) * u with g, u the split-ordered sums of the gate_up
// partials; written as hi = bf16(hd), lo = bf16(hd - hi).  One thread per 4
// consecutive n.
__global__ void __launch_bounds__(256) dense_act_kernel(const float* __restrict__ part, int splits, int T,
                                                        uint16_t* __restrict__ hi, uint16_t* __restrict__ lo) {
  constexpr int per_tok = kDenseI / 4;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * per_tok) return;
  const int t = (int)(i / per_tok), n = (int)(i % per_tok) * 4;
  float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < splits; ++s) {
    const float* p = part + ((size_t)s * T + t) * (2 * kDenseI);
    const float4 a = *reinterpret_cast<const float4*>(p + n);
    const float4 b = *reinterpret_cast<const float4*>(p + kDenseI + n);
    g[0] += a.x; g[1] += a.y; g[2] += a.z; g[3] += a.w;
    u[0] += b.x; u[1] += b.y; u[2] += b.z; u[3] += b.w;
  }
  uint32_t wh[2], wl[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float h0 = gelu_tanh(g[2 * k]) * u[2 * k], h1 = gelu_tanh(g[2 * k + 1]) * u[2 * k + 1];
    const __nv_bfloat16 a0 = __float2bfloat16_rn(h0), a1 = __float2bfloat16_rn(h1);
    wh[k] = pack_bf16x2(a0, a1);
    wl[k] = pack_bf16x2(__float2bfloat16_rn(h0 - __bfloat162float(a0)), __float2bfloat16_rn(h1 - __bfloat162float(a1)));
  }
  *reinterpret_cast<uint2*>(hi + (size_t)t * kDenseI + n) = make_uint2(wh[0], wh[1]);
  *reinterpret_cast<uint2*>(lo + (size_t)t * kDenseI + n) = make_uint2(wl[0], wl[1]);
}

__global__ void __launch_bounds__(kBT) block_final_kernel(BlockFinalArgs a) {
  __shared__ float red[kBT / 32];
  const int t = blockIdx.x;
  const int c = threadIdx.x * 8;
  // the sparse branch: the token's 8 per-slot rows (already x routing weight x
  // G_d) summed in slot order
  float ym[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < kTopK; ++j) {
    const int pos = a.slot_pos[t * kTopK + j];
    if (pos < 0) continue;
    const float4* src = reinterpret_cast<const float4*>(a.obuf + (size_t)pos * kH + c);
    const float4 p0 = __ldcs(src), p1 = __ldcs(src + 1);
    ym[0] += p0.x; ym[1] += p0.y; ym[2] += p0.z; ym[3] += p0.w;
    ym[4] += p1.x; ym[5] += p1.y; ym[6] += p1.z; ym[7] += p1.w;
  }
  // the dense branch: its K-split partials summed in split order
  float hd[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < a.splits; ++s) {
    const float4* src = reinterpret_cast<const float4*>(a.dense + ((size_t)s * a.T + t) * kH + c);
    const float4 p0 = __ldcs(src), p1 = __ldcs(src + 1);
    hd[0] += p0.x; hd[1] += p0.y; hd[2] += p0.z; hd[3] += p0.w;
    hd[4] += p1.x; hd[5] += p1.y; hd[6] += p1.z; hd[7] += p1.w;
  }
  float q2 = 0.f, q1 = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    q2 = __fmaf_rn(ym[k], ym[k], q2);
    q1 = __fmaf_rn(hd[k], hd[k], q1);
  }
  const float inv2 = 1.0f / sqrtf(block_sum(q2, red) / (float)kH + a.eps);
  const float inv1 = 1.0f / sqrtf(block_sum(q1, red) / (float)kH + a.eps);
  float wp1[8], wp2[8], wp[8], xv[8], s[8];
  load_bf16x8(a.post1 + c, wp1);
  load_bf16x8(a.post2 + c, wp2);
  load_bf16x8(a.post + c, wp);
  load_bf16x8(a.x + (size_t)t * kH + c, xv);
  float qs = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    s[k] = hd[k] * inv1 * wp1[k] + ym[k] * inv2 * wp2[k];  // h1 + h2
    qs = __fmaf_rn(s[k], s[k], qs);
  }
  const float invs = 1.0f / sqrtf(block_sum(qs, red) / (float)kH + a.eps);
  const float ls = bf16_bits_to_f32(__ldg(a.layer_scalar));
  float o[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = (xv[k] + s[k] * invs * wp[k]) * ls;
  *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.y) + (size_t)t * kH + c) = pack_bf16x8(o);
}

}  // namespace

cudaError_t launch_block_prenorm(const uint16_t* x, const uint16_t* g1, const uint16_t* g2, float eps, int T,
                                 uint16_t* x1, uint16_t* x2, cudaStream_t st) {
  block_prenorm_kernel<<<T, kBT, 0, st>>>(x, g1, g2, eps, x1, x2);
  return cudaGetLastError();
}

cudaError_t launch_dense_act(const float* part, int splits, int T, uint16_t* hi, uint16_t* lo, cudaStream_t st) {
  const int64_t n = (int64_t)T * (kDenseI / 4);
  dense_act_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, splits, T, hi, lo);
  return cudaGetLastError();
}

cudaError_t launch_block_final(const BlockFinalArgs& a, cudaStream_t st) {
  block_final_kernel<<<a.T, kBT, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
