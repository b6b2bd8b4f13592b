// Weighted combine of the routed experts' outputs ("Gemma 4 26B-A4B (MoE) -
// Core AI": the token's output is the router-weighted sum over its top-8
// experts).  The down GEMMs already multiplied each slot's row by its routing
// weight and the expert's global scale and stored it at the slot's sorted
// position; this kernel sums the rows of a token in slot order j = 0, 1, ...
// (8 slots, or 128 in the dense over-read) and rounds once to bf16, so the
// result does not depend on launch order.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

// One thread per 8 consecutive outputs of a token: two 16-byte loads per slot,
// one 16-byte bf16 store.
__global__ void __launch_bounds__(256) finalize_kernel(ExpertArgs p) {
  const int per_tok = kH / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)p.T * per_tok) return;
  const int t = (int)(i / per_tok), c = (int)(i % per_tok) * 8;
  float v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = 0.f;
  for (int j = 0; j < p.spt; ++j) {
    const int pos = p.slot_pos[t * p.spt + j];
    if (pos < 0) continue;
    const float4* src = reinterpret_cast<const float4*>(p.obuf + (size_t)pos * kH + c);
    const float4 x0 = __ldcs(src), x1 = __ldcs(src + 1);
    v[0] += x0.x; v[1] += x0.y; v[2] += x0.z; v[3] += x0.w;
    v[4] += x1.x; v[5] += x1.y; v[6] += x1.z; v[7] += x1.w;
  }
  uint4 o;
  o.x = pack_bf16x2(__float2bfloat16_rn(v[0]), __float2bfloat16_rn(v[1]));
  o.y = pack_bf16x2(__float2bfloat16_rn(v[2]), __float2bfloat16_rn(v[3]));
  o.z = pack_bf16x2(__float2bfloat16_rn(v[4]), __float2bfloat16_rn(v[5]));
  o.w = pack_bf16x2(__float2bfloat16_rn(v[6]), __float2bfloat16_rn(v[7]));
  *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.y) + (size_t)t * kH + c) = o;
}

}  // namespace

cudaError_t launch_finalize(const ExpertArgs& a, cudaStream_t st) {
  const int64_t n = (int64_t)a.T * (kH / 8);
  finalize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
