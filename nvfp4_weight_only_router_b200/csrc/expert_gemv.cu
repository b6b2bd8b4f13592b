// Grouped NVFP4 expert GEMMs for few tokens per expert (decode), on warp-level
// tensor-core MMAs with the weights dequantised in registers.
//
// Per expert e and routed token x ("Gemma 4 26B-A4B (MoE) - Core AI": GELU-tanh
// gated experts; fused gate||up rows, gate first):
//   gate = G_gu[e] * (Wq[e, 0:I] x),  up = G_gu[e] * (Wq[e, I:2I] x)
//   h    = gelu_tanh(gate) * up
//   out  = G_d[e] * (Wq_d[e] h)
// with Wq = e2m1 * e4m3 (exact in f16; "Gemma-4-26B-A4B-NVFP4-mlx",
// "Quantization recipe").
//
// Decode is bound by the bytes of the selected experts (the same card's
// "gather kernel" note: only the routed experts are read).  Each weight byte is
// loaded once, with 16-byte coalesced loads, and turned into f16 MMA operands
// by the hardware E2M1->f16x2 conversion and one f16x2 multiply by the block
// scale.  Tokens are the MMA's N dimension (8 per n-tile).
//
// MMA fragment correspondence (m16n8k16, A row-major, B column-major): within a
// 128-element K segment, lane quad q holds K elements [32q, 32q+32) -- one
// 16-byte chunk of packed weights and 64 bytes of the f16 activation row; MMA
// step j takes elements 32q+4j+{0,1} as the fragment's low k-pair and
// 32q+4j+{2,3} as its high k-pair, for both operands.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kGuRowBlocks = kI / 8;    // 88 CTAs per expert: 8 gate + 8 up rows each
constexpr int kDnRowsPerCta = 64;       // 4 warps x 16 rows
constexpr int kDnCtas = kH / kDnRowsPerCta;  // 44 CTAs per expert
constexpr int kGuSegsPerWarp = 6;       // 22 segments over 4 warps: 6, 6, 5, 5

// Weight fragment for one 16-byte chunk of rows (r, r+8): dequantise word w
// (elements 8w..8w+7) of each row and multiply by the block scale.  Produces
// the A registers of MMA steps 2w and 2w+1.
__device__ __forceinline__ void dequant_word(uint32_t wr0, uint32_t wr1, uint32_t s0, uint32_t s1,
                                             uint32_t (&A0)[4], uint32_t (&A1)[4]) {
  uint32_t f0[4], f1[4];
  e2m1x8_to_f16x2(wr0, f0);
  e2m1x8_to_f16x2(wr1, f1);
  A0[0] = hmul2_u32(f0[0], s0);
  A0[1] = hmul2_u32(f1[0], s1);
  A0[2] = hmul2_u32(f0[1], s0);
  A0[3] = hmul2_u32(f1[1], s1);
  A1[0] = hmul2_u32(f0[2], s0);
  A1[1] = hmul2_u32(f1[2], s1);
  A1[2] = hmul2_u32(f0[3], s0);
  A1[3] = hmul2_u32(f1[3], s1);
}

// acc += W(rows r, r+8; one 32-element chunk) * X(8 tokens; same chunk)
__device__ __forceinline__ void mma_chunk(float (&acc)[4], const uint4& w0, const uint4& w1,
                                          uint32_t sc0, uint32_t sc1, const uint4 (&xb)[4]) {
  const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w};
  const uint32_t a1[4] = {w1.x, w1.y, w1.z, w1.w};
  const uint32_t s0lo = bcast_lo(sc0), s0hi = bcast_hi(sc0);
  const uint32_t s1lo = bcast_lo(sc1), s1hi = bcast_hi(sc1);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t A0[4], A1[4];
    dequant_word(a0[w], a1[w], w < 2 ? s0lo : s0hi, w < 2 ? s1lo : s1hi, A0, A1);
    mma_f16_16816(acc, A0, xb[w].x, xb[w].y);
    mma_f16_16816(acc, A1, xb[w].z, xb[w].w);
  }
}

__device__ __forceinline__ void load_x_chunk(const __half* row, bool valid, uint4 (&xb)[4]) {
  if (valid) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
#pragma unroll
    for (int i = 0; i < 4; ++i) xb[i] = __ldg(p + i);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) xb[i] = make_uint4(0, 0, 0, 0);
  }
}

// gate_up + GELU gate.  CTA = (active expert, 8-row block): MMA rows 0..7 are
// gate rows 8rb..8rb+7 and rows 8..15 the matching up rows, so each lane holds
// the gate and up value of the same hidden unit.  The 4 warps split K and meet
// in shared memory.
__global__ void __launch_bounds__(128) gate_up_gemv_kernel(ExpertArgs p) {
  const int a = blockIdx.x / kGuRowBlocks, rb = blockIdx.x % kGuRowBlocks;
  if (a >= p.meta[kMetaNAct]) return;
  const int e = p.meta[kMetaAct + a];
  const int off = p.meta[kMetaOffsets + e];
  const int cnt = p.meta[kMetaOffsets + e + 1] - off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, qd = lane & 3;

  const size_t rowG = (size_t)e * (2 * kI) + rb * 8 + g, rowU = rowG + kI;
  const uint8_t* wG = p.gu_q + rowG * kGuRowBytes + qd * 16;
  const uint8_t* wU = p.gu_q + rowU * kGuRowBytes + qd * 16;
  const uint8_t* sG = p.gu_s + rowG * kGuScaleRow + qd * 2;
  const uint8_t* sU = p.gu_s + rowU * kGuScaleRow + qd * 2;

  uint4 wg[kGuSegsPerWarp], wu[kGuSegsPerWarp];
  uint32_t scg[kGuSegsPerWarp], scu[kGuSegsPerWarp];
#pragma unroll
  for (int i = 0; i < kGuSegsPerWarp; ++i) {
    const int seg = warp + 4 * i;
    if (seg < kGuSegs) {
      wg[i] = ldg_nc_v4(wG + seg * 64);
      wu[i] = ldg_nc_v4(wU + seg * 64);
      scg[i] = e4m3x2_to_f16x2(ldg_nc_u16(sG + seg * 8));
      scu[i] = e4m3x2_to_f16x2(ldg_nc_u16(sU + seg * 8));
    }
  }

  __shared__ float4 red[4][32];
  const float G = p.gu_g[e];
  for (int n0 = 0; n0 < cnt; n0 += 8) {
    int tok = -1;
    if (n0 + g < cnt) {
      tok = p.sorted_slot[off + n0 + g] / kTopK;
      if (tok < 0 || tok >= p.T) {
        record_status(p.status, kStatusDevice);
        tok = -1;
      }
    }
    const __half* xrow = p.x16 + (size_t)(tok < 0 ? 0 : tok) * kH + qd * 32;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kGuSegsPerWarp; ++i) {
      const int seg = warp + 4 * i;
      if (seg < kGuSegs) {
        uint4 xb[4];
        load_x_chunk(xrow + seg * kSegK, tok >= 0, xb);
        mma_chunk(acc, wg[i], wu[i], scg[i], scu[i], xb);
      }
    }
    red[warp][lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (warp == 0) {
      float4 v = red[0][lane];
#pragma unroll
      for (int w = 1; w < 4; ++w) {
        const float4 o = red[w][lane];
        v.x += o.x;
        v.y += o.y;
        v.z += o.z;
        v.w += o.w;
      }
      // v.x, v.y: gate row g, tokens 2qd, 2qd+1; v.z, v.w: up row g, same tokens
      const int c0 = n0 + 2 * qd;
      if (c0 < cnt) {
        const float hv = gelu_tanh(G * v.x) * (G * v.z);
        p.h[(size_t)(off + c0) * kI + rb * 8 + g] = f32_to_f16_sat(hv);
      }
      if (c0 + 1 < cnt) {
        const float hv = gelu_tanh(G * v.y) * (G * v.w);
        p.h[(size_t)(off + c0 + 1) * kI + rb * 8 + g] = f32_to_f16_sat(hv);
      }
    }
    __syncthreads();
  }
}

// down projection.  CTA = (active expert, 64 output rows); warp = 16 rows over
// the whole K = 704 (5.5 segments; lanes beyond K in the last one idle).
// mode 0 writes per-slot outputs (deterministic combine in finalize);
// mode 1 accumulates w * out into the fp32 token accumulator with atomics.
__global__ void __launch_bounds__(128) down_gemv_kernel(ExpertArgs p) {
  const int a = blockIdx.x / kDnCtas, cb = blockIdx.x % kDnCtas;
  if (a >= p.meta[kMetaNAct]) return;
  const int e = p.meta[kMetaAct + a];
  const int off = p.meta[kMetaOffsets + e];
  const int cnt = p.meta[kMetaOffsets + e + 1] - off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, qd = lane & 3;
  const int r0 = cb * kDnRowsPerCta + warp * 16 + g, r1 = r0 + 8;

  const uint8_t* w0p = p.dn_q + ((size_t)e * kH + r0) * kDnRowBytes + qd * 16;
  const uint8_t* w1p = p.dn_q + ((size_t)e * kH + r1) * kDnRowBytes + qd * 16;
  const uint8_t* s0p = p.dn_s + ((size_t)e * kH + r0) * kDnScaleRow + qd * 2;
  const uint8_t* s1p = p.dn_s + ((size_t)e * kH + r1) * kDnScaleRow + qd * 2;

  uint4 w0[kDnSegs], w1[kDnSegs];
  uint32_t sc0[kDnSegs], sc1[kDnSegs];
#pragma unroll
  for (int seg = 0; seg < kDnSegs; ++seg) {
    const bool valid = seg * kSegK + qd * 32 < kI;
    if (valid) {
      w0[seg] = ldg_nc_v4(w0p + seg * 64);
      w1[seg] = ldg_nc_v4(w1p + seg * 64);
      sc0[seg] = e4m3x2_to_f16x2(ldg_nc_u16(s0p + seg * 8));
      sc1[seg] = e4m3x2_to_f16x2(ldg_nc_u16(s1p + seg * 8));
    } else {
      w0[seg] = w1[seg] = make_uint4(0, 0, 0, 0);
      sc0[seg] = sc1[seg] = 0;
    }
  }
  const float G = p.dn_g[e];
  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool has = n0 + g < cnt;
    const __half* hrow = p.h + (size_t)(off + (has ? n0 + g : 0)) * kI + qd * 32;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int seg = 0; seg < kDnSegs; ++seg) {
      const bool valid = seg * kSegK + qd * 32 < kI;
      uint4 xb[4];
      load_x_chunk(hrow + seg * kSegK, has && valid, xb);
      mma_chunk(acc, w0[seg], w1[seg], sc0[seg], sc1[seg], xb);
    }
    // acc: (row r0, cols 2qd, 2qd+1), (row r1, same cols)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = n0 + 2 * qd + c;
      if (col >= cnt) continue;
      const int pos = off + col;
      const int slot = p.sorted_slot[pos];
      const float wgt = p.wts[slot] * G;
      const float o0 = acc[c] * wgt, o1 = acc[2 + c] * wgt;
      if (p.mode == 0) {
        p.obuf[(size_t)pos * kH + r0] = o0;
        p.obuf[(size_t)pos * kH + r1] = o1;
      } else {
        const int tok = slot / kTopK;
        atomicAdd(p.yacc + (size_t)tok * kH + r0, o0);
        atomicAdd(p.yacc + (size_t)tok * kH + r1, o1);
      }
    }
  }
}

// y = bf16(sum_j out_j) per token.  mode 0 sums the 8 per-slot rows in slot
// order (deterministic); mode 1 converts the fp32 accumulator.  One thread per
// 8 consecutive outputs.
__global__ void __launch_bounds__(256) finalize_kernel(ExpertArgs p) {
  const int per_tok = kH / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)p.T * per_tok) return;
  const int t = (int)(i / per_tok), c = (int)(i % per_tok) * 8;
  float v[8];
  if (p.mode == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = 0.f;
    for (int j = 0; j < kTopK; ++j) {
      const int pos = p.slot_pos[t * kTopK + j];
      if (pos < 0) continue;
      const float4* src = reinterpret_cast<const float4*>(p.obuf + (size_t)pos * kH + c);
      const float4 x0 = src[0], x1 = src[1];
      v[0] += x0.x; v[1] += x0.y; v[2] += x0.z; v[3] += x0.w;
      v[4] += x1.x; v[5] += x1.y; v[6] += x1.z; v[7] += x1.w;
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(p.yacc + (size_t)t * kH + c);
    const float4 x0 = src[0], x1 = src[1];
    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
  }
  uint4 o;
  o.x = pack_bf16x2(__float2bfloat16_rn(v[0]), __float2bfloat16_rn(v[1]));
  o.y = pack_bf16x2(__float2bfloat16_rn(v[2]), __float2bfloat16_rn(v[3]));
  o.z = pack_bf16x2(__float2bfloat16_rn(v[4]), __float2bfloat16_rn(v[5]));
  o.w = pack_bf16x2(__float2bfloat16_rn(v[6]), __float2bfloat16_rn(v[7]));
  *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.y) + (size_t)t * kH + c) = o;
}

}  // namespace

cudaError_t launch_gate_up_gemv(const ExpertArgs& a, cudaStream_t st) {
  gate_up_gemv_kernel<<<a.max_active * kGuRowBlocks, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_down_gemv(const ExpertArgs& a, cudaStream_t st) {
  down_gemv_kernel<<<a.max_active * kDnCtas, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const ExpertArgs& a, cudaStream_t st) {
  const int64_t n = (int64_t)a.T * (kH / 8);
  finalize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
