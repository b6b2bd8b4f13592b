// Router: scale-free RMSNorm -> x scale x H^-0.5 -> linear to 128 experts ->
// fp32 softmax -> top-8 -> renormalise -> x per_expert_scale ("Gemma 4
// 26B-A4B (MoE) - Core AI", router description under the layer dataflow
// listing).
//
// The linear map is computed on the tensor cores without changing its fp32
// meaning: logit_e = inv_rms * H^-0.5 * sum_k (x_k * scale_k) * proj_ek.  The
// product x_k * scale_k of two bf16 values has at most 16 significant bits, so
// it splits exactly into hi + lo with hi = bf16(p) and lo = bf16(p - hi); two
// bf16 MMAs (hi and lo against the same proj fragment) accumulate the exact
// products in fp32.
//
// Work split: a CTA (4 warps) owns 16 tokens x 128 experts over a K range;
// warp w owns experts [32w, 32w+32).  For small T the K range is split over
// `ksplit` CTAs whose partial sums meet in the workspace; the last CTA of a
// token tile to finish (arrival counter) reduces them in a fixed order and runs
// softmax / top-8 for the tile, one warp per token.
//
// Within a 128-element K segment, lane quad q holds elements [32q, 32q+32);
// MMA step j of the segment takes elements 32q+4j+{0,1} into the low k-pair of
// the fragment and 32q+4j+{2,3} into the high k-pair.  A and B use the same
// correspondence, so each lane loads 16 contiguous bytes per operand row.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

__device__ __forceinline__ void split_hi_lo(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
  const __nv_bfloat16 l0 = __float2bfloat16_rn(p0 - __bfloat162float(h0));
  const __nv_bfloat16 l1 = __float2bfloat16_rn(p1 - __bfloat162float(h1));
  hi = pack_bf16x2(h0, h1);
  lo = pack_bf16x2(l0, l1);
}

// Top-8 of 128 logits held 4 per lane (expert lane + 32 i).  Ordered by
// descending logit (= descending probability); equal logits -> lower id first.
__device__ void finish_token(const RouteArgs& a, int t, const float (&lg)[4]) {
  const int lane = threadIdx.x & 31;
  float m = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float ex[4], z = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ex[i] = expf(lg[i] - m);
    z += ex[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  float p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = ex[i] / z;

  bool taken[4] = {false, false, false, false};
  int sel_id = 0;
  float sel_p = 0.f, psum = 0.f;
  for (int r = 0; r < kTopK; ++r) {
    // best remaining candidate of this lane (ids ascend with i)
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!taken[i] && (lg[i] > bv || bi == 0x7fffffff)) {
        bv = lg[i];
        bi = lane + 32 * i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    const int owner = bi & 31, slot = bi >> 5;
    float pw = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane == owner && slot == i) {
        taken[i] = true;
        pw = p[i];
      }
    pw = __shfl_sync(0xffffffffu, pw, owner);
    psum += pw;
    if (lane == r) {
      sel_id = bi;
      sel_p = pw;
    }
  }
  if (lane < kTopK) {
    const float pes = bf16_bits_to_f32(a.pes[sel_id]);
    a.ids[(size_t)t * kTopK + lane] = sel_id;
    a.wts[(size_t)t * kTopK + lane] = (sel_p / psum) * pes;
  }
}

__global__ void __launch_bounds__(128) route_kernel(RouteArgs a) {
  const int tile = blockIdx.x, ks = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int t0 = tile * 16 + g, t1 = t0 + 8;
  const bool v0 = t0 < a.T, v1 = t1 < a.T;
  const int nseg = a.H / kSegK;
  const int s_begin = ks * a.segs_per_split;
  const int s_end = min(nseg, s_begin + a.segs_per_split);
  const uint16_t* x0 = a.x + (size_t)(v0 ? t0 : 0) * a.H + 32 * q;
  const uint16_t* x1 = a.x + (size_t)(v1 ? t1 : 0) * a.H + 32 * q;
  const uint16_t* prow = a.proj + (size_t)(warp * 32 + g) * a.H + 32 * q;

  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
  float ss0 = 0.f, ss1 = 0.f;

  for (int seg = s_begin; seg < s_end; ++seg) {
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      const int k = seg * kSegK + 8 * sub;
      const uint4 zero = make_uint4(0, 0, 0, 0);
      const uint4 xa = v0 ? ldg_nc_v4(x0 + k) : zero;
      const uint4 xb = v1 ? ldg_nc_v4(x1 + k) : zero;
      const uint4 sc = ldg_nc_v4(a.scale + k + 32 * q);
      const uint32_t xaw[4] = {xa.x, xa.y, xa.z, xa.w}, xbw[4] = {xb.x, xb.y, xb.z, xb.w};
      const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
      uint32_t hi_a[4], lo_a[4], hi_b[4], lo_b[4];  // per 32-bit word (2 elements)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float s0 = bf16_bits_to_f32(scw[w] & 0xFFFFu), s1 = bf16_bits_to_f32(scw[w] >> 16);
        const float xa0 = bf16_bits_to_f32(xaw[w] & 0xFFFFu), xa1 = bf16_bits_to_f32(xaw[w] >> 16);
        const float xb0 = bf16_bits_to_f32(xbw[w] & 0xFFFFu), xb1 = bf16_bits_to_f32(xbw[w] >> 16);
        split_hi_lo(__fmul_rn(xa0, s0), __fmul_rn(xa1, s1), hi_a[w], lo_a[w]);
        split_hi_lo(__fmul_rn(xb0, s0), __fmul_rn(xb1, s1), hi_b[w], lo_b[w]);
        if (warp == 0) {
          ss0 = __fmaf_rn(xa0, xa0, ss0);
          ss0 = __fmaf_rn(xa1, xa1, ss0);
          ss1 = __fmaf_rn(xb0, xb0, ss1);
          ss1 = __fmaf_rn(xb1, xb1, ss1);
        }
      }
      if (warp == 0 && a.x16 != nullptr) {
        // f16 copy of x for the expert GEMMs (saturating)
        uint32_t o0[4], o1[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          o0[w] = pack_f16x2(f32_to_f16_sat(bf16_bits_to_f32(xaw[w] & 0xFFFFu)),
                             f32_to_f16_sat(bf16_bits_to_f32(xaw[w] >> 16)));
          o1[w] = pack_f16x2(f32_to_f16_sat(bf16_bits_to_f32(xbw[w] & 0xFFFFu)),
                             f32_to_f16_sat(bf16_bits_to_f32(xbw[w] >> 16)));
        }
        if (v0)
          *reinterpret_cast<uint4*>(a.x16 + (size_t)t0 * a.H + 32 * q + k) =
              make_uint4(o0[0], o0[1], o0[2], o0[3]);
        if (v1)
          *reinterpret_cast<uint4*>(a.x16 + (size_t)t1 * a.H + 32 * q + k) =
              make_uint4(o1[0], o1[1], o1[2], o1[3]);
      }
      // step 2*sub uses words 0,1; step 2*sub+1 uses words 2,3
      const uint32_t Ah0[4] = {hi_a[0], hi_b[0], hi_a[1], hi_b[1]};
      const uint32_t Al0[4] = {lo_a[0], lo_b[0], lo_a[1], lo_b[1]};
      const uint32_t Ah1[4] = {hi_a[2], hi_b[2], hi_a[3], hi_b[3]};
      const uint32_t Al1[4] = {lo_a[2], lo_b[2], lo_a[3], lo_b[3]};
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const uint4 b = ldg_nc_v4(prow + (size_t)n * 8 * a.H + k);
        mma_bf16_16816(acc[n], Ah0, b.x, b.y);
        mma_bf16_16816(acc[n], Al0, b.x, b.y);
        mma_bf16_16816(acc[n], Ah1, b.z, b.w);
        mma_bf16_16816(acc[n], Al1, b.z, b.w);
      }
    }
  }

  // partial results of this K range
  float* pl = a.part_logits + (size_t)ks * a.T * kE;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int ecol = warp * 32 + n * 8 + 2 * q;
    if (v0) *reinterpret_cast<float2*>(pl + (size_t)t0 * kE + ecol) = make_float2(acc[n][0], acc[n][1]);
    if (v1) *reinterpret_cast<float2*>(pl + (size_t)t1 * kE + ecol) = make_float2(acc[n][2], acc[n][3]);
  }
  if (warp == 0) {
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
    if (q == 0) {
      if (v0) a.part_ss[(size_t)ks * a.T + t0] = ss0;
      if (v1) a.part_ss[(size_t)ks * a.T + t1] = ss1;
    }
  }

  __shared__ int s_last;
  if (a.ksplit > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(a.tile_counter + tile, 1);
      s_last = (prev == a.ksplit - 1);
      if (s_last) a.tile_counter[tile] = 0;  // leave the counter zero for the next call
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
  } else {
    __syncthreads();
  }

  // finisher: warp w handles tokens 4w .. 4w+3 of the tile
  for (int j = 0; j < 4; ++j) {
    const int t = tile * 16 + warp * 4 + j;
    if (t >= a.T) break;
    float ss = 0.f;
    for (int s = 0; s < a.ksplit; ++s) ss += __ldcg(a.part_ss + (size_t)s * a.T + t);
    const float inv_rms = 1.0f / sqrtf(ss / (float)a.H + a.eps);
    const float f = inv_rms * a.inv_sqrt_h;
    float lg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = lane + 32 * i;
      float raw = 0.f;
      for (int s = 0; s < a.ksplit; ++s) raw += __ldcg(a.part_logits + ((size_t)s * a.T + t) * kE + e);
      lg[i] = raw * f + (a.bias ? a.bias[e] : 0.f);
    }
    finish_token(a, t, lg);
  }
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  dim3 grid((a.T + 15) / 16, a.ksplit);
  route_kernel<<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
