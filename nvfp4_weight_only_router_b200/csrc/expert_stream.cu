// Persistent streaming grouped GEMV for decode (few tokens per expert).
//
// Decode reads each selected expert's NVFP4 bytes once and is bound by HBM
// bandwidth ("Gemma-4-26B-A4B-NVFP4-mlx", "Caveats": decode is
// expert-memory-bandwidth-bound; "Gemma 4 26B-A4B (MoE) - Core AI": only the
// routed experts are read).  To keep enough bytes in flight, one CTA per SM
// streams its share of the work items through a ring of shared-memory stages
// filled by 1-D bulk copies (TMA) that a producer warp issues ahead of the
// consumers, with mbarrier full/empty handshakes.
//
// Work item = 25,344 bytes of one active expert:
//   gate_up: 8 gate rows + the 8 matching up rows (16 x 1408 B codes,
//            16 x 176 B scales) -> 88 items per expert;
//   down:    64 output rows (64 x 352 B codes, 64 x 44 B scales)
//            -> 44 items per expert.
// Items are numbered expert-major over the active experts and each CTA takes
// a contiguous range, so consecutive items mostly share an expert and the
// activation fragments (x for gate_up, h for down; up to 16 tokens) stay in
// registers across them.
//
// Consumers: 8 warps.  MMA = m16n8k16 f16 -> f32 with weights dequantised in
// registers (hardware E2M1 -> f16x2, one f16x2 multiply by the E4M3 scale),
// tokens on N.  Within a 128-element K segment, lane quad q holds elements
// [32q, 32q+32); step j of the segment takes 32q+4j+{0,1} as the low k-pair
// and 32q+4j+{2,3} as the high k-pair for both operands.
//   gate_up: warp w takes K segments w, w+8, w+16 of all 16 rows; the eight
//            partial tiles meet in shared memory, where every consumer thread
//            adds up one (row, token) pair and applies
//            G * gelu_tanh(gate) * (G * up) -> h (f16).
//   down:    warp w takes rows 16*(w%4).. of the item and K half w/4
//            (segments 0-2 or 3-5); the two halves meet in shared memory and
//            every consumer thread finishes a (row pair, token pair): x G_d x
//            routing weight -> per-slot output (or the fp32 token
//            accumulator).
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kStages = 7;
constexpr int kItemBytes = 25344;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kNtMax = 2;  // 8-token n-tiles held in registers per pass
constexpr int kSegsPerWarp = 3;

constexpr int kGuItemsPerExpert = kI / 8;  // 88
constexpr int kDnItemsPerExpert = kH / 64; // 44

// gate_up stage layout
constexpr int kGuUpOff = 8 * kGuRowBytes;                 // 11264
constexpr int kGuGsOff = 16 * kGuRowBytes;                // 22528
constexpr int kGuUsOff = kGuGsOff + 8 * kGuScaleRow;      // 23936
// down stage layout
constexpr int kDnSOff = 64 * kDnRowBytes;                 // 22528

struct alignas(128) StreamSmem {
  uint8_t stage[kStages][kItemBytes];
  float4 red[2][kConsumerWarps][kNtMax][32];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort_flag;
  int consumed;
  int issued;
};

enum Kind { kGateUp = 0, kDown = 1 };

// acc[nt][w] += W(rows r, r+8; word w of one 32-element chunk) * X[nt] for
// the n-tiles nt < n_nt.  The weight chunk is dequantised once; the four
// words feed four independent accumulator chains so that consecutive MMAs do
// not wait on each other.
template <int NT>
__device__ __forceinline__ void mma_chunk_nt(float (&acc)[NT][4][4], const uint4& w0, const uint4& w1,
                                             uint32_t sc0, uint32_t sc1, const uint4 (&xb)[NT][4],
                                             int n_nt) {
  const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w};
  const uint32_t a1[4] = {w1.x, w1.y, w1.z, w1.w};
  const uint32_t s0lo = bcast_lo(sc0), s0hi = bcast_hi(sc0);
  const uint32_t s1lo = bcast_lo(sc1), s1hi = bcast_hi(sc1);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t f0[4], f1[4];
    e2m1x8_to_f16x2(a0[w], f0);
    e2m1x8_to_f16x2(a1[w], f1);
    const uint32_t s0 = w < 2 ? s0lo : s0hi, s1 = w < 2 ? s1lo : s1hi;
    const uint32_t A0[4] = {hmul2_u32(f0[0], s0), hmul2_u32(f1[0], s1), hmul2_u32(f0[1], s0),
                            hmul2_u32(f1[1], s1)};
    const uint32_t A1[4] = {hmul2_u32(f0[2], s0), hmul2_u32(f1[2], s1), hmul2_u32(f0[3], s0),
                            hmul2_u32(f1[3], s1)};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (nt < n_nt) {
        mma_f16_16816(acc[nt][w], A0, xb[nt][w].x, xb[nt][w].y);
        mma_f16_16816(acc[nt][w], A1, xb[nt][w].z, xb[nt][w].w);
      }
    }
  }
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) stream_gemv_kernel(ExpertArgs p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  StreamSmem& sm = *reinterpret_cast<StreamSmem*>(smem_raw);
  constexpr int per_expert = KIND == kGateUp ? kGuItemsPerExpert : kDnItemsPerExpert;

  const int n_act = p.meta[kMetaNAct];
  const int n_items = n_act * per_expert;
  const int begin = (int)(((long long)blockIdx.x * n_items) / gridDim.x);
  const int end = (int)(((long long)(blockIdx.x + 1) * n_items) / gridDim.x);
  if (begin >= end) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    sm.abort_flag = 0;
    sm.consumed = 0;
    sm.issued = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int j = begin; j < end; ++j) {
        const int it = j - begin, stage = it % kStages, round = it / kStages;
        if (it >= kStages && !mbar_wait_bounded(&sm.empty[stage], (round - 1) & 1)) {
          atomicExch(&sm.abort_flag, 1);
          record_status(p.status, kStatusTimeout);
          break;
        }
        if (*(volatile int*)&sm.abort_flag) break;
        const int a = j / per_expert, r = j % per_expert;
        const int e = p.meta[kMetaAct + a];
        uint8_t* dst = sm.stage[stage];
        mbar_arrive_expect_tx(&sm.full[stage], kItemBytes);
        if (KIND == kGateUp) {
          const size_t rowG = (size_t)e * (2 * kI) + 8 * r, rowU = rowG + kI;
          bulk_g2s(dst, p.gu_q + rowG * kGuRowBytes, 8 * kGuRowBytes, &sm.full[stage]);
          bulk_g2s(dst + kGuUpOff, p.gu_q + rowU * kGuRowBytes, 8 * kGuRowBytes, &sm.full[stage]);
          bulk_g2s(dst + kGuGsOff, p.gu_s + rowG * kGuScaleRow, 8 * kGuScaleRow, &sm.full[stage]);
          bulk_g2s(dst + kGuUsOff, p.gu_s + rowU * kGuScaleRow, 8 * kGuScaleRow, &sm.full[stage]);
        } else {
          const size_t row = (size_t)e * kH + 64 * r;
          bulk_g2s(dst, p.dn_q + row * kDnRowBytes, 64 * kDnRowBytes, &sm.full[stage]);
          bulk_g2s(dst + kDnSOff, p.dn_s + row * kDnScaleRow, 64 * kDnScaleRow, &sm.full[stage]);
        }
        ++issued;
      }
      sm.issued = issued;
    }
    goto join;
  }

  // -------------------------------------------------------------- consumers
  {
  const int g = lane >> 2, q = lane & 3;
  int cached_e = -1, cached_grp = -1;
  uint4 xb[kNtMax][kSegsPerWarp][4];
  // the K segments of this warp
  int segs[kSegsPerWarp];
  int mt = 0;
  if (KIND == kGateUp) {
#pragma unroll
    for (int i = 0; i < kSegsPerWarp; ++i) segs[i] = warp + 8 * i;  // < 22 valid
  } else {
    mt = warp & 3;
#pragma unroll
    for (int i = 0; i < kSegsPerWarp; ++i) segs[i] = (warp >> 2) * 3 + i;  // < 6 valid
  }
  const int seg_lim = KIND == kGateUp ? kGuSegs : kDnSegs;

  int round_ctr = 0;  // reduction rounds (one per item and token group)
  for (int j = begin; j < end; ++j) {
    const int it = j - begin, stage = it % kStages;
    const int a = j / per_expert, r = j % per_expert;
    const int e = p.meta[kMetaAct + a];
    const int off = p.meta[kMetaOffsets + e];
    const int cnt = p.meta[kMetaOffsets + e + 1] - off;
    const int n_grp = (cnt + 8 * kNtMax - 1) / (8 * kNtMax);
    const uint8_t* st = sm.stage[stage];
    bool waited = false, data_ok = true;

    for (int grp = 0; grp < n_grp; ++grp) {
      const int n0 = grp * 8 * kNtMax;
      const int n_nt = min(kNtMax, (cnt - n0 + 7) / 8);
      if (e != cached_e || grp != cached_grp) {
        // activation fragments of this expert / token group (L2-resident)
#pragma unroll
        for (int nt = 0; nt < kNtMax; ++nt) {
          const int n = n0 + nt * 8 + g;
          const bool has = nt < n_nt && n < cnt;
          const __half* row;
          if (KIND == kGateUp) {
            int tok = has ? p.sorted_slot[off + n] / kTopK : 0;
            if (tok < 0 || tok >= p.T) {
              record_status(p.status, kStatusDevice);
              tok = 0;
            }
            row = p.x16 + (size_t)tok * kH + q * 32;
          } else {
            row = p.h + (size_t)(off + (has ? n : 0)) * kI + q * 32;
          }
#pragma unroll
          for (int i = 0; i < kSegsPerWarp; ++i) {
            const bool ok = has && segs[i] < seg_lim && segs[i] * kSegK + q * 32 < (KIND == kGateUp ? kH : kI);
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4)
              xb[nt][i][w4] = ok ? __ldg(reinterpret_cast<const uint4*>(row + segs[i] * kSegK) + w4)
                                 : make_uint4(0, 0, 0, 0);
          }
        }
        cached_e = e;
        cached_grp = grp;
      }
      if (!waited) {
        // A wait that gives up marks the CTA aborted; the warp still takes
        // part in the barrier below so that no other warp waits for it.
        if (!mbar_wait_bounded(&sm.full[stage], (it / kStages) & 1)) {
          atomicExch(&sm.abort_flag, 1);
          record_status(p.status, kStatusTimeout);
          data_ok = false;
        }
        waited = true;
      }
      float acc[kNtMax][4][4];
#pragma unroll
      for (int nt = 0; nt < kNtMax; ++nt)
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[nt][w][c] = 0.f;

#pragma unroll
      for (int i = 0; i < kSegsPerWarp; ++i) {
        const int seg = segs[i];
        if (seg >= seg_lim || !data_ok) continue;  // uniform across the warp
        uint4 w0, w1;
        uint32_t s0, s1;
        if (KIND == kGateUp) {
          w0 = lds_v4(st + g * kGuRowBytes + seg * 64 + q * 16);
          w1 = lds_v4(st + kGuUpOff + g * kGuRowBytes + seg * 64 + q * 16);
          s0 = e4m3x2_to_f16x2(lds_u16(st + kGuGsOff + g * kGuScaleRow + seg * 8 + 2 * q));
          s1 = e4m3x2_to_f16x2(lds_u16(st + kGuUsOff + g * kGuScaleRow + seg * 8 + 2 * q));
        } else {
          // lanes past K = 704 (the idle half of the last segment) keep zero
          // operands: every lane of the warp must still issue the MMA
          w0 = w1 = make_uint4(0, 0, 0, 0);
          s0 = s1 = 0;
          if (seg * kSegK + q * 32 < kI) {
            const int r0 = 16 * mt + g;
            w0 = lds_v4(st + r0 * kDnRowBytes + seg * 64 + q * 16);
            w1 = lds_v4(st + (r0 + 8) * kDnRowBytes + seg * 64 + q * 16);
            s0 = e4m3x2_to_f16x2(lds_u16(st + kDnSOff + r0 * kDnScaleRow + seg * 8 + 2 * q));
            s1 = e4m3x2_to_f16x2(lds_u16(st + kDnSOff + (r0 + 8) * kDnScaleRow + seg * 8 + 2 * q));
          }
        }
        uint4 xs[kNtMax][4];
#pragma unroll
        for (int nt = 0; nt < kNtMax; ++nt)
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) xs[nt][w4] = xb[nt][i][w4];
        mma_chunk_nt<kNtMax>(acc, w0, w1, s0, s1, xs, n_nt);
      }
      if (grp == n_grp - 1) {
        // this warp is done with the stage's bytes
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
      }

      // cross-warp reduction and epilogue, spread over all consumer threads
      const int par = round_ctr & 1;
#pragma unroll
      for (int nt = 0; nt < kNtMax; ++nt) {
        float4 v;
        v.x = acc[nt][0][0] + acc[nt][1][0] + acc[nt][2][0] + acc[nt][3][0];
        v.y = acc[nt][0][1] + acc[nt][1][1] + acc[nt][2][1] + acc[nt][3][1];
        v.z = acc[nt][0][2] + acc[nt][1][2] + acc[nt][2][2] + acc[nt][3][2];
        v.w = acc[nt][0][3] + acc[nt][1][3] + acc[nt][2][3] + acc[nt][3][3];
        sm.red[par][warp][nt][lane] = v;
      }
      named_bar_sync(1, kConsumerWarps * 32);
      // every consumer warp reads the flag after the same barrier and leaves together
      if (*(volatile int*)&sm.abort_flag) goto done;
      const int t = threadIdx.x;  // 0 .. 255
      if (KIND == kGateUp) {
        // thread -> (n-tile, lane L = 4 row + quad, token parity c): one h value
        const int nt = t >> 6, L = (t >> 1) & 31, c = t & 1;
        if (nt < n_nt) {
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float4 o = sm.red[par][w][nt][L];
            gs += c ? o.y : o.x;
            us += c ? o.w : o.z;
          }
          const int col = n0 + nt * 8 + 2 * (L & 3) + c;
          if (col < cnt) {
            const float G = p.gu_g[e];
            p.h[(size_t)(off + col) * kI + 8 * r + (L >> 2)] = f32_to_f16_sat(gelu_tanh(G * gs) * (G * us));
          }
        }
      } else {
        // thread -> (n-tile, m-tile, lane): rows 16 m + L/4 (+8), tokens 2(L%4) (+1)
        const int nt = t >> 7, mtile = (t >> 5) & 3, L = t & 31;
        if (nt < n_nt) {
          float4 v = sm.red[par][mtile][nt][L];
          const float4 o = sm.red[par][mtile + 4][nt][L];
          v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
          const float vv[4] = {v.x, v.y, v.z, v.w};
          const float G = p.dn_g[e];
          const int row0 = 64 * r + 16 * mtile + (L >> 2);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col = n0 + nt * 8 + 2 * (L & 3) + c;
            if (col >= cnt) continue;
            const int pos = off + col;
            const int slot = p.sorted_slot[pos];
            const float wgt = p.wts[slot] * G;
            const float o0 = vv[c] * wgt, o1 = vv[2 + c] * wgt;
            p.obuf[(size_t)pos * kH + row0] = o0;
            p.obuf[(size_t)pos * kH + row0 + 8] = o1;
          }
        }
      }
      ++round_ctr;
    }
    if (warp == 0 && lane == 0) *(volatile int*)&sm.consumed = it + 1;
  }
  }
done:
join:
  // After an abort, wait (bounded) for copies that were issued but not
  // consumed, so that none lands after the CTA has exited.
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort_flag) {
    for (int it = sm.consumed; it < sm.issued; ++it)
      mbar_wait_bounded(&sm.full[it % kStages], (it / kStages) & 1, kAbortDrainNs);
  }
}

template <int KIND>
cudaError_t launch_stream(const ExpertArgs& a, cudaStream_t st) {
  static int configured_dev = -1;  // attribute set for this device
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int smem = (int)sizeof(StreamSmem);
  if (configured_dev != dev) {
    err = cudaFuncSetAttribute(stream_gemv_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  int sms = 0;
  err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  stream_gemv_kernel<KIND><<<sms, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up_stream(const ExpertArgs& a, cudaStream_t st) { return launch_stream<kGateUp>(a, st); }
cudaError_t launch_down_stream(const ExpertArgs& a, cudaStream_t st) { return launch_stream<kDown>(a, st); }

}  // namespace nvfp4moe
