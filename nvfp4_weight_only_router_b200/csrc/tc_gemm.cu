// Grouped NVFP4 expert GEMMs on the 5th-generation tensor cores (tcgen05) for
// many tokens per expert (prefill).
//
// Per expert e ("Gemma 4 26B-A4B (MoE) - Core AI": GELU-tanh gated experts,
// fused gate||up rows with gate first; weights E2M1 x E4M3 x FP32 per the
// NVFP4A16 card, "Quantization details"):
//   gate_up:  h[tok, j] = gelu_tanh(G_gu * x.Wg[j]) * (G_gu * x.Wu[j])
//   down:     y[tok, n] += w_slot * G_d * h.Wd[n]        (fp32 accumulator)
// Work tile = (expert, 128 of its tokens, 256 weight rows), K in chunks of 64:
//   A = the tile's 128 activation rows (x in f16, gathered through the slot
//       permutation; or h rows, contiguous per expert), K-major;
//   B = 256 weight rows dequantised to f16 (e2m1 * e4m3 is exact in f16),
//       K-major; a gate_up tile holds 128 gate rows then the 128 matching up
//       rows (the last tile 64 + 64), so each accumulator row carries both
//       halves of its GELU gate;
//   D = 128 x 256 fp32 in tensor memory (two buffers, so the epilogue of one
//       tile overlaps the main loop of the next).
// Warp roles (12 warps): 0 activation producer (cp.async, swizzled),
// 1 weight producer (cp.async of packed codes and scales), 2 MMA issuer
// (one thread), 4-7 epilogue (tensor memory -> registers -> global),
// 8-11 dequantisation (packed codes -> f16 B tile).  Stages are handed over
// with mbarriers; MMA completion is signalled by tcgen05.commit.
// Every wait is bounded in wall time; a wait that gives up records a timeout
// status and the CTA drains its copies and MMAs, frees its tensor memory and
// exits.
#include "tc_common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kBM = 128;       // tokens per tile (MMA M)
constexpr int kBN = 256;       // weight rows per tile (MMA N)
constexpr int kBK = 64;        // K per stage (128 bytes of f16 per row)
constexpr int kNS = 3;         // pipeline stages
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kWarpProdX = 0, kWarpProdW = 1, kWarpMma = 2, kWarpEpi0 = 4, kWarpDeq0 = 8;
constexpr int kTmemCols = 512;

enum Kind { kGateUp = 0, kDown = 1 };

struct alignas(1024) TcSmem {
  uint8_t a[kNS][kBM * 128];     // activation tiles (1024-aligned, SW128)
  uint8_t b[kNS][kBN * 128];     // dequantised weight tiles (SW128)
  uint8_t wraw[kNS][kBN * 32];   // packed codes: 64 K per row = 32 bytes
  uint8_t wsc[kNS][kBN * 4];     // E4M3 scales: 4 per row
  uint64_t a_full[kNS], w_full[kNS], b_full[kNS], empty[kNS];
  uint64_t tfull[2], tempty[2], final_bar;
  uint32_t taddr;
  int mt_prefix[kE + 1];         // prefix of per-expert m-tile counts
  int abort_flag;
};

template <int KIND>
struct Geometry {
  static constexpr int NJ = KIND == kGateUp ? 6 : 11;            // n-tiles per m-tile
  static constexpr int KC = (KIND == kGateUp ? kH : kI) / kBK;   // K chunks: 44 or 11
  __device__ static int bn(int j) { return (KIND == kGateUp && j == 5) ? 128 : 256; }
};

struct TileInfo {
  int e, i, j, off, cnt;
};

template <int KIND>
__device__ __forceinline__ TileInfo decode_tile(const TcSmem& sm, const int* meta, int t) {
  constexpr int NJ = Geometry<KIND>::NJ;
  const int mt = t / NJ;
  int lo = 0, hi = kE - 1;  // largest e with mt_prefix[e] <= mt (and a non-empty range)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sm.mt_prefix[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.e = lo;
  ti.i = mt - sm.mt_prefix[lo];
  ti.j = t % NJ;
  ti.off = meta[kMetaOffsets + lo];
  ti.cnt = meta[kMetaOffsets + lo + 1] - ti.off;
  return ti;
}

__device__ __forceinline__ bool wait_or_abort(TcSmem& sm, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_wait_bounded(bar, parity)) return true;
  atomicExch(&sm.abort_flag, 1);
  record_status(status, kStatusTimeout);
  return false;
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(ExpertArgs p) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using Geo = Geometry<KIND>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- set-up
  if (warp == 0) {
    // m-tile prefix over experts (4 experts per lane)
    int c[4], run = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 4 * lane + k;
      const int cnt = p.meta[kMetaOffsets + e + 1] - p.meta[kMetaOffsets + e];
      c[k] = (cnt + kBM - 1) / kBM;
      run += c[k];
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int base = incl - run;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      sm.mt_prefix[4 * lane + k] = base;
      base += c[k];
    }
    if (lane == 31) sm.mt_prefix[kE] = incl;
    if (lane == 0) {
      for (int s = 0; s < kNS; ++s) {
        mbar_init(&sm.a_full[s], 32);
        mbar_init(&sm.w_full[s], 32);
        mbar_init(&sm.b_full[s], 128);
        mbar_init(&sm.empty[s], 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.tfull[b], 1);
        mbar_init(&sm.tempty[b], 128);
      }
      mbar_init(&sm.final_bar, 1);
      sm.abort_flag = 0;
      fence_mbar_init();
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(&sm.taddr, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = sm.taddr;
  const int n_tiles = Geo::NJ * sm.mt_prefix[kE];

  if (warp == kWarpProdX) {
    // ------------------------------------------------- activation producer
    uint32_t kiter = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile<KIND>(sm, p.meta, t);
      const __half* src[4];
      bool valid[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int m = lane + 32 * r;
        const int n = ti.i * kBM + m;
        valid[r] = n < ti.cnt;
        const int pos = ti.off + (valid[r] ? n : 0);
        if (KIND == kGateUp) {
          int tok = valid[r] ? p.sorted_slot[pos] / kTopK : 0;
          if (tok < 0 || tok >= p.T) {
            record_status(p.status, kStatusDevice);
            tok = 0;
            valid[r] = false;
          }
          src[r] = p.x16 + (size_t)tok * kH;
        } else {
          src[r] = p.h + (size_t)pos * kI;
        }
      }
      for (int kc = 0; kc < Geo::KC; ++kc, ++kiter) {
        const int s = kiter % kNS, use = kiter / kNS;
        if (use > 0 && !wait_or_abort(sm, &sm.empty[s], (use - 1) & 1, p.status)) { ok = false; break; }
        const uint32_t a_base = smem_u32(sm.a[s]);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int m = lane + 32 * r;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t dst = a_base + sw128_offset(m, c);
            if (valid[r]) cp_async16(dst, src[r] + kc * kBK + c * 8);
            else sts_v4(dst, make_uint4(0, 0, 0, 0));
          }
        }
        fence_proxy_async_smem();  // the zero-filled rows are generic-proxy writes
        cp_async_arrive(&sm.a_full[s]);
      }
    }
    cp_async_wait_all();
  } else if (warp == kWarpProdW) {
    // ----------------------------------------------------- weight producer
    const uint8_t* q = KIND == kGateUp ? p.gu_q : p.dn_q;
    const uint8_t* sc = KIND == kGateUp ? p.gu_s : p.dn_s;
    constexpr int row_bytes = KIND == kGateUp ? kGuRowBytes : kDnRowBytes;
    constexpr int srow = KIND == kGateUp ? kGuScaleRow : kDnScaleRow;
    uint32_t kiter = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile<KIND>(sm, p.meta, t);
      const int bn = Geo::bn(ti.j);
      size_t rows[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = lane + 32 * u;
        size_t row;
        if (KIND == kGateUp) {
          const int half = bn / 2;
          row = (size_t)ti.e * (2 * kI) + (r < half ? ti.j * 128 + r : kI + ti.j * 128 + (r - half));
        } else {
          row = (size_t)ti.e * kH + ti.j * 256 + r;
        }
        rows[u] = row;
      }
      for (int kc = 0; kc < Geo::KC; ++kc, ++kiter) {
        const int s = kiter % kNS, use = kiter / kNS;
        if (use > 0 && !wait_or_abort(sm, &sm.empty[s], (use - 1) & 1, p.status)) { ok = false; break; }
        const uint32_t wr = smem_u32(sm.wraw[s]), ws = smem_u32(sm.wsc[s]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int r = lane + 32 * u;
          if (r < bn) {
            const uint8_t* g = q + rows[u] * row_bytes + kc * 32;
            cp_async16(wr + r * 32, g);
            cp_async16(wr + r * 32 + 16, g + 16);
            cp_async4(ws + r * 4, sc + rows[u] * srow + kc * 4);
          }
        }
        cp_async_arrive(&sm.w_full[s]);
      }
    }
    cp_async_wait_all();
  } else if (warp >= kWarpDeq0) {
    // ------------------------------------------------------ dequantisation
    const int dt = threadIdx.x - kWarpDeq0 * 32;  // 0..127
    uint32_t kiter = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile<KIND>(sm, p.meta, t);
      const int bn = Geo::bn(ti.j);
      for (int kc = 0; kc < Geo::KC; ++kc, ++kiter) {
        const int s = kiter % kNS, use = kiter / kNS;
        if (!wait_or_abort(sm, &sm.w_full[s], use & 1, p.status)) { ok = false; break; }
        const uint8_t* wraw = sm.wraw[s];
        const uint32_t b_base = smem_u32(sm.b[s]);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = dt + 128 * rr;
          if (r >= bn) continue;
          const uint4 w0 = lds_v4(wraw + r * 32), w1 = lds_v4(wraw + r * 32 + 16);
          uint32_t scw;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(scw) : "r"(smem_u32(sm.wsc[s] + r * 4)));
          const uint32_t s01 = e4m3x2_to_f16x2((uint16_t)(scw & 0xFFFFu));
          const uint32_t s23 = e4m3x2_to_f16x2((uint16_t)(scw >> 16));
          const uint32_t sb[4] = {bcast_lo(s01), bcast_hi(s01), bcast_lo(s23), bcast_hi(s23)};
          const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            uint32_t f[4];
            e2m1x8_to_f16x2(words[w], f);
            const uint32_t scl = sb[w >> 1];
            sts_v4(b_base + sw128_offset(r, w),
                   make_uint4(hmul2_u32(f[0], scl), hmul2_u32(f[1], scl), hmul2_u32(f[2], scl),
                              hmul2_u32(f[3], scl)));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.b_full[s]);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t kiter = 0, titer = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
        const TileInfo ti = decode_tile<KIND>(sm, p.meta, t);
        const int bn = Geo::bn(ti.j);
        const uint32_t idesc = make_idesc_f16(kBM, bn);
        const int b = titer & 1, tuse = titer >> 1;
        if (tuse > 0 && !wait_or_abort(sm, &sm.tempty[b], (tuse - 1) & 1, p.status)) break;
        tc_fence_after();
        const uint32_t d = taddr + (uint32_t)(b * kBN);
        for (int kc = 0; kc < Geo::KC; ++kc, ++kiter) {
          const int s = kiter % kNS, use = kiter / kNS;
          if (!wait_or_abort(sm, &sm.a_full[s], use & 1, p.status) ||
              !wait_or_abort(sm, &sm.b_full[s], use & 1, p.status)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t ad = make_sw128_desc(smem_u32(sm.a[s]));
          const uint64_t bd = make_sw128_desc(smem_u32(sm.b[s]));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_f16(d, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kc | kk) != 0);
          tc_commit(&sm.empty[s]);
        }
        if (!ok) break;
        tc_commit(&sm.tfull[b]);
      }
      // all MMAs issued by this thread have completed before the CTA moves on
      tc_commit(&sm.final_bar);
      mbar_wait_bounded(&sm.final_bar, 0);
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp - kWarpEpi0;   // tensor-memory lanes 32*quarter ..
    const int m = quarter * 32 + lane;       // tile row = token index in the tile
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++titer) {
      const TileInfo ti = decode_tile<KIND>(sm, p.meta, t);
      const int bn = Geo::bn(ti.j);
      const int b = titer & 1, tuse = titer >> 1;
      if (!wait_or_abort(sm, &sm.tfull[b], tuse & 1, p.status)) break;
      tc_fence_after();
      const int n = ti.i * kBM + m;
      const bool valid = n < ti.cnt;
      const int pos = ti.off + (valid ? n : 0);
      const uint32_t trow = taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * kBN);
      if (KIND == kGateUp) {
        const int half = bn / 2;
        const float G = p.gu_g[ti.e];
        for (int cc = 0; cc < half / 32; ++cc) {
          float g[32], u[32];
          tmem_ld32(trow + cc * 32, g);
          tmem_ld32(trow + half + cc * 32, u);
          if (valid) {
            uint32_t hv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              hv[k] = pack_f16x2(f32_to_f16_sat(gelu_tanh(G * g[2 * k]) * (G * u[2 * k])),
                                 f32_to_f16_sat(gelu_tanh(G * g[2 * k + 1]) * (G * u[2 * k + 1])));
            uint4* dst = reinterpret_cast<uint4*>(p.h + (size_t)pos * kI + ti.j * 128 + cc * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
          }
        }
      } else {
        int slot = 0;
        float wgt = 0.f;
        if (valid) {
          slot = p.sorted_slot[pos];
          wgt = p.wts[slot] * p.dn_g[ti.e];
        }
        float* yrow = p.yacc + (size_t)(slot / kTopK) * kH + ti.j * 256;
        for (int cc = 0; cc < 8; ++cc) {
          float v[32];
          tmem_ld32(trow + cc * 32, v);
          if (valid) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              red_add_v4(yrow + cc * 32 + 4 * k, v[4 * k] * wgt, v[4 * k + 1] * wgt, v[4 * k + 2] * wgt,
                         v[4 * k + 3] * wgt);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.tempty[b]);
    }
  }

  // ------------------------------------------------------------- tear-down
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

template <int KIND>
cudaError_t launch_tc(const ExpertArgs& a, cudaStream_t st) {
  static int configured_dev = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int smem = (int)sizeof(TcSmem) + 1024;  // + alignment slack
  if (configured_dev != dev) {
    err = cudaFuncSetAttribute(tc_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  int sms = 0;
  err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  tc_gemm_kernel<KIND><<<sms, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up_tc(const ExpertArgs& a, cudaStream_t st) { return launch_tc<kGateUp>(a, st); }
cudaError_t launch_down_tc(const ExpertArgs& a, cudaStream_t st) { return launch_tc<kDown>(a, st); }

}  // namespace nvfp4moe
