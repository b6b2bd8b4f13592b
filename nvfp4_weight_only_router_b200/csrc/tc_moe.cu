// Grouped NVFP4 expert GEMMs on the 5th-generation tensor cores with the
// dequantised weights in tensor memory.
//
// Per expert e ("Gemma 4 26B-A4B (MoE) - Core AI": GELU-tanh gated experts,
// fused gate||up rows with gate first; weights E2M1 x E4M3 x FP32 per the
// NVFP4A16 card, "Quantization details"):
//   gate_up:  h[tok, j] = gelu_tanh(G_gu * Wg[j].x) * (G_gu * Wu[j].x)
//   down:     o[slot, n] = w_slot * G_d * Wd[n].h          (per-slot rows)
//
// Work tile = (expert, NT of its tokens, 128 weight rows), K in chunks of 64.
//   D[128 rows x NT tokens] (fp32, tensor memory) += A x B^T with
//   A = 128 weight rows x 64 K dequantised to f16 by the dequant warps and
//       stored straight into tensor memory (tcgen05.st): e2m1 * e4m3 is
//       exact in f16, and the converted operand never touches shared memory;
//   B = NT activation rows x 64 K, f16, 128B-swizzled in shared memory by
//       one 2-D TMA box per chunk (activations are in expert-sorted order).
// A gate_up tile interleaves 64 gate rows with the 64 matching up rows
// (A row 2r = gate r, 2r+1 = up r), so the GELU gate of a hidden unit is a
// shuffle between adjacent lanes.
//
// Warp roles (16 warps): 0 TMA producer (activation box, packed-code boxes,
// the tile's E4M3 scales by a bulk copy), 1 MMA issuer (one thread),
// 4-7 epilogue (tensor memory -> registers -> global), 8-15 dequantisation
// (warp w owns tensor-memory lanes 32(w%4).. and K half (w-8)/4).
// Every wait is bounded in wall time; a wait that gives up records a timeout
// status, and the CTA drains its copies and MMAs, frees its tensor memory and
// exits.
#include "tc_common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kRows = 128;      // weight rows per tile (MMA M)
constexpr int kBK = 64;         // K per chunk
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpEpi0 = 4, kWarpDeq0 = 8;
constexpr int kTmemCols = 512;

enum Kind { kGateUp = 0, kDown = 1 };

template <int KIND, int NT>
struct Cfg {
  static constexpr int NJ = KIND == kGateUp ? (2 * kI) / kRows : kH / kRows;  // 11 or 22 row tiles
  static constexpr int KC = (KIND == kGateUp ? kH : kI) / kBK;               // 44 or 11 chunks
  static constexpr int SROW = KIND == kGateUp ? kGuScaleRow : kDnScaleRow;   // scale bytes per row
  static constexpr int SC_BYTES = kRows * SROW;                             // scales of a tile
  static constexpr int X_BYTES = NT * 128;
  static constexpr int CODE_BYTES = kRows * 32;
  // epilogue staging per warp: gate_up h values (NT tokens x 16 units, f16),
  // down one 16-token chunk of 32 rows (fp32)
  static constexpr int STAGE_BYTES = KIND == kGateUp ? NT * 32 : 16 * 32 * 4;
  // load stages: as many as fit next to the scale buffers and the staging
  static constexpr int NS_RAW = (206 * 1024 - 2 * SC_BYTES - 4 * STAGE_BYTES) / (X_BYTES + CODE_BYTES);
  static constexpr int NS = NS_RAW > 24 ? 24 : NS_RAW;
  static constexpr int NA = 4;                                             // A stages (32 columns each)
  // independent accumulators per tile: small-N MMAs into one accumulator
  // would wait on each other, so the K sub-steps rotate over NACC of them
  static constexpr int NACC = NT <= 16 ? 4 : (NT <= 64 ? 2 : 1);
  static constexpr int ND = (2 * NACC * NT + NA * 32 <= kTmemCols) ? 2 : 1; // accumulator buffers
  static constexpr int A_COL0 = ND * NACC * NT;                           // first A-stage column
  static_assert(A_COL0 + NA * 32 <= kTmemCols, "tensor memory budget");
};

template <int KIND, int NT>
struct alignas(1024) MoeSmem {
  using C = Cfg<KIND, NT>;
  uint8_t x[C::NS][C::X_BYTES];          // B tiles (SW128, 1024-aligned since X_BYTES % 1024 == 0)
  uint8_t code[C::NS][C::CODE_BYTES];    // packed codes: 128 rows x 32 bytes
  uint8_t sc[2][C::SC_BYTES];            // E4M3 scales of a tile (rows in tile-row order)
  uint8_t stage[4][C::STAGE_BYTES];      // epilogue staging, one per epilogue warp
  uint64_t full[C::NS], empty[C::NS];
  uint64_t a_full[C::NA], a_empty[C::NA];
  uint64_t sc_full[2], sc_empty[2];
  uint64_t d_full[2], d_empty[2];
  uint64_t fin;
  uint32_t taddr;
  int mt_prefix[kE + 1];
  int abort_flag;
  int issued_chunks, issued_tiles;       // producer progress (for draining after an abort)
  float wslot[4][NT];                    // down: routing weight x G_d per token (one copy per epilogue warp)
};

struct TileInfo {
  int e, i, j, off, cnt;
};

template <int KIND, int NT>
__device__ __forceinline__ TileInfo decode_tile(const MoeSmem<KIND, NT>& sm, const int* meta, int t) {
  constexpr int NJ = Cfg<KIND, NT>::NJ;
  const int mt = t / NJ;
  int lo = 0, hi = kE - 1;  // largest e with mt_prefix[e] <= mt
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

template <int KIND, int NT>
__device__ __forceinline__ bool wait_or_abort(MoeSmem<KIND, NT>& sm, uint64_t* bar, uint32_t parity,
                                              int* status) {
  if (mbar_wait_bounded(bar, parity)) return true;
  atomicExch(&sm.abort_flag, 1);
  record_status(status, kStatusTimeout);
  return false;
}

// global weight row of tile row L (0..127)
template <int KIND>
__device__ __forceinline__ int tile_row(int e, int j, int L) {
  if (KIND == kGateUp) return e * (2 * kI) + (L & 1) * kI + j * 64 + (L >> 1);
  return e * kH + j * kRows + L;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int KIND, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    tc_moe_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  ExpertArgs p) {
  using C = Cfg<KIND, NT>;
  using Smem = MoeSmem<KIND, NT>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- set-up
  if (warp == 0) {
    int c[4], run = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 4 * lane + k;
      const int cnt = p.meta[kMetaOffsets + e + 1] - p.meta[kMetaOffsets + e];
      c[k] = (cnt + NT - 1) / NT;
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
      for (int s = 0; s < C::NS; ++s) {
        mbar_init(&sm.full[s], 1);
        mbar_init(&sm.empty[s], 1);
      }
      for (int a = 0; a < C::NA; ++a) {
        mbar_init(&sm.a_full[a], 8);    // one arrival per dequant warp
        mbar_init(&sm.a_empty[a], 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.sc_full[b], 1);
        mbar_init(&sm.sc_empty[b], 8);
        mbar_init(&sm.d_full[b], 1);
        mbar_init(&sm.d_empty[b], 4);   // one arrival per epilogue warp
      }
      mbar_init(&sm.fin, 1);
      sm.abort_flag = 0;
      sm.issued_chunks = 0;
      sm.issued_tiles = 0;
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
  const int n_tiles = C::NJ * sm.mt_prefix[kE];

  if (warp == kWarpProd) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint8_t* sc_src = KIND == kGateUp ? p.gu_s : p.dn_s;
      uint32_t kiter = 0, titer = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
        const TileInfo ti = decode_tile<KIND, NT>(sm, p.meta, t);
        const int xrow = ti.off + ti.i * NT;
        // the tile's scales: gate_up = two runs of 64 rows (gate, up), down = one run of 128
        const int sb = titer & 1, suse = titer >> 1;
        if (suse > 0 && !wait_or_abort(sm, &sm.sc_empty[sb], (suse - 1) & 1, p.status)) break;
        mbar_arrive_expect_tx(&sm.sc_full[sb], C::SC_BYTES);
        if (KIND == kGateUp) {
          const int g0 = tile_row<KIND>(ti.e, ti.j, 0), u0 = tile_row<KIND>(ti.e, ti.j, 1);
          bulk_g2s_u32(smem_u32(sm.sc[sb]), sc_src + (size_t)g0 * C::SROW, 64 * C::SROW, &sm.sc_full[sb]);
          bulk_g2s_u32(smem_u32(sm.sc[sb]) + 64 * C::SROW, sc_src + (size_t)u0 * C::SROW, 64 * C::SROW,
                       &sm.sc_full[sb]);
        } else {
          const int r0 = tile_row<KIND>(ti.e, ti.j, 0);
          bulk_g2s_u32(smem_u32(sm.sc[sb]), sc_src + (size_t)r0 * C::SROW, C::SC_BYTES, &sm.sc_full[sb]);
        }
        for (int kc = 0; kc < C::KC; ++kc, ++kiter) {
          const int s = kiter % C::NS, use = kiter / C::NS;
          if (use > 0 && !wait_or_abort(sm, &sm.empty[s], (use - 1) & 1, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[s], C::X_BYTES + C::CODE_BYTES);
          tma_load_2d(smem_u32(sm.x[s]), &tm_x, kc * kBK, xrow, &sm.full[s]);
          // packed codes: tile rows 0..63 and 64..127 (gate_up: gate rows, up rows)
          const int ra = KIND == kGateUp ? tile_row<KIND>(ti.e, ti.j, 0) : tile_row<KIND>(ti.e, ti.j, 0);
          const int rb = KIND == kGateUp ? tile_row<KIND>(ti.e, ti.j, 1) : tile_row<KIND>(ti.e, ti.j, 64);
          tma_load_2d(smem_u32(sm.code[s]), &tm_w, kc * 32, ra, &sm.full[s]);
          tma_load_2d(smem_u32(sm.code[s]) + 64 * 32, &tm_w, kc * 32, rb, &sm.full[s]);
          sm.issued_chunks = kiter + 1;
        }
        sm.issued_tiles = titer + 1;
      }
    }
  } else if (warp >= kWarpDeq0) {
    // ------------------------------------------------------ dequantisation
    const int quarter = warp & 3, khalf = (warp - kWarpDeq0) >> 2;
    const int L = quarter * 32 + lane;  // tensor-memory lane = A row
    // code / scale row in shared memory: gate_up stores gate rows 0..63 then up rows 64..127
    const int crow = KIND == kGateUp ? ((L & 1) * 64 + (L >> 1)) : L;
    uint32_t kiter = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
      const int sb = titer & 1, suse = titer >> 1;
      if (!wait_or_abort(sm, &sm.sc_full[sb], suse & 1, p.status)) break;
      const uint8_t* scrow = sm.sc[sb] + crow * C::SROW;
      for (int kc = 0; kc < C::KC; ++kc, ++kiter) {
        const int s = kiter % C::NS, use = kiter / C::NS;
        const int a = kiter % C::NA, ause = kiter / C::NA;
        if (!wait_or_abort(sm, &sm.full[s], use & 1, p.status)) { ok = false; break; }
        if (ause > 0 && !wait_or_abort(sm, &sm.a_empty[a], (ause - 1) & 1, p.status)) { ok = false; break; }
        const uint4 w = lds_v4(sm.code[s] + crow * 32 + khalf * 16);   // 32 K of this row
        const uint32_t s2 = e4m3x2_to_f16x2(lds_u16(scrow + kc * 4 + khalf * 2));
        const uint32_t slo = bcast_lo(s2), shi = bcast_hi(s2);
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
        uint32_t v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t f[4];
          e2m1x8_to_f16x2(words[q], f);
          const uint32_t scl = q < 2 ? slo : shi;
#pragma unroll
          for (int i = 0; i < 4; ++i) v[4 * q + i] = hmul2_u32(f[i], scl);
        }
        tmem_st16(taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(C::A_COL0 + a * 32 + khalf * 16), v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.a_full[a]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sc_empty[sb]);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc_f16(kRows, NT);
      uint32_t kiter = 0, titer = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
        const int db = titer % C::ND, duse = titer / C::ND;
        if (duse > 0 && !wait_or_abort(sm, &sm.d_empty[db], (duse - 1) & 1, p.status)) break;
        tc_fence_after();
        const uint32_t d = taddr + (uint32_t)(db * C::NACC * NT);
        for (int kc = 0; kc < C::KC; ++kc, ++kiter) {
          const int s = kiter % C::NS, use = kiter / C::NS;
          const int a = kiter % C::NA, ause = kiter / C::NA;
          if (!wait_or_abort(sm, &sm.full[s], use & 1, p.status) ||
              !wait_or_abort(sm, &sm.a_full[a], ause & 1, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = make_sw128_desc(smem_u32(sm.x[s]));
          const uint32_t a0 = taddr + (uint32_t)(C::A_COL0 + a * 32);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_ts(d + (uint32_t)((kk % C::NACC) * NT), a0 + (uint32_t)(kk * 8), bd + (uint64_t)(kk * 2), idesc,
                      kc != 0 || kk >= C::NACC);
          tc_commit(&sm.empty[s]);
          tc_commit(&sm.a_empty[a]);
        }
        if (!ok) break;
        tc_commit(&sm.d_full[db]);
      }
      tc_commit(&sm.fin);
      mbar_wait_bounded(&sm.fin, 0);
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp - kWarpEpi0;
    const int L = quarter * 32 + lane;
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++titer) {
      const TileInfo ti = decode_tile<KIND, NT>(sm, p.meta, t);
      const int db = titer % C::ND, duse = titer / C::ND;
      const int nvalid = min(NT, ti.cnt - ti.i * NT);
      const int pos0 = ti.off + ti.i * NT;
      if (KIND == kDown) {
        // routing weight x G_d of each token column, in this warp's own copy
        __syncwarp();
        const float G = p.dn_g[ti.e];
        for (int n = lane; n < NT; n += 32)
          sm.wslot[quarter][n] = n < nvalid ? p.wts[p.sorted_slot[pos0 + n]] * G : 0.f;
        __syncwarp();
      }
      if (!wait_or_abort(sm, &sm.d_full[db], duse & 1, p.status)) break;
      tc_fence_after();
      const uint32_t trow = taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(db * C::NACC * NT);
      uint8_t* stg = sm.stage[quarter];
      if (KIND == kGateUp) {
        // lane pair (2r, 2r+1) = (gate, up) of hidden unit 16*quarter + r of the
        // tile; h values go to this warp's staging [token][16 units] and leave
        // as 32-byte row pieces (two lanes per token row)
        const float G = p.gu_g[ti.e];
        const bool odd = L & 1;
        const int ul = lane >> 1;  // unit within the warp's 16
        for (int cc = 0; cc < NT / 16; ++cc) {
          float v[16];
          tmem_ld16(trow + cc * 16, v);
#pragma unroll
          for (int acc = 1; acc < C::NACC; ++acc) {
            float w[16];
            tmem_ld16(trow + acc * NT + cc * 16, w);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] += w[k];
          }
          float o[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __shfl_xor_sync(0xffffffffu, v[k], 1);
          // even lane: tokens 0..7 of the chunk, odd lane: tokens 8..15
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float g = odd ? o[k + 8] : v[k];
            const float u = odd ? v[k + 8] : o[k];
            const int n = cc * 16 + (odd ? k + 8 : k);
            reinterpret_cast<__half*>(stg)[n * 16 + ul] = f32_to_f16_sat(gelu_tanh(G * g) * (G * u));
          }
        }
        __syncwarp();
        const int jbase = ti.j * 64 + quarter * 16;
        for (int idx = lane; idx < nvalid * 2; idx += 32) {
          const int n = idx >> 1, half = idx & 1;
          const uint4 val = *reinterpret_cast<const uint4*>(stg + n * 32 + half * 16);
          *reinterpret_cast<uint4*>(p.h + (size_t)(pos0 + n) * kI + jbase + half * 8) = val;
        }
        __syncwarp();
      } else {
        // 16-token chunks: rows of this warp x tokens -> staging [token][32 rows]
        // -> one 16-byte store per 4 rows of a token
        const int row0 = ti.j * kRows + quarter * 32;
        float* st = reinterpret_cast<float*>(stg);
        for (int cc = 0; cc < NT / 16; ++cc) {
          float v[16];
          tmem_ld16(trow + cc * 16, v);
#pragma unroll
          for (int acc = 1; acc < C::NACC; ++acc) {
            float w[16];
            tmem_ld16(trow + acc * NT + cc * 16, w);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] += w[k];
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) st[k * 32 + lane] = v[k] * sm.wslot[quarter][cc * 16 + k];
          __syncwarp();
          const int nmax = min(16, nvalid - cc * 16);
#pragma unroll
          for (int rep4 = 0; rep4 < 4; ++rep4) {
            const int k = rep4 * 4 + (lane >> 3), r4 = (lane & 7) * 4;
            if (k < nmax)
              *reinterpret_cast<float4*>(p.obuf + (size_t)(pos0 + cc * 16 + k) * kH + row0 + r4) =
                  *reinterpret_cast<const float4*>(st + k * 32 + r4);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.d_empty[db]);
    }
  }

  // ------------------------------------------------------------- tear-down
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort_flag) {
    // after an abort, let the copies still in flight land before exiting
    // (older stages were reused, so only the last NS chunks and 2 tiles can be)
    for (int it = max(0, sm.issued_chunks - C::NS); it < sm.issued_chunks; ++it)
      mbar_wait_bounded(&sm.full[it % C::NS], (it / C::NS) & 1, kAbortDrainNs);
    for (int it = max(0, sm.issued_tiles - 2); it < sm.issued_tiles; ++it)
      mbar_wait_bounded(&sm.sc_full[it & 1], (it >> 1) & 1, kAbortDrainNs);
  }
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

template <int KIND, int NT>
cudaError_t launch_moe(const ExpertArgs& a, cudaStream_t st) {
  static int configured_dev = -1;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int smem = (int)sizeof(MoeSmem<KIND, NT>) + 1024;  // + alignment slack
  if (configured_dev != dev) {
    err = cudaFuncSetAttribute(tc_moe_kernel<KIND, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  const uint64_t S = (uint64_t)a.T * kTopK;
  CUtensorMap tm_x, tm_w;
  bool ok;
  if (KIND == kGateUp) {
    ok = encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.xs, kH, S, kH * 2, kBK, NT, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.gu_q, kGuRowBytes, (uint64_t)kE * 2 * kI, kGuRowBytes, 32,
                   64, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    ok = encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.h, kI, S, kI * 2, kBK, NT, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.dn_q, kDnRowBytes, (uint64_t)kE * kH, kDnRowBytes, 32, 64,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!ok) return cudaErrorInvalidValue;
  int sms = 0;
  err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  tc_moe_kernel<KIND, NT><<<sms, kThreads, smem, st>>>(tm_x, tm_w, a);
  return cudaGetLastError();
}

// x_sorted[pos] = x16[token of sorted slot pos]: the activations in expert
// order, so that every tile of the expert GEMMs reads contiguous rows.
__global__ void __launch_bounds__(256) gather_sorted_kernel(const __half* __restrict__ x16,
                                                            const int* __restrict__ sorted_slot,
                                                            const int* __restrict__ meta, int T,
                                                            __half* __restrict__ xs, int* status) {
  constexpr int per_row = kH / 8;  // 16-byte chunks per row
  const int S = meta[kMetaOffsets + kE];
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)S * per_row;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int pos = (int)(i / per_row), c = (int)(i % per_row);
    int tok = sorted_slot[pos] / kTopK;
    if (tok < 0 || tok >= T) {
      record_status(status, kStatusDevice);
      tok = 0;
    }
    reinterpret_cast<uint4*>(xs + (size_t)pos * kH)[c] = reinterpret_cast<const uint4*>(x16 + (size_t)tok * kH)[c];
  }
}

}  // namespace

cudaError_t launch_gather_sorted(const ExpertArgs& a, cudaStream_t st) {
  const int64_t n = (int64_t)a.T * kTopK * (kH / 8);
  int blocks = (int)((n + 255) / 256);
  if (blocks > 4096) blocks = 4096;
  gather_sorted_kernel<<<blocks, 256, 0, st>>>(a.x16, a.sorted_slot, a.meta, a.T, a.xs, a.status);
  return cudaGetLastError();
}

cudaError_t launch_moe_gate_up(const ExpertArgs& a, int nt, cudaStream_t st) {
  switch (nt) {
    case 16: return launch_moe<kGateUp, 16>(a, st);
    case 64: return launch_moe<kGateUp, 64>(a, st);
    default: return launch_moe<kGateUp, 192>(a, st);
  }
}

cudaError_t launch_moe_down(const ExpertArgs& a, int nt, cudaStream_t st) {
  switch (nt) {
    case 16: return launch_moe<kDown, 16>(a, st);
    case 64: return launch_moe<kDown, 64>(a, st);
    default: return launch_moe<kDown, 192>(a, st);
  }
}

}  // namespace nvfp4moe
