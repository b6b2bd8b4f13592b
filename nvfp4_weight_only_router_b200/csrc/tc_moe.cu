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
// Warp roles (16 warps): 0 TMA producer (activation box, packed-code boxes),
// 1-3 MMA issuers (the whole warp runs the loop so the MMA operands stay
// warp-uniform, one elected lane issues; from 64 tokens on two or three split
// the tile's tokens), 4-7 epilogue (tensor memory -> registers -> global), 8-15
// dequantisation (warp w owns tensor-memory lanes 32(w%4).. and K half
// (w-8)/4; it reads its row's e4m3 scales from global memory three chunks
// ahead, so the shared memory goes to a deeper load ring).
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
  static constexpr int X_BYTES = NT * 128;
  static constexpr int CODE_BYTES = kRows * 32;
  // epilogue staging per warp: gate_up h values (NT tokens x 16 units, f16);
  // down stores straight from registers
  static constexpr int STAGE_BYTES = KIND == kGateUp ? NT * 32 : 16;
  // load stages: as many as fit next to the scale buffers and the staging
  static constexpr int NS_RAW = (222 * 1024 - 4 * STAGE_BYTES) / (X_BYTES + CODE_BYTES);
  static constexpr int NS = NS_RAW > 24 ? 24 : NS_RAW;
  static constexpr int NA = 4;                                             // A stages (32 columns each)
  static_assert(NA <= NS, "an A stage is released through the empty barrier of its chunk's load stage");
  // independent accumulators per tile: small-N MMAs into one accumulator
  // would wait on each other, so the K sub-steps rotate over NACC of them
  static constexpr int NACC = NT <= 16 ? 4 : (NT <= 64 ? 2 : 1);
  static constexpr int ND = (2 * NACC * NT + NA * 32 <= kTmemCols) ? 2 : 1; // accumulator buffers
  static constexpr int A_COL0 = ND * NACC * NT;                           // first A-stage column
  // MMA-issuing warps: one thread issues a tcgen05.mma only every ~110
  // cycles, well below the tensor core's rate, so from 64 tokens on two or
  // three warps split the tile's tokens (N), each with its own share of the
  // accumulator columns and of the activation rows
  static constexpr int NI = NT >= 192 ? 3 : (NT >= 64 ? 2 : 1);
  static constexpr int NH = NT / NI;                                      // MMA N per issuer
  static_assert(A_COL0 + NA * 32 <= kTmemCols, "tensor memory budget");
};

template <int KIND, int NT>
struct alignas(1024) MoeSmem {
  using C = Cfg<KIND, NT>;
  uint8_t x[C::NS][C::X_BYTES];          // B tiles (SW128, 1024-aligned since X_BYTES % 1024 == 0)
  uint8_t code[C::NS][C::CODE_BYTES];    // packed codes: 128 rows x 32 bytes
  uint8_t stage[4][C::STAGE_BYTES];      // epilogue staging, one per epilogue warp
  // empty[s]: the MMAs of the chunk in stage s completed, so both its shared
  // memory stage and its tensor-memory A stage (NA <= NS) are free again
  uint64_t full[C::NS], empty[C::NS];
  uint64_t a_full[C::NA];
  uint64_t d_full[2], d_empty[2];
  uint64_t fin;
  uint32_t taddr;
  int mt_prefix[kE + 1];
  int abort_flag;
  int issued_chunks;                     // producer progress (for draining after an abort)
  // per token column of the current tile, one copy per epilogue warp:
  // gate_up: the token's prescale exponent e; down: routing weight x G_d x 2^(2 h_exp(e))
  union {
    float w;
    int e;
  } tokc[4][NT];
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

// D[tmem] (+)= A[tmem] * B[smem]^T, issued by the whole (converged) warp and
// performed by one elected lane: every lane computes the same operands, so
// they stay warp-uniform.
__device__ __forceinline__ void tc_mma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}
// The commit of the same elected lane (elect.sync in a converged warp picks
// the same lane every time, so it covers that lane's MMAs).
__device__ __forceinline__ void tc_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

template <int KIND, int NT, int CODEC>
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
        mbar_init(&sm.empty[s], C::NI);
      }
      for (int a = 0; a < C::NA; ++a) {
        mbar_init(&sm.a_full[a], 8);    // one arrival per dequant warp
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.d_full[b], C::NI);
        mbar_init(&sm.d_empty[b], 4);   // one arrival per epilogue warp
      }
      mbar_init(&sm.fin, C::NI);
      sm.abort_flag = 0;
      sm.issued_chunks = 0;
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
      uint32_t kiter = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile<KIND, NT>(sm, p.meta, t);
        const int xrow = ti.off + ti.i * NT;
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
      }
    }
  } else if (warp >= kWarpDeq0) {
    // ------------------------------------------------------ dequantisation
    const int quarter = warp & 3, khalf = (warp - kWarpDeq0) >> 2;
    const int L = quarter * 32 + lane;  // tensor-memory lane = A row
    // code / scale row in shared memory: gate_up stores gate rows 0..63 then up rows 64..127
    const int crow = KIND == kGateUp ? ((L & 1) * 64 + (L >> 1)) : L;
    // this lane's block scales of each chunk, read from global memory three
    // chunks ahead of its use (the walk crosses tile boundaries): NVFP4, the
    // two e4m3 scales of its 32 K; aff4, the one fp16 scale and (high half)
    // fp16 bias of its 32 K, which sit at the same byte offsets
    const uint8_t* sc_src = KIND == kGateUp ? p.gu_s : p.dn_s;
    const uint8_t* bi_src = reinterpret_cast<const uint8_t*>(KIND == kGateUp ? p.gu_b : p.dn_b);
    int pt = blockIdx.x, pkc = 0;
    size_t prow = 0;
    auto prow_of = [&](int t) -> size_t {
      const TileInfo ti = decode_tile<KIND, NT>(sm, p.meta, t);
      return (size_t)tile_row<KIND>(ti.e, ti.j, L) * C::SROW + khalf * 2;
    };
    if (pt < n_tiles) prow = prow_of(pt);
    auto next_scale = [&]() -> uint32_t {
      if (pt >= n_tiles) return 0;
      uint32_t v = ldg_nc_u16(sc_src + prow + pkc * 4);
      if (CODEC == kCodecAff4) v |= (uint32_t)ldg_nc_u16(bi_src + prow + pkc * 4) << 16;
      if (++pkc == C::KC) {
        pkc = 0;
        pt += gridDim.x;
        if (pt < n_tiles) prow = prow_of(pt);
      }
      return v;
    };
    uint32_t sq0 = next_scale(), sq1 = next_scale(), sq2 = next_scale();
    uint32_t kiter = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      for (int kc = 0; kc < C::KC; ++kc, ++kiter) {
        const int s = kiter % C::NS, use = kiter / C::NS;
        const int a = kiter % C::NA, ause = kiter / C::NA;
        const uint32_t sq = sq0;
        sq0 = sq1;
        sq1 = sq2;
        sq2 = next_scale();
        if (!wait_or_abort(sm, &sm.full[s], use & 1, p.status)) { ok = false; break; }
        // A stage a was last used by chunk kiter - NA (its MMAs signal empty[] of that chunk's stage)
        if (ause > 0 && !wait_or_abort(sm, &sm.empty[(kiter - C::NA) % C::NS], ((kiter - C::NA) / C::NS) & 1, p.status)) {
          ok = false;
          break;
        }
        const uint4 w = lds_v4(sm.code[s] + crow * 32 + khalf * 16);   // 32 K of this row
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
        uint32_t v[16];
        if (CODEC == kCodecNvfp4) {
          const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)sq);
          const uint32_t slo = bcast_lo(s2), shi = bcast_hi(s2);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t f[4];
            e2m1x8_to_f16x2(words[q], f);
            const uint32_t scl = q < 2 ? slo : shi;
#pragma unroll
            for (int i = 0; i < 4; ++i) v[4 * q + i] = hmul2_u32(f[i], scl);
          }
        } else {
          const uint32_t scl = bcast_lo(sq), bia = bcast_hi(sq);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t f[4];
            u4x8_affine_f16x2(words[q], scl, bia, f);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[4 * q + i] = f[i];
          }
        }
        tmem_st16(taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(C::A_COL0 + a * 32 + khalf * 16), v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.a_full[a]);
      }
    }
  } else if (warp >= kWarpMma && warp < kWarpMma + C::NI) {
    // ---------------------------------------------------------- MMA issuers
    // The whole warp runs the loop (so descriptors and addresses are
    // warp-uniform); one elected lane issues each MMA and commit.
    {
      const int hh = warp - kWarpMma;  // token share of this issuer
      uint32_t kiter = 0, titer = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
        const int db = titer % C::ND, duse = titer / C::ND;
        // only the columns of the tile's valid tokens (rounded up to 16): the
        // tensor core's time grows with N, and an expert's last tile is often
        // mostly empty; an issuer with no valid column issues nothing
        const TileInfo ti = decode_tile<KIND, NT>(sm, p.meta, t);
        const int mine = min(C::NH, min(NT, ti.cnt - ti.i * NT) - hh * C::NH);
        const int nmma = mine <= 0 ? 0 : ((mine + 15) & ~15);
        const uint32_t idesc = make_idesc_f16(kRows, nmma > 0 ? nmma : 16);
        if (duse > 0) ok = wait_or_abort(sm, &sm.d_empty[db], (duse - 1) & 1, p.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);  // one decision for the warp
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = taddr + (uint32_t)(db * C::NACC * NT + hh * C::NH);
        for (int kc = 0; kc < C::KC; ++kc, ++kiter) {
          const int s = kiter % C::NS, use = kiter / C::NS;
          const int a = kiter % C::NA, ause = kiter / C::NA;
          ok = wait_or_abort(sm, &sm.full[s], use & 1, p.status) && wait_or_abort(sm, &sm.a_full[a], ause & 1, p.status);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          // rows hh*NH.. of the 128B-swizzled activation tile (NH*128 bytes = whole 8-row atoms)
          const uint64_t bd = make_sw128_desc(smem_u32(sm.x[s]) + (uint32_t)(hh * C::NH * 128));
          const uint32_t a0 = taddr + (uint32_t)(C::A_COL0 + a * 32);
          if (nmma > 0) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_ts_warp(d + (uint32_t)((kk % C::NACC) * NT), a0 + (uint32_t)(kk * 8), bd + (uint64_t)(kk * 2),
                             idesc, kc != 0 || kk >= C::NACC);
          }
          tc_commit_warp(&sm.empty[s]);  // with no MMA in flight the arrival is immediate
        }
        if (!ok) break;
        tc_commit_warp(&sm.d_full[db]);
      }
      tc_commit_warp(&sm.fin);
      mbar_wait_bounded(&sm.fin, 0);
      __syncwarp();
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
      {
        // per token column: its prescale exponent (gate_up) or routing weight x
        // G_d x 2^(2 h_exp(e)) (down), in this warp's own copy; all slot ids and
        // exponents first, then the weights: two memory round trips per tile
        __syncwarp();
        constexpr int PER = (NT + 31) / 32;
        int ex[PER], slot[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int n = lane + 32 * i;
          ex[i] = n < nvalid ? __ldg(p.xexp + pos0 + n) : 0;
          slot[i] = (KIND == kDown && n < nvalid) ? __ldg(p.sorted_slot + pos0 + n) : -1;
        }
        if (KIND == kDown) {
          const float G = CODEC == kCodecAff4 ? 1.0f : p.dn_g[ti.e];
          float wv[PER];
#pragma unroll
          for (int i = 0; i < PER; ++i) wv[i] = slot[i] >= 0 ? __ldg(p.wts + slot[i]) : 0.f;
#pragma unroll
          for (int i = 0; i < PER; ++i)
            if (lane + 32 * i < NT) sm.tokc[quarter][lane + 32 * i].w = wv[i] * G * exp2i(2 * h_exp(ex[i]));
        } else {
#pragma unroll
          for (int i = 0; i < PER; ++i)
            if (lane + 32 * i < NT) sm.tokc[quarter][lane + 32 * i].e = ex[i];
        }
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
        const float G = CODEC == kCodecAff4 ? 1.0f : p.gu_g[ti.e];
        const bool odd = L & 1;
        const int ul = lane >> 1;  // unit within the warp's 16
        bool over = false;
        for (int cc = 0; cc * 16 < nvalid; ++cc) {
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
            // undo the activation prescale, then apply the hidden one
            const int e = sm.tokc[quarter][n].e;
            const float gs = G * exp2i(e - 15);
            reinterpret_cast<__half*>(stg)[n * 16 + ul] =
                f32_to_f16_sat(gelu_tanh(gs * g) * (gs * u) * exp2i(-2 * h_exp(e)), over);
          }
        }
        if (__any_sync(0xffffffffu, over) && lane == 0) record_status(p.status, kStatusRange);
        __syncwarp();
        const int jbase = ti.j * 64 + quarter * 16;
        for (int idx = lane; idx < nvalid * 2; idx += 32) {
          const int n = idx >> 1, half = idx & 1;
          const uint4 val = *reinterpret_cast<const uint4*>(stg + n * 32 + half * 16);
          *reinterpret_cast<uint4*>(p.h + (size_t)(pos0 + n) * kI + jbase + half * 8) = val;
        }
        __syncwarp();
      } else {
        // lane = output row; per token one 4-byte store per lane, i.e. 128
        // contiguous bytes per warp store; only the tile's valid tokens
        const int row = ti.j * kRows + quarter * 32 + lane;
        constexpr int CW = NT % 32 == 0 ? 32 : 16;  // tokens per tensor-memory load
        for (int cc = 0; cc * CW < nvalid; ++cc) {
          float v[CW];
          if constexpr (CW == 32) tmem_ld32(trow + cc * CW, v); else tmem_ld16(trow + cc * CW, v);
#pragma unroll
          for (int acc = 1; acc < C::NACC; ++acc) {
            float w[CW];
            if constexpr (CW == 32) tmem_ld32(trow + acc * NT + cc * CW, w); else tmem_ld16(trow + acc * NT + cc * CW, w);
#pragma unroll
            for (int k = 0; k < CW; ++k) v[k] += w[k];
          }
          const int nmax = min(CW, nvalid - cc * CW);
#pragma unroll
          for (int k = 0; k < CW; ++k)
            if (k < nmax) p.obuf[(size_t)(pos0 + cc * CW + k) * kH + row] = v[k] * sm.tokc[quarter][cc * CW + k].w;
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
  }
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

static_assert(sizeof(MoeSmem<kGateUp, 192>) + 1024 <= 232448, "shared memory budget (gate_up)");
static_assert(sizeof(MoeSmem<kDown, 192>) + 1024 <= 232448, "shared memory budget (down)");

template <int KIND, int NT, int CODEC>
cudaError_t launch_moe(const ExpertArgs& a, cudaStream_t st) {
  const int smem = (int)sizeof(MoeSmem<KIND, NT>) + 1024;  // + alignment slack
  cudaError_t err = configure_kernel_once((const void*)tc_moe_kernel<KIND, NT, CODEC>, smem);
  if (err != cudaSuccess) return err;
  const uint64_t S = (uint64_t)a.T * a.spt;
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
  err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  tc_moe_kernel<KIND, NT, CODEC><<<sms, kThreads, smem, st>>>(tm_x, tm_w, a);
  return cudaGetLastError();
}

// xs[pos] = f16(x[t] * 2^(15 - e_t)) and xexp[pos] = e_t for the token t of
// sorted slot pos, e_t = floor(log2 max|x[t]|) clamped to [kXExpMin,
// kXExpMax] (e_t = 0 for a zero row): the activations in expert order and in
// the f16 of the MMA operands, so that every tile of the expert GEMMs reads
// contiguous rows.  The scaled row's maximum lies in [2^15, 2^16), so every
// bf16 element down to 2^-32 of the row maximum is exact in f16.  One warp
// per row: 352 16-byte chunks, 11 per lane, all loads in flight before the
// stores.
__global__ void __launch_bounds__(256) gather_sorted_kernel(const uint16_t* __restrict__ x,
                                                            const int* __restrict__ sorted_slot,
                                                            const int* __restrict__ meta, int T, int spt,
                                                            __half* __restrict__ xs, int* __restrict__ xexp,
                                                            int* status) {
  constexpr int per_row = kH / 8;              // 352
  constexpr int per_lane = per_row / 32;       // 11
  const int S = meta[kMetaOffsets + kE];
  const int lane = threadIdx.x & 31;
  for (int pos = blockIdx.x * 8 + (threadIdx.x >> 5); pos < S; pos += gridDim.x * 8) {
    int tok = sorted_slot[pos] / spt;
    if (tok < 0 || tok >= T) {
      record_status(status, kStatusDevice);
      tok = 0;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok * kH);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)pos * kH);
    uint4 v[per_lane];
#pragma unroll
    for (int i = 0; i < per_lane; ++i) v[i] = ldg_nc_v4(src + lane + 32 * i);
    // the row maximum of |x| as a bf16 bit pattern (monotone for finite values)
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < per_lane; ++i)
      m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu),
                                 __vmaxu2(v[i].z & 0x7FFF7FFFu, v[i].w & 0x7FFF7FFFu)));
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    // floor(log2 max|x|) is the unbiased exponent field (a subnormal maximum
    // clamps to kXExpMin)
    const int e = m == 0 ? 0 : max(kXExpMin, min(kXExpMax, (int)(m >> 7) - 127));
    const float sc = exp2i(15 - e);
    bool over = false;
#pragma unroll
    for (int i = 0; i < per_lane; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o[k] = pack_f16x2(f32_to_f16_sat(bf16_bits_to_f32(w[k] & 0xFFFFu) * sc, over),
                          f32_to_f16_sat(bf16_bits_to_f32(w[k] >> 16) * sc, over));
      __stcs(dst + lane + 32 * i, make_uint4(o[0], o[1], o[2], o[3]));
    }
    if (lane == 0) xexp[pos] = e;
    if (__any_sync(0xffffffffu, over) && lane == 0) record_status(status, kStatusRange);
  }
}

}  // namespace

cudaError_t launch_gather_sorted(const ExpertArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.T * a.spt;
  int blocks = (int)((rows + 7) / 8);
  if (blocks > 148 * 32) blocks = 148 * 32;
  gather_sorted_kernel<<<blocks, 256, 0, st>>>(a.x, a.sorted_slot, a.meta, a.T, a.spt, a.xs, a.xexp, a.status);
  return cudaGetLastError();
}

template <int KIND, int CODEC>
cudaError_t launch_moe_nt(const ExpertArgs& a, int nt, cudaStream_t st) {
  switch (nt) {
    case 16: return launch_moe<KIND, 16, CODEC>(a, st);
    case 64: return launch_moe<KIND, 64, CODEC>(a, st);
    default: return launch_moe<KIND, 192, CODEC>(a, st);
  }
}

cudaError_t launch_moe_gate_up(const ExpertArgs& a, int nt, cudaStream_t st) {
  return a.codec == kCodecAff4 ? launch_moe_nt<kGateUp, kCodecAff4>(a, nt, st)
                               : launch_moe_nt<kGateUp, kCodecNvfp4>(a, nt, st);
}

cudaError_t launch_moe_down(const ExpertArgs& a, int nt, cudaStream_t st) {
  return a.codec == kCodecAff4 ? launch_moe_nt<kDown, kCodecAff4>(a, nt, st)
                               : launch_moe_nt<kDown, kCodecNvfp4>(a, nt, st);
}

}  // namespace nvfp4moe
