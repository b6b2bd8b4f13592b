// Grouped NVFP4 expert GEMV for few tokens per expert (decode), streaming
// each routed expert's packed weights through shared memory once.
//
// Per expert e and routed token x ("Gemma 4 26B-A4B (MoE) - Core AI":
// GELU-tanh gated experts, fused gate||up rows with gate first; weights
// e2m1 x e4m3 x fp32 per "Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe"):
//   gate_up:  h[tok, u] = gelu_tanh(G_gu * Wg[u].x) * (G_gu * Wu[u].x)
//   down:     o[slot, n] = w_slot * G_d * Wd[n].h          (per-slot rows)
//
// Decode reads only the routed experts' bytes and is bound by HBM bandwidth
// ("Gemma-4-26B-A4B-NVFP4-mlx", "Caveats").  The tensor-core MMA of this chip
// costs the same per instruction for any N up to 256, so a handful of tokens
// would leave it starved of work per weight; instead the weights are turned
// into f16 MMA operands in registers (hardware e2m1 -> f16x2 conversion, one
// f16x2 multiply by the e4m3 block scale) and fed to the warp-level
// m16n8k16 MMA with the tokens as its N dimension.
//
// Work unit = (expert, group of up to 16 of its tokens, block of 128 weight
// rows) with the whole K; a gate_up block holds 64 gate rows and the matching
// 64 up rows.  K is streamed in stages of 256 (gate_up 11, down 3 -- the last
// one only 192 wide; the rest reads as zero).  A stage holds, in shared
// memory:
//   codes  128 rows x 128 B, 128B-swizzled: with the packed codes of
//          moe_nvfp4_pack_codes, one contiguous 16 KB bulk copy (whole DRAM
//          pages; gate_up tiles interleave 16 gate rows with their 16 up rows
//          four times); else ONE TMA box (gate_up: a 3-D box over {K bytes,
//          row, gate/up half}, so 64 gate rows and their 64 up rows come
//          together; down: 128 consecutive rows) gathering 128-byte row
//          pieces.
//   x      the unit's 8 or 16 token rows x 256 K in f16, by one 3-D TMA box
//          over {64 elements, K block, row} of the activations in
//          expert-sorted order (x gathered for gate_up, h for down), so each
//          (row, 64-K block) is a 128-byte line and the 128B swizzle leaves
//          the consumers' reads free of bank conflicts.
// The e4m3 block scales (2 KB a stage) are read by the consumer lanes
// straight from global memory, three stages ahead of their use.
//
// Warps: 16 consumer warps in two groups of 8 that take alternate units of
// the CTA's contiguous unit range; warp w of a group owns 16 MMA rows of the
// unit (gate_up: gate units 8w..8w+7 and their up rows, so h is computed in
// registers; down: rows 16w..16w+15) and accumulates the whole K, so no
// cross-warp reduction is needed.  Warp 16 is the producer.  Every wait is
// bounded; a timeout records a status and the CTA drains its copies and exits.
#include "tc_common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kURows = 128;          // weight rows per unit
constexpr int kSK = 256;             // K per stage
constexpr int kUTok = 16;            // tokens per unit (two n-tiles of 8)
constexpr int kGroups = 2;
constexpr int kGroupWarps = 8;
constexpr int kConsumerWarps = kGroups * kGroupWarps;
constexpr int kProdWarp = kConsumerWarps;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // 544
constexpr int kNS = 8;               // stages in the ring

constexpr int kCodeBytes = kURows * 128;     // 16384
constexpr int kXRowBytes = kSK * 2;          // 512
constexpr int kXBytes = kUTok * kXRowBytes;  // 8192

enum Kind { kGateUp = 0, kDown = 1 };

template <int KIND>
struct SCfg {
  static constexpr int KC = KIND == kGateUp ? kH / kSK : (kI + kSK - 1) / kSK;  // 11 or 3
  static constexpr int NJ = KIND == kGateUp ? (2 * kI) / kURows : kH / kURows;   // 11 or 22
  static constexpr int KX = KIND == kGateUp ? kH : kI;                          // activation row
};

struct alignas(1024) SSmem {
  uint8_t code[kNS][kCodeBytes];   // 1024-aligned: 128B-swizzled TMA destination
  uint8_t x[kNS][kXBytes];
  uint64_t full[kNS], empty[kNS];
  int unit_prefix[kE + 1];
  int offs[kE + 1];                // per-expert slot offsets (copied from meta once)
  int abort_flag;
  int issued;       // stages issued
};

struct Unit {
  int e, tg, j, off, nvalid;
};

// Unit u of the launch: expert by binary search over the per-expert unit
// prefix, then (token group, row block) with the row block fastest.  All
// reads are shared memory (offs = the per-expert slot offsets).
template <int KIND>
__device__ __forceinline__ Unit decode_unit(const int* prefix, const int* offs, int u) {
  int lo = 0, hi = kE - 1;  // largest e with prefix[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  Unit r;
  r.e = lo;
  const int local = u - prefix[lo];
  r.tg = local / SCfg<KIND>::NJ;
  r.j = local % SCfg<KIND>::NJ;
  r.off = offs[lo];
  const int cnt = offs[lo + 1] - r.off;
  r.nvalid = min(kUTok, cnt - r.tg * kUTok);
  return r;
}

// Ring position of stage kc of local unit u: units are issued in pairs
// (2p, 2p+1), the pair's stages interleaved; a last unpaired unit follows.
__device__ __forceinline__ int stage_counter(int u, int kc, int n_local, int KC) {
  const int p = u >> 1;
  const bool pair = (u & 1) || (u + 1 < n_local);
  return p * 2 * KC + (pair ? kc * 2 + (u & 1) : kc);
}

__device__ __forceinline__ bool wait_or_abort(SSmem& sm, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_wait_bounded(bar, parity)) return true;
  atomicExch(&sm.abort_flag, 1);
  record_status(status, kStatusTimeout);
  return false;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// acc[nt][w % CH] += W(rows g, g+8; one 32-K code chunk) * X[nt] for the NNT
// n-tiles.  Word w of the chunk (K 8w..8w+7) feeds MMA steps with k-pairs
// (8w, 8w+1), (8w+2, 8w+3) [A0] and (8w+4, 8w+5), (8w+6, 8w+7) [A1]; the
// activation chunk of word w (loaded from shared memory at xo ^ 16w, plus
// 8 rows per n-tile) carries the same eight K in the same order.
//
// NVFP4: sc0 / sc1 hold the two e4m3 block scales (as f16x2) of rows g and
// g+8 for the chunk's two 16-K blocks.  aff4: the chunk is one 32-K block,
// sc0 / sc1 its fp16 scale and bi0 / bi1 its fp16 bias (each broadcast to
// both halves), and the weights are q * scale + bias.
template <int NNT, int CH, int CODEC>
__device__ __forceinline__ void mma_chunk(float (&acc)[NNT][CH][4], const uint4& w0, const uint4& w1, uint32_t sc0,
                                          uint32_t sc1, uint32_t bi0, uint32_t bi1, const uint8_t* xs, uint32_t xo) {
  const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w};
  const uint32_t a1[4] = {w1.x, w1.y, w1.z, w1.w};
  const uint32_t s0lo = bcast_lo(sc0), s0hi = bcast_hi(sc0);
  const uint32_t s1lo = bcast_lo(sc1), s1hi = bcast_hi(sc1);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint4 xb[NNT];
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt) xb[nt] = lds_v4(xs + ((xo + nt * 8 * kXRowBytes) ^ (uint32_t)(w << 4)));
    uint32_t f0[4], f1[4];
    if (CODEC == kCodecNvfp4) {
      e2m1x8_to_f16x2(a0[w], f0);
      e2m1x8_to_f16x2(a1[w], f1);
      const uint32_t s0 = w < 2 ? s0lo : s0hi, s1 = w < 2 ? s1lo : s1hi;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f0[i] = hmul2_u32(f0[i], s0);
        f1[i] = hmul2_u32(f1[i], s1);
      }
    } else {
      u4x8_affine_f16x2(a0[w], sc0, bi0, f0);
      u4x8_affine_f16x2(a1[w], sc1, bi1, f1);
    }
    const uint32_t A0[4] = {f0[0], f1[0], f0[1], f1[1]};
    const uint32_t A1[4] = {f0[2], f1[2], f0[3], f1[3]};
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt) {
      mma_f16_16816(acc[nt][w % CH], A0, xb[nt].x, xb[nt].y);
      mma_f16_16816(acc[nt][w % CH], A1, xb[nt].z, xb[nt].w);
    }
  }
}

// A lane's block-scale words of one stage: NVFP4 .x / .y = the four e4m3
// scales of rows A / B; aff4 also .z / .w = the rows' two fp16 biases (and
// .x / .y their two fp16 scales).
template <int CODEC>
struct SWord {
  using T = uint2;
};
template <>
struct SWord<kCodecAff4> {
  using T = uint4;
};

// The consumer's walk over its (unit, stage) sequence, used twice: once to
// prefetch the block scales three stages ahead, once to compute.
template <int KIND, int CODEC>
struct ScalePrefetch {
  using W = typename SWord<CODEC>::T;
  const int* offs;           // per-expert slot offsets (shared memory)
  const uint8_t* scales;     // gate_up or down scale matrix
  const uint8_t* biases;     // aff4: gate_up or down bias matrix
  const int* prefix;
  int begin, n_local, rowA, rowB, q;
  int u, kc;                 // next stage to prefetch
  size_t ra, rb;             // byte offsets of the scale rows of unit u

  __device__ __forceinline__ void set_unit() {
    if (u >= n_local) return;
    const Unit U = decode_unit<KIND>(prefix, offs, begin + u);
    if (KIND == kGateUp) {
      const size_t g0 = (size_t)U.e * (2 * kI) + (size_t)U.j * 64;  // first gate row of the unit
      ra = (g0 + rowA) * kGuScaleRow;                               // rowA < 64: gate row
      rb = (g0 + kI + (rowB - 64)) * kGuScaleRow;                   // rowB >= 64: up row
    } else {
      const size_t r0 = (size_t)U.e * kH + (size_t)U.j * kURows;
      ra = (r0 + rowA) * kDnScaleRow;
      rb = (r0 + rowB) * kDnScaleRow;
    }
  }
  // scale bytes [16 kc + 4q, +4) of both rows (the lane's 64 K of the stage:
  // four e4m3 scales, or two fp16 aff4 scales and, at the same offsets, two
  // biases); zero past the end of the unit range or of a down row
  __device__ __forceinline__ W next() {
    W v;
    v.x = v.y = 0u;
    if constexpr (CODEC == kCodecAff4) v.z = v.w = 0u;
    if (u < n_local) {
      const int b = kc * 16 + 4 * q;
      if (KIND == kGateUp || b < kDnScaleRow) {
        v.x = ldg_nc_u32(scales + ra + b);
        v.y = ldg_nc_u32(scales + rb + b);
        if constexpr (CODEC == kCodecAff4) {
          v.z = ldg_nc_u32(biases + ra + b);
          v.w = ldg_nc_u32(biases + rb + b);
        }
      }
      if (++kc == SCfg<KIND>::KC) {
        kc = 0;
        u += kGroups;
        set_unit();
      }
    }
    return v;
  }
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst_smem, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst_smem),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// Per-lane constants of a consumer warp and its scale prefetch queue.
template <int CODEC>
struct Lane {
  uint32_t cA[2], cB[2];  // code byte offsets in a stage, per segment half s
  uint32_t xo[2];         // activation byte offset of chunk 8q + 4s (n-tile 0), per s
  typename SWord<CODEC>::T sq[3];  // scale words of the next three stages
};

// All stages of one unit for one consumer warp, then its epilogue.  False if
// a wait gave up.
template <int KIND, int CODEC, int NNT>
__device__ __forceinline__ bool consume_unit(SSmem& sm, const ExpertArgs& p, const Unit& U, int u, int n_local,
                                             Lane<CODEC>& L, ScalePrefetch<KIND, CODEC>& pf, int wq, int g, int q) {
  using C = SCfg<KIND>;
  constexpr int CH = 4 / NNT;  // independent accumulator chains per n-tile
  // the epilogue's global reads, issued now so their latency hides behind the
  // unit's stages: the expert's global scale and (down) the routing weight of
  // each of this lane's token columns
  // the expert's global scale, each token column's prescale exponent and
  // (down) its routing weight, folded into one factor per column:
  //   gate_up: G_gu * 2^(e - 15) (undoes the activation prescale)
  //   down:    w * G_d * 2^(2 h_exp(e)) (undoes the hidden prescale)
  // the expert's global scale (NVFP4; aff4 has none)
  const float G = CODEC == kCodecAff4 ? 1.0f : (KIND == kGateUp ? __ldg(p.gu_g + U.e) : __ldg(p.dn_g + U.e));
  float wgt[NNT][2];  // gate_up: G_gu * 2^(e - 15); down: w * G_d * 2^(2 h_exp(e))
  float hsc[NNT][2];  // gate_up: 2^(-2 h_exp(e))
#pragma unroll
  for (int nt = 0; nt < NNT; ++nt)
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int n = nt * 8 + 2 * q + c2;
      const int pos = U.off + U.tg * kUTok + n;
      const int e = n < U.nvalid ? __ldg(p.xexp + pos) : 0;
      if (KIND == kGateUp) {
        wgt[nt][c2] = G * exp2i(e - 15);
        hsc[nt][c2] = exp2i(-2 * h_exp(e));
      } else {
        wgt[nt][c2] = n < U.nvalid ? __ldg(p.wts + __ldg(p.sorted_slot + pos)) * G * exp2i(2 * h_exp(e)) : 0.f;
      }
    }
  float acc[NNT][CH][4];
#pragma unroll
  for (int nt = 0; nt < NNT; ++nt)
#pragma unroll
    for (int w = 0; w < CH; ++w)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[nt][w][k] = 0.f;

  for (int kc = 0; kc < C::KC; ++kc) {
    const auto sq = L.sq[0];
    L.sq[0] = L.sq[1];
    L.sq[1] = L.sq[2];
    L.sq[2] = pf.next();
    const int c = stage_counter(u, kc, n_local, C::KC);
    const int slot = c % kNS;
    if (!wait_or_abort(sm, &sm.full[slot], (c / kNS) & 1, p.status)) return false;
    const uint8_t* code = sm.code[slot];
    const uint8_t* xs = sm.x[slot];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const uint4 w0 = lds_v4(code + L.cA[s2]);
      const uint4 w1 = lds_v4(code + L.cB[s2]);
      // blocks 2cc, 2cc+1 (cc = 2q + s2) of each row: half s2 of the lane's scale word
      if constexpr (CODEC == kCodecNvfp4) {
        // blocks 2s2, 2s2+1 of the lane's four: half s2 of each row's scale word
        const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(s2 ? (sq.x >> 16) : (sq.x & 0xFFFFu)));
        const uint32_t s1 = e4m3x2_to_f16x2((uint16_t)(s2 ? (sq.y >> 16) : (sq.y & 0xFFFFu)));
        mma_chunk<NNT, CH, CODEC>(acc, w0, w1, s0, s1, 0u, 0u, xs, L.xo[s2]);
      } else {
        // block s2 of the lane's two: half s2 of each row's scale and bias words
        const uint32_t s0 = s2 ? bcast_hi(sq.x) : bcast_lo(sq.x), s1 = s2 ? bcast_hi(sq.y) : bcast_lo(sq.y);
        const uint32_t b0 = s2 ? bcast_hi(sq.z) : bcast_lo(sq.z), b1 = s2 ? bcast_hi(sq.w) : bcast_lo(sq.w);
        mma_chunk<NNT, CH, CODEC>(acc, w0, w1, s0, s1, b0, b1, xs, L.xo[s2]);
      }
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.empty[slot]);
  }

  // ------------------------------------------------------------ epilogue
  bool over = false;
#pragma unroll
  for (int nt = 0; nt < NNT; ++nt) {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k] = acc[nt][0][k];
#pragma unroll
      for (int w = 1; w < CH; ++w) v[k] += acc[nt][w][k];
    }
    // v[0], v[1]: MMA row g, tokens 2q, 2q+1; v[2], v[3]: row g + 8
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int n = nt * 8 + 2 * q + c2;
      if (n >= U.nvalid) continue;
      const int pos = U.off + U.tg * kUTok + n;
      if (KIND == kGateUp) {
        const int unit = U.j * 64 + 8 * wq + g;
        const float gs = wgt[nt][c2];
        p.h[(size_t)pos * kI + unit] = f32_to_f16_sat(gelu_tanh(gs * v[c2]) * (gs * v[2 + c2]) * hsc[nt][c2], over);
      } else {
        const float wg = wgt[nt][c2];
        const int row0 = U.j * kURows + 16 * wq + g;
        p.obuf[(size_t)pos * kH + row0] = v[c2] * wg;
        p.obuf[(size_t)pos * kH + row0 + 8] = v[2 + c2] * wg;
      }
    }
  }
  if (KIND == kGateUp && __any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0)
    record_status(p.status, kStatusRange);
  return true;
}

template <int KIND, int CODEC>
__global__ void __launch_bounds__(kThreads, 1)
    stream_gemv_kernel(const __grid_constant__ CUtensorMap tm_code, const __grid_constant__ CUtensorMap tm_x8,
                       const __grid_constant__ CUtensorMap tm_x16, ExpertArgs p) {
  using C = SCfg<KIND>;
  extern __shared__ uint8_t smem_raw[];
  SSmem& sm = *reinterpret_cast<SSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- set-up
  if (warp == 0) {
    // units per expert = token groups x row blocks; exclusive prefix over experts
    int c[4], run = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 4 * lane + k;
      const int cnt = p.meta[kMetaOffsets + e + 1] - p.meta[kMetaOffsets + e];
      c[k] = ((cnt + kUTok - 1) / kUTok) * C::NJ;
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
      sm.unit_prefix[4 * lane + k] = base;
      base += c[k];
    }
    if (lane == 31) sm.unit_prefix[kE] = incl;
  }
  for (int i = threadIdx.x; i <= kE; i += kThreads) sm.offs[i] = p.meta[kMetaOffsets + i];
  if (warp == kProdWarp && lane == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kGroupWarps);
    }
    sm.abort_flag = 0;
    sm.issued = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int n_units = sm.unit_prefix[kE];
  const int begin = (int)(((long long)blockIdx.x * n_units) / gridDim.x);
  const int end = (int)(((long long)(blockIdx.x + 1) * n_units) / gridDim.x);
  const int n_local = end - begin;
  if (n_local <= 0) return;  // uniform over the CTA, nothing issued

  const uint8_t* pk = KIND == kGateUp ? p.gu_pk : p.dn_pk;
  if (warp == kProdWarp) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      int c = 0;
      bool ok = true;
      for (int pp = 0; 2 * pp < n_local && ok; ++pp) {
        const int nm = (2 * pp + 1 < n_local) ? 2 : 1;
        Unit U[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) U[m] = decode_unit<KIND>(sm.unit_prefix, sm.offs, begin + 2 * pp + (m < nm ? m : 0));
        for (int kc = 0; kc < C::KC && ok; ++kc) {
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            if (m >= nm) break;
            const int slot = c % kNS, use = c / kNS;
            if (use > 0 && !wait_or_abort(sm, &sm.empty[slot], (use - 1) & 1, p.status)) ok = false;
            if (*(volatile int*)&sm.abort_flag) ok = false;
            if (!ok) break;
            const bool small = U[m].nvalid <= 8;
            mbar_arrive_expect_tx(&sm.full[slot], kCodeBytes + (small ? kXBytes / 2 : kXBytes));
            if (pk != nullptr)    // the packed tile (expert, row block, K stage)
              bulk_g2s(sm.code[slot], pk + ((size_t)(U[m].e * C::NJ + U[m].j) * C::KC + kc) * kCodeBytes, kCodeBytes,
                       &sm.full[slot]);
            else if (KIND == kGateUp)  // {K bytes, row in half, gate/up half of expert e}
              tma_load_3d(smem_u32(sm.code[slot]), &tm_code, kc * 128, U[m].j * 64, U[m].e * 2, &sm.full[slot]);
            else
              tma_load_2d(smem_u32(sm.code[slot]), &tm_code, kc * 128, U[m].e * kH + U[m].j * kURows,
                          &sm.full[slot]);
            // the unit's activation rows in expert-sorted order, K blocks 4kc..4kc+3
            // of 64 (blocks past the row end read as zero)
            tma_load_3d(smem_u32(sm.x[slot]), small ? &tm_x8 : &tm_x16, 0, kc * 4, U[m].off + U[m].tg * kUTok,
                        &sm.full[slot]);
            sm.issued = c + 1;
            ++c;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- consumers
    const int grp = warp / kGroupWarps, wq = warp % kGroupWarps;
    const int g = lane >> 2, q = lane & 3;
    // the warp's 16 MMA rows inside the unit's 128 code rows (gate_up: gate
    // units 8wq..8wq+7 in rows 0..63, their up rows in 64..127)
    const int rowA = KIND == kGateUp ? 8 * wq + g : 16 * wq + g;
    const int rowB = KIND == kGateUp ? 64 + 8 * wq + g : 16 * wq + g + 8;
    // their rows in the stage's code tile: a packed gate_up tile holds gate
    // unit u in row 32 (u / 16) + u % 16 and its up row 16 rows further
    int tA = rowA, tB = rowB;
    if (KIND == kGateUp && pk != nullptr) {
      tA = 32 * (wq >> 1) + 8 * (wq & 1) + g;
      tB = tA + 16;
    }
    Lane<CODEC> L;
    // code chunk cc = 2q + s of rows tA / tB (128B swizzle: chunk ^ (row & 7) = chunk ^ g)
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      L.cA[s2] = (uint32_t)(tA * 128 + (((2 * q + s2) ^ g) << 4));
      L.cB[s2] = (uint32_t)(tB * 128 + (((2 * q + s2) ^ g) << 4));
      // activation chunk 4s2 + i of the 128-byte row (token g, K block q): the
      // 128B swizzle XORs the chunk with that row's index 4g + q (mod 8)
      const int k = (4 * (g & 1) + q) & 7;
      L.xo[s2] = (uint32_t)(g * kXRowBytes + 128 * q + (((4 * s2) ^ k) << 4));
    }
    ScalePrefetch<KIND, CODEC> pf;
    pf.offs = sm.offs;
    pf.scales = KIND == kGateUp ? p.gu_s : p.dn_s;
    pf.biases = reinterpret_cast<const uint8_t*>(KIND == kGateUp ? p.gu_b : p.dn_b);
    pf.prefix = sm.unit_prefix;
    pf.begin = begin;
    pf.n_local = n_local;
    pf.rowA = rowA;
    pf.rowB = rowB;
    pf.q = q;
    pf.u = grp;
    pf.kc = 0;
    pf.set_unit();
    L.sq[0] = pf.next();
    L.sq[1] = pf.next();
    L.sq[2] = pf.next();
    for (int u = grp; u < n_local; u += kGroups) {
      const Unit U = decode_unit<KIND>(sm.unit_prefix, sm.offs, begin + u);
      const bool ok = U.nvalid > 8 ? consume_unit<KIND, CODEC, 2>(sm, p, U, u, n_local, L, pf, wq, g, q)
                                   : consume_unit<KIND, CODEC, 1>(sm, p, U, u, n_local, L, pf, wq, g, q);
      if (!ok) break;
    }
  }

  // -------------------------------------------------------------- tear-down
  __syncthreads();
  if (threadIdx.x == kProdWarp * 32 && sm.abort_flag) {
    // after an abort, let the copies still in flight land before exiting
    for (int c = max(0, sm.issued - kNS); c < sm.issued; ++c)
      mbar_wait_bounded(&sm.full[c % kNS], (c / kNS) & 1, kAbortDrainNs);
  }
  __syncthreads();
}

template <int KIND, int CODEC>
cudaError_t launch_stream(const ExpertArgs& a, cudaStream_t st) {
  using C = SCfg<KIND>;
  const int smem = (int)sizeof(SSmem) + 1024;  // + alignment slack
  cudaError_t err = configure_kernel_once((const void*)stream_gemv_kernel<KIND, CODEC>, smem);
  if (err != cudaSuccess) return err;
  CUtensorMap tm_code;
  bool ok;
  if (KIND == kGateUp) {
    // codes viewed as {1408 K bytes, 704 rows, 2E halves}: a box of 64 rows
    // from both halves of expert e brings gate rows and their up rows together
    const uint64_t dims[3] = {(uint64_t)kGuRowBytes, (uint64_t)kI, (uint64_t)kE * 2};
    const uint64_t pitch[2] = {(uint64_t)kGuRowBytes, (uint64_t)kGuRowBytes * kI};
    const uint32_t box[3] = {128, 64, 2};
    ok = encode_tma_3d(&tm_code, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.gu_q, dims, pitch, box, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    ok = encode_tma_2d(&tm_code, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.dn_q, kDnRowBytes, (uint64_t)kE * kH, kDnRowBytes,
                       128, kURows, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  // activations in expert-sorted order viewed as {64 elements, K/64 blocks,
  // rows}: a box of 4 blocks x 8 or 16 rows lands as 128-byte rows
  // (row, block) with the 128B swizzle
  CUtensorMap tm_x8, tm_x16;
  {
    const uint64_t S = (uint64_t)a.T * a.spt;
    const int KX = C::KX;
    const uint64_t dims[3] = {64, (uint64_t)(KX / 64), S};
    const uint64_t pitch[2] = {128, (uint64_t)KX * 2};
    const uint32_t box8[3] = {64, 4, 8}, box16[3] = {64, 4, 16};
    const void* xsrc = KIND == kGateUp ? (const void*)a.xs : (const void*)a.h;
    ok = ok && encode_tma_3d(&tm_x8, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xsrc, dims, pitch, box8, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_3d(&tm_x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xsrc, dims, pitch, box16, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  int sms = 0;
  err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  stream_gemv_kernel<KIND, CODEC><<<sms, kThreads, smem, st>>>(tm_code, tm_x8, tm_x16, a);
  return cudaGetLastError();
}

static_assert(sizeof(SSmem) + 1024 <= 232448, "shared memory budget");

}  // namespace

cudaError_t launch_gate_up_stream(const ExpertArgs& a, cudaStream_t st) {
  return a.codec == kCodecAff4 ? launch_stream<kGateUp, kCodecAff4>(a, st) : launch_stream<kGateUp, kCodecNvfp4>(a, st);
}
cudaError_t launch_down_stream(const ExpertArgs& a, cudaStream_t st) {
  return a.codec == kCodecAff4 ? launch_stream<kDown, kCodecAff4>(a, st) : launch_stream<kDown, kCodecNvfp4>(a, st);
}

}  // namespace nvfp4moe
