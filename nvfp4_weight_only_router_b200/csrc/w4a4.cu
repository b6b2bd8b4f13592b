// W4A4 form of the routed experts: the activations are quantised to NVFP4 as
// well, and each expert GEMM runs on the block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, E2M1 x E2M1 with one E4M3 scale per 16
// elements of each operand, fp32 accumulation in tensor memory).
//
// Sources: "Gemma-4-26B-A4B-it-NVFP4" (native FP4 tensor-core execution;
// block-scale formulas), "Gemma-4-26B-A4B-NVFP4-mlx" (the checkpoint's
// input_scale sidecar: a static FP32 global per projection input), and
// "gemma-4-26B-A4B . NVFP4A16" (W4A16 forgoes the activation speed-up that
// this form takes).  Per expert e:
//   gate_up:  acc[n, u] = sum_k (E2M1 x E4M3)_x[n, k] (E2M1 x E4M3)_w[u, k]
//             h = gelu_tanh(Gx G_gu acc_gate) * (Gx G_gu acc_up), then h is
//             quantised per 16 hidden units under the static global Gh;
//   down:     o[slot, r] = w_slot G_d Gh sum_k deq(h)[k] deq(W_d)[r, k].
//
// Layouts.  Every operand stage is one contiguous block that a single bulk
// copy brings into shared memory in the form the MMA reads (K-major rows of
// 128 bytes = 256 codes, 8-row atoms of 1024 bytes with the 16-byte piece
// index XOR-ed with the row index: the 128-byte swizzle), so the weight
// stream reads whole 16 KB blocks of HBM.  Each expert's tokens are padded to
// whole tiles of NT rows:
//   weight codes      [E][N/128][K/256][128 rows][128 B]   (moe_nvfp4_pack_codes)
//   weight scales     [E][N/128][K/64][512]                (moe_w4a4_pack_scales)
//   activation codes  [tiles][K/256][NT rows][128 B]
//   activation scales [tiles][K/64][512]
// A 512-byte chunk holds the 4 scales of one K step for 128 rows, row
// r = r0 + 32 r1 at byte 16 r0 + 4 r1 + (k / 16): the order in which one
// tcgen05.cp (32 x 128 bit, copied to all four lane quarters) leaves them
// where the MMA reads them (row r at lane r0, column r1).
//
// Tiles and warps as in the W4A16 tensor-core kernel: work tile = (expert,
// token tile, 128 weight rows), K in 128-byte chunks (4 MMA K steps); warp 0
// issues the bulk copies, warp 2 the copies of the block scales into tensor
// memory, warp 1 the MMAs (one elected lane), warps 4.. the epilogue (one,
// two or four sets of 4 warps for 16-, 64- and 128-token tiles, each set
// taking a share of the tile's tokens).  A gate_up tile holds 64 hidden
// units: lane quarter q has gate rows of units 16q.. in lanes 0-15 and the
// matching up rows in lanes 16-31.  Every wait is bounded.
#include <algorithm>

#include "kernels.h"
#include "nvfp4_encode.cuh"
#include "tc_common.cuh"

namespace nvfp4moe {

namespace {

constexpr int kF4Rows = 128;    // weight rows per tile (MMA M)
constexpr int kSfChunk = 512;   // one MMA K step's block scales for 128 rows
constexpr int kF4Prod = 0, kF4Mma = 1, kF4Sf = 2, kF4Epi0 = 4;
constexpr int kF4TmemCols = 512;

template <int KIND>
struct F4Dims {
  static constexpr int NJ = KIND == 0 ? (2 * kI) / kF4Rows : kH / kF4Rows;  // 11 / 22 row tiles
  static constexpr int K = KIND == 0 ? kH : kI;                            // 2816 / 704
  static constexpr int KB = K / 2;                                         // code bytes per row
  static constexpr int KS = K / 64;                                        // MMA K steps: 44 / 11
  static constexpr int KCH = (KS + 3) / 4;                                 // 128-byte chunks: 11 / 3
};

template <int KIND, int NT>
struct F4Cfg {
  using D = F4Dims<KIND>;
  static_assert(NT % 16 == 0 && NT <= 128, "token tile");
  static constexpr int A_BYTES = kF4Rows * 128;
  static constexpr int B_BYTES = NT * 128;
  static constexpr int SF_BYTES = 4 * kSfChunk;                // 4 K steps per chunk
  static constexpr int STAGE = A_BYTES + B_BYTES + 2 * SF_BYTES;
  // epilogue: NEPI sets of 4 warps (one per tensor-memory lane quarter), set
  // h taking token columns [h TPS, (h + 1) TPS) of each tile
  static constexpr int NEPI = NT >= 128 ? 4 : (NT >= 64 ? 2 : 1);
  static constexpr int TPS = NT / NEPI;
  static constexpr int THREADS = 32 * (kF4Epi0 + 4 * NEPI);
  static constexpr int STG = KIND == 0 ? TPS * 16 : 1;         // epilogue staging floats per warp
  static constexpr int NS_SMEM = (224 * 1024 - 4 * NEPI * 4 * STG) / STAGE;
  static constexpr int NS_TMEM = (kF4TmemCols - 2 * NT) / 32;  // 32 scale columns per stage
  static constexpr int NS_MIN = NS_SMEM < NS_TMEM ? NS_SMEM : NS_TMEM;
  static constexpr int NS = NS_MIN < 8 ? NS_MIN : 8;
  static constexpr int SF_COL0 = 2 * NT;                       // after the two accumulators
  static_assert(NS >= 2, "pipeline depth");
};

template <int KIND, int NT>
struct alignas(1024) F4Smem {
  using C = F4Cfg<KIND, NT>;
  uint8_t a[C::NS][C::A_BYTES];     // weight codes, 128 rows x 128 bytes, 128B-swizzled
  uint8_t b[C::NS][C::B_BYTES];     // activation codes, NT rows x 128 bytes, 128B-swizzled
  uint8_t sfa[C::NS][C::SF_BYTES];  // weight scale chunks
  uint8_t sfb[C::NS][C::SF_BYTES];  // activation scale chunks
  float stage[4 * C::NEPI][C::STG];  // gate_up: per epilogue warp, h[token][16 units]
  // full[s]: the stage's copies landed; sf_ready[s]: its scales are in tensor
  // memory; empty[s]: its MMAs completed (stage and scale columns free)
  uint64_t full[C::NS], sf_ready[C::NS], empty[C::NS];
  uint64_t d_full[2], d_empty[2];
  uint64_t fin, sf_fin;
  uint32_t taddr;
  int mt_prefix[kE + 1];
  int abort_flag;
  int issued_chunks;
};

// Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// E4M3 scales (scale format 0), dense K = 64, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_mxf4(int M, int N) {
  return (1u << 7)                          // A format: E2M1
         | (1u << 10)                       // B format: E2M1
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory descriptor of one 512-byte scale chunk as the source of a
// 32 x 128-bit tcgen05.cp: 32 rows of 16 bytes, no swizzle, 8-row core
// matrices 128 bytes apart (there is one core matrix along K).
__device__ __forceinline__ uint64_t make_sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                 // leading byte offset (single core matrix along K)
  d |= (uint64_t)(128u >> 4) << 32;        // stride byte offset
  d |= (uint64_t)1u << 46;                 // descriptor version
  return d;                                // layout 0: no swizzle
}

// Copy a scale chunk into tensor memory (the same 32 lanes x 4 columns into
// each lane quarter), issued by one elected lane of the converged warp.
__device__ __forceinline__ void tc_cp_sf_warp(uint32_t taddr, uint64_t desc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(desc)
      : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T with E4M3 block scales from tensor memory.
__device__ __forceinline__ void tc_mma_fp4_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tc_commit_warp_f4(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// Weight row of tile row L (0..127) of row tile j of expert e.
template <int KIND>
__device__ __forceinline__ int f4_tile_row(int e, int j, int L) {
  if (KIND == 0) {
    const int q = L >> 5, w = L & 31;
    return e * (2 * kI) + (w < 16 ? 0 : kI) + j * 64 + q * 16 + (w & 15);
  }
  return e * kH + j * kF4Rows + L;
}

// Byte offset of byte k (0..127) of row r inside a block of 128-byte rows
// stored in the 128-byte swizzle (16-byte piece index XOR row % 8).
__host__ __device__ __forceinline__ uint32_t sw128(int r, int k) {
  return (uint32_t)r * 128u + ((uint32_t)(((k >> 4) ^ r) & 7) << 4) + (uint32_t)(k & 15);
}

// Exclusive prefix over experts of their token tiles (ceil(count / nt)) into
// prefix[0..E]; run by one full warp.
__device__ __forceinline__ void tile_prefix_warp(const int* meta, int nt, int* prefix) {
  const int lane = threadIdx.x & 31;
  int c[4], run = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = 4 * lane + k;
    const int cnt = meta[kMetaOffsets + e + 1] - meta[kMetaOffsets + e];
    c[k] = (cnt + nt - 1) / nt;
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
    prefix[4 * lane + k] = base;
    base += c[k];
  }
  if (lane == 31) prefix[kE] = incl;
}

// largest e with prefix[e] <= tile
__device__ __forceinline__ int expert_of_tile(const int* prefix, int tile) {
  int lo = 0, hi = kE - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------- code packing
// out[(((e NJ + j) KCH + c) 128 + L) 128 + swizzled piece] = 16 bytes of
// K bytes 128 c.. of weight row row(e, j, L) (zero past the row's end); one
// 16-byte piece per thread.
template <int KIND>
__global__ void __launch_bounds__(256) pack_mma_codes_kernel(const uint8_t* __restrict__ q, int E,
                                                             uint8_t* __restrict__ out) {
  using D = F4Dims<KIND>;
  const int64_t pieces = (int64_t)E * D::NJ * D::KCH * kF4Rows * 8;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < pieces; w += (int64_t)gridDim.x * blockDim.x) {
    const int piece = (int)(w & 7);                  // physical 16-byte piece of the row
    const int L = (int)((w >> 3) % kF4Rows);
    const int64_t blk = (w >> 3) / kF4Rows;          // (e, j, c)
    const int c = (int)(blk % D::KCH);
    const int64_t ej = blk / D::KCH;
    const int j = (int)(ej % D::NJ), e = (int)(ej / D::NJ);
    const int k = c * 128 + ((piece ^ L) & 7) * 16;  // logical K byte of this piece
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < D::KB) v = *reinterpret_cast<const uint4*>(q + (size_t)f4_tile_row<KIND>(e, j, L) * D::KB + k);
    *reinterpret_cast<uint4*>(out + (blk * kF4Rows + L) * 128 + piece * 16) = v;
  }
}

// ------------------------------------------------------------ scale packing
// out[((e NJ + j) KS + q) 512 + 16 r0 + 4 r1 + i] = s[row(e, j, r0 + 32 r1), 4 q + i]:
// one 32-bit word (the 4 scales of one row and K step) per thread.
template <int KIND>
__global__ void __launch_bounds__(256) pack_mma_scales_kernel(const uint8_t* __restrict__ s, int E,
                                                              uint8_t* __restrict__ out) {
  using D = F4Dims<KIND>;
  constexpr int SROW = D::K / kBlock;  // scale bytes per weight row
  const int64_t words = (int64_t)E * D::NJ * D::KS * (kSfChunk / 4);
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t chunk = w / (kSfChunk / 4);
    const int wi = (int)(w % (kSfChunk / 4));
    const int r0 = wi >> 2, r1 = wi & 3;
    const int q = (int)(chunk % D::KS);
    const int64_t ej = chunk / D::KS;
    const int j = (int)(ej % D::NJ), e = (int)(ej / D::NJ);
    const int row = f4_tile_row<KIND>(e, j, r0 + 32 * r1);
    const uint32_t v = *reinterpret_cast<const uint32_t*>(s + (size_t)row * SROW + 4 * q);
    *reinterpret_cast<uint32_t*>(out + chunk * kSfChunk + 4 * wi) = v;
  }
}

// ---------------------------------------------------- activation quantising
// Padded row of sorted position pos: the tile start of its expert plus its
// rank within the expert (prefix = token tiles per expert, offsets = slots).
__device__ __forceinline__ int padded_row(const int* prefix, const int* meta, int nt, int pos) {
  int lo = 0, hi = kE - 1;  // largest e with offsets[e] <= pos
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (meta[kMetaOffsets + mid] <= pos) lo = mid; else hi = mid - 1;
  }
  return prefix[lo] * nt + (pos - meta[kMetaOffsets + lo]);
}

// Each token's x quantised once under the static global gx, its codes and
// scales written to the padded rows of its 8 slots, and each slot's routing
// weight to its padded row.  Work item = (token, 32 consecutive 16-element
// blocks), one warp each, one block per lane, so that few tokens still spread
// over many SMs.  Padding rows are left as they are: a padding row only feeds
// its own (unused) accumulator column.
template <int NT>
__global__ void __launch_bounds__(256) act_quant_kernel(const uint16_t* __restrict__ x, const int* __restrict__ meta,
                                                        const int* __restrict__ slot_pos, int T, float gx,
                                                        const float* __restrict__ wts, uint8_t* __restrict__ aq,
                                                        uint8_t* __restrict__ asf, float* __restrict__ roww,
                                                        int* status) {
  constexpr int NB = kH / kBlock;          // 176 blocks per row
  constexpr int NSEG = (NB + 31) / 32;     // 6 segments of 32 blocks (the last one 16)
  constexpr int KS = kH / 64;
  constexpr int KCH = kH / 256;
  __shared__ int prefix[kE + 1];
  if (threadIdx.x < 32) tile_prefix_warp(meta, NT, prefix);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const TensorScale ts = scale_consts(gx);
  for (int item = blockIdx.x * 8 + (threadIdx.x >> 5); item < T * NSEG; item += gridDim.x * 8) {
    const int t = item / NSEG, seg = item % NSEG;
    // lanes 0..7: the padded row of slot j = lane (-1: a position outside the permutation)
    int R = 0;
    if (lane < kTopK) {
      const int pos = slot_pos[t * kTopK + lane];
      if (pos < 0 || pos >= meta[kMetaOffsets + kE]) {
        record_status(status, kStatusDevice);
        R = -1;
      } else {
        R = padded_row(prefix, meta, NT, pos);
        if (seg == 0) roww[R] = wts[t * kTopK + lane];
      }
    }
    int rows[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, R, j);
    const int kb = seg * 32 + lane;
    uint2 codes = make_uint2(0u, 0u);
    uint32_t sc = 0;
    if (kb < NB) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * kH + kb * kBlock);
      const uint4 v0 = ldg_nc_v4(src), v1 = ldg_nc_v4(src + 1);
      const uint32_t pr[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      float xv[16];
      uint32_t key2 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        xv[2 * k] = bf16_bits_to_f32(pr[k] & 0xFFFFu);
        xv[2 * k + 1] = bf16_bits_to_f32(pr[k] >> 16);
        key2 = __vmaxu2(key2, pr[k] & 0x7FFF7FFFu);
      }
      sc = encode_block16f(xv, bf16_bits_to_f32(max(key2 & 0xFFFFu, key2 >> 16)), ts, codes);
    }
    // the 4 scales of one MMA K step (lanes 4g..4g+3) as one word in lane 4g
    uint32_t word = sc;
    word |= __shfl_down_sync(0xffffffffu, sc, 1) << 8;
    word |= __shfl_down_sync(0xffffffffu, sc, 2) << 16;
    word |= __shfl_down_sync(0xffffffffu, sc, 3) << 24;
    if (kb < NB) {
#pragma unroll
      for (int j = 0; j < kTopK; ++j) {
        const int Rj = rows[j];
        if (Rj < 0) continue;
        const int tile = Rj / NT, r = Rj % NT;
        const int c = kb >> 4, kbyte = (kb & 15) * 8;
        *reinterpret_cast<uint2*>(aq + ((size_t)tile * KCH + c) * (NT * 128) + sw128(r, kbyte)) = codes;
        if ((kb & 3) == 0)
          *reinterpret_cast<uint32_t*>(asf + ((size_t)tile * KS + (kb >> 2)) * kSfChunk + 16 * (r & 31) + 4 * (r >> 5)) =
              word;
      }
    }
  }
}

// ------------------------------------------------------------ grouped GEMMs
template <int KIND, int NT>
__device__ __forceinline__ bool f4_wait(F4Smem<KIND, NT>& sm, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_wait_bounded(bar, parity)) return true;
  atomicExch(&sm.abort_flag, 1);
  record_status(status, kStatusTimeout);
  return false;
}

template <int KIND, int NT>
__global__ void __launch_bounds__(F4Cfg<KIND, NT>::THREADS, 1)
    fp4_moe_kernel(W4A4Args p) {
  using C = F4Cfg<KIND, NT>;
  using D = F4Dims<KIND>;
  using Smem = F4Smem<KIND, NT>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    tile_prefix_warp(p.meta, NT, sm.mt_prefix);
    if (lane == 0) {
      for (int s = 0; s < C::NS; ++s) {
        mbar_init(&sm.full[s], 1);
        mbar_init(&sm.sf_ready[s], 1);
        mbar_init(&sm.empty[s], 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.d_full[b], 1);
        mbar_init(&sm.d_empty[b], 4 * C::NEPI);  // one arrival per epilogue warp
      }
      mbar_init(&sm.fin, 1);
      mbar_init(&sm.sf_fin, 1);
      sm.abort_flag = 0;
      sm.issued_chunks = 0;
      fence_mbar_init();
    }
  }
  if (warp == kF4Mma) {
    tmem_alloc(&sm.taddr, kF4TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = sm.taddr;
  const int n_tiles = D::NJ * sm.mt_prefix[kE];

  if (warp == kF4Prod) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t kiter = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int mt = t / D::NJ, j = t % D::NJ;
        const int e = expert_of_tile(sm.mt_prefix, mt);
        for (int c = 0; c < D::KCH; ++c, ++kiter) {
          const int s = kiter % C::NS, use = kiter / C::NS;
          if (use > 0 && !f4_wait(sm, &sm.empty[s], (use - 1) & 1, p.status)) { ok = false; break; }
          const int nks = min(4, D::KS - 4 * c);
          mbar_arrive_expect_tx(&sm.full[s], C::A_BYTES + C::B_BYTES + 2 * nks * kSfChunk);
          bulk_g2s(sm.a[s], p.wq + ((size_t)(e * D::NJ + j) * D::KCH + c) * C::A_BYTES, C::A_BYTES, &sm.full[s]);
          bulk_g2s(sm.b[s], p.aq + ((size_t)mt * D::KCH + c) * C::B_BYTES, C::B_BYTES, &sm.full[s]);
          bulk_g2s(sm.sfa[s], p.wsf + ((size_t)(e * D::NJ + j) * D::KS + 4 * c) * kSfChunk, nks * kSfChunk,
                   &sm.full[s]);
          bulk_g2s(sm.sfb[s], p.asf + ((size_t)mt * D::KS + 4 * c) * kSfChunk, nks * kSfChunk, &sm.full[s]);
          sm.issued_chunks = kiter + 1;
        }
      }
    }
  } else if (warp == kF4Sf) {
    // ------------------------------------------- block scales -> tensor memory
    // per stage: one 32 x 128-bit copy per K step and operand into the
    // stage's own columns, then a commit that tells the MMA warp they landed
    uint32_t kiter = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      for (int c = 0; c < D::KCH; ++c, ++kiter) {
        const int s = kiter % C::NS, use = kiter / C::NS;
        ok = f4_wait(sm, &sm.full[s], use & 1, p.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const int nks = min(4, D::KS - 4 * c);
        const uint32_t sfa_t = taddr + (uint32_t)(C::SF_COL0 + 32 * s), sfb_t = sfa_t + 16;
        for (int q = 0; q < nks; ++q) {
          tc_cp_sf_warp(sfa_t + 4 * q, make_sf_desc(smem_u32(sm.sfa[s]) + q * kSfChunk));
          tc_cp_sf_warp(sfb_t + 4 * q, make_sf_desc(smem_u32(sm.sfb[s]) + q * kSfChunk));
        }
        tc_commit_warp_f4(&sm.sf_ready[s]);
      }
    }
    tc_commit_warp_f4(&sm.sf_fin);
    mbar_wait_bounded(&sm.sf_fin, 0);
    __syncwarp();
  } else if (warp == kF4Mma) {
    // ----------------------------------------------------------------- MMAs
    uint32_t kiter = 0, titer = 0;
    bool ok = true;
    constexpr uint32_t idesc = make_idesc_mxf4(kF4Rows, NT);
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
      const int db = titer & 1, duse = titer >> 1;
      if (duse > 0) ok = f4_wait(sm, &sm.d_empty[db], (duse - 1) & 1, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = taddr + (uint32_t)(db * NT);
      for (int c = 0; c < D::KCH; ++c, ++kiter) {
        const int s = kiter % C::NS, use = kiter / C::NS;
        ok = f4_wait(sm, &sm.full[s], use & 1, p.status) && f4_wait(sm, &sm.sf_ready[s], use & 1, p.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const int nks = min(4, D::KS - 4 * c);
        const uint32_t sfa_t = taddr + (uint32_t)(C::SF_COL0 + 32 * s), sfb_t = sfa_t + 16;
        const uint64_t ad = make_sw128_desc(smem_u32(sm.a[s])), bd = make_sw128_desc(smem_u32(sm.b[s]));
        for (int q = 0; q < nks; ++q) {
          // K step q: 64 codes = 32 bytes further along the swizzled rows
          tc_mma_fp4_warp(d, ad + (uint64_t)(2 * q), bd + (uint64_t)(2 * q), idesc, sfa_t + 4 * q, sfb_t + 4 * q,
                          c != 0 || q != 0);
        }
        tc_commit_warp_f4(&sm.empty[s]);
      }
      if (!ok) break;
      tc_commit_warp_f4(&sm.d_full[db]);
    }
    tc_commit_warp_f4(&sm.fin);
    mbar_wait_bounded(&sm.fin, 0);
    __syncwarp();
  } else if (warp >= kF4Epi0) {
    // ------------------------------------------------------------ epilogue
    constexpr int TPS = C::TPS, PW = (TPS + 31) / 32;
    const int qd = warp & 3;                  // tensor-memory lane quarter
    const int ew = warp - kF4Epi0;            // epilogue warp 0 .. 4 NEPI - 1
    const int n0 = (ew >> 2) * TPS;           // this set's first token column
    const TensorScale tsh = scale_consts(p.gh);
    // the tile's expert, token range, global and (down) per-token weights,
    // loaded one tile ahead so that their latency hides behind the previous tile
    struct TileMeta {
      int mt, j, e, off, cnt;
      float g;
      float w[PW];
    };
    auto load_meta = [&](int t) {
      TileMeta m;
      m.mt = t / D::NJ;
      m.j = t % D::NJ;
      m.e = expert_of_tile(sm.mt_prefix, m.mt);
      m.off = __ldg(p.meta + kMetaOffsets + m.e);
      m.cnt = __ldg(p.meta + kMetaOffsets + m.e + 1) - m.off;
      m.g = __ldg(p.wg + m.e) * p.gin;
#pragma unroll
      for (int i = 0; i < PW; ++i)
        m.w[i] = (KIND == 1 && lane + 32 * i < TPS) ? __ldg(p.roww + (size_t)m.mt * NT + n0 + lane + 32 * i) : 0.f;
      return m;
    };
    TileMeta nxt;
    if ((int)blockIdx.x < n_tiles) nxt = load_meta(blockIdx.x);
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++titer) {
      const TileMeta cur = nxt;
      if (t + (int)gridDim.x < n_tiles) nxt = load_meta(t + gridDim.x);
      const int i = cur.mt - sm.mt_prefix[cur.e];
      const int nvalid = min(NT, cur.cnt - i * NT), pos0 = cur.off + i * NT;
      const int nend = min(nvalid, n0 + TPS);  // this set's valid columns: n0 .. nend - 1
      const int db = titer & 1, duse = titer >> 1;
      if (!f4_wait(sm, &sm.d_full[db], duse & 1, p.status)) break;
      tc_fence_after();
      const uint32_t trow = taddr + ((uint32_t)(qd * 32) << 16) + (uint32_t)(db * NT);
      if (KIND == 0) {
        float* stg = sm.stage[ew];
        const bool up = lane >= 16;
        for (int cc = n0 / 16; cc * 16 < nend; ++cc) {
          float v[16], o[16];
          tmem_ld16(trow + cc * 16, v);
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __shfl_xor_sync(0xffffffffu, v[k], 16);
          // lanes 0-15: tokens 0..7 of the chunk, lanes 16-31: tokens 8..15
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float g = up ? o[k + 8] : v[k];
            const float u = up ? v[k + 8] : o[k];
            const int n = cc * 16 + (up ? k + 8 : k);
            stg[(n - n0) * 16 + (lane & 15)] = gelu_tanh(cur.g * g) * (cur.g * u);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.d_empty[db]);
        // quantise: one token's 16 hidden units per lane
        for (int n = n0 + lane; n < n0 + TPS; n += 32) {
          uint2 codes = make_uint2(0u, 0u);
          uint32_t sc = 0;
          if (n < nvalid) {
            float hv[16];
            const float4* src = reinterpret_cast<const float4*>(stg + (n - n0) * 16);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float4 f = src[k];
              hv[4 * k] = f.x; hv[4 * k + 1] = f.y; hv[4 * k + 2] = f.z; hv[4 * k + 3] = f.w;
            }
            float amax = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(hv[k]));
            sc = encode_block16f(hv, amax, tsh, codes);
          }
          // K byte 32 j + 8 qd of the hidden row: chunk (32 j + 8 qd) / 128 of the down operand
          const int kbyte = cur.j * 32 + qd * 8;
          *reinterpret_cast<uint2*>(p.hq + ((size_t)cur.mt * F4Dims<1>::KCH + (kbyte >> 7)) * (NT * 128) +
                                    sw128(n, kbyte & 127)) = codes;
          p.hsf[((size_t)cur.mt * (kI / 64) + cur.j) * kSfChunk + 16 * (n & 31) + 4 * (n >> 5) + qd] = (uint8_t)sc;
        }
        __syncwarp();
      } else {
        // lane = output row; per token one 4-byte store per lane (128 bytes per warp)
        const int row = cur.j * kF4Rows + qd * 32 + lane;
        constexpr int CW = NT % 32 == 0 ? 32 : 16;
        for (int cc = n0 / CW; cc * CW < nend; ++cc) {
          float v[CW];
          if constexpr (CW == 32) tmem_ld32(trow + cc * CW, v); else tmem_ld16(trow + cc * CW, v);
          const int nmax = min(CW, nvalid - cc * CW);
          const int ln = cc * CW - n0;          // first column of the chunk within the set
          const float wr = (ln >> 5) == 0 ? cur.w[0] : cur.w[PW - 1];
#pragma unroll
          for (int k = 0; k < CW; ++k) {
            const float wk = __shfl_sync(0xffffffffu, wr, (ln & 31) + k) * cur.g;
            if (k < nmax) p.obuf[(size_t)(pos0 + cc * CW + k) * kH + row] = v[k] * wk;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.d_empty[db]);
      }
    }
  }

  // ------------------------------------------------------------- tear-down
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && sm.abort_flag) {
    for (int it = max(0, sm.issued_chunks - C::NS); it < sm.issued_chunks; ++it)
      mbar_wait_bounded(&sm.full[it % C::NS], (it / C::NS) & 1, kAbortDrainNs);
  }
  __syncthreads();
  if (warp == kF4Mma) {
    tc_fence_after();
    tmem_dealloc(taddr, kF4TmemCols);
  }
}

template <int KIND, int NT>
cudaError_t launch_fp4(const W4A4Args& a, cudaStream_t st) {
  static_assert(sizeof(F4Smem<KIND, NT>) + 1024 <= 232448, "shared memory budget");
  const int smem = (int)sizeof(F4Smem<KIND, NT>) + 1024;
  cudaError_t err = configure_kernel_once((const void*)fp4_moe_kernel<KIND, NT>, smem);
  if (err != cudaSuccess) return err;
  int sms = 0;
  err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  fp4_moe_kernel<KIND, NT><<<sms, F4Cfg<KIND, NT>::THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t packed_code_bytes(int E, int kind) {
  return (size_t)E * (kind == 0 ? F4Dims<0>::NJ * F4Dims<0>::KCH : F4Dims<1>::NJ * F4Dims<1>::KCH) * kF4Rows * 128;
}

int w4a4_tile_tokens(int T) { return T <= 256 ? 16 : (T <= 1024 ? 64 : 128); }

cudaError_t launch_w4a4_pack_scales(const uint8_t* s, int E, int kind, uint8_t* out, cudaStream_t st) {
  const int64_t words = (int64_t)E * (kind == 0 ? F4Dims<0>::NJ * F4Dims<0>::KS : F4Dims<1>::NJ * F4Dims<1>::KS) *
                        (kSfChunk / 4);
  const int blocks = (int)std::min<int64_t>((words + 255) / 256, 148 * 16);
  if (kind == 0) pack_mma_scales_kernel<0><<<blocks, 256, 0, st>>>(s, E, out);
  else pack_mma_scales_kernel<1><<<blocks, 256, 0, st>>>(s, E, out);
  return cudaGetLastError();
}

cudaError_t launch_pack_codes(const uint8_t* q, int E, int kind, uint8_t* out, cudaStream_t st) {
  const int64_t pieces = (int64_t)E * (kind == 0 ? F4Dims<0>::NJ * F4Dims<0>::KCH : F4Dims<1>::NJ * F4Dims<1>::KCH) *
                         kF4Rows * 8;
  const int blocks = (int)std::min<int64_t>((pieces + 255) / 256, 148 * 16);
  if (kind == 0) pack_mma_codes_kernel<0><<<blocks, 256, 0, st>>>(q, E, out);
  else pack_mma_codes_kernel<1><<<blocks, 256, 0, st>>>(q, E, out);
  return cudaGetLastError();
}

cudaError_t launch_w4a4_act_quant(const uint16_t* x, const int* meta, const int* slot_pos, const float* wts, int T,
                                  float gx, int nt, uint8_t* aq, uint8_t* asf, float* roww, int* status,
                                  cudaStream_t st) {
  const int blocks = (int)std::min<int64_t>(((int64_t)T * 6 + 7) / 8, 148 * 8);  // 6 work items per token
  switch (nt) {
    case 16: act_quant_kernel<16><<<blocks, 256, 0, st>>>(x, meta, slot_pos, T, gx, wts, aq, asf, roww, status); break;
    case 64: act_quant_kernel<64><<<blocks, 256, 0, st>>>(x, meta, slot_pos, T, gx, wts, aq, asf, roww, status); break;
    case 128: act_quant_kernel<128><<<blocks, 256, 0, st>>>(x, meta, slot_pos, T, gx, wts, aq, asf, roww, status); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_w4a4_gemm(const W4A4Args& a, int kind, int nt, cudaStream_t st) {
  switch (nt) {
    case 16: return kind == 0 ? launch_fp4<0, 16>(a, st) : launch_fp4<1, 16>(a, st);
    case 64: return kind == 0 ? launch_fp4<0, 64>(a, st) : launch_fp4<1, 64>(a, st);
    case 128: return kind == 0 ? launch_fp4<0, 128>(a, st) : launch_fp4<1, 128>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4moe
