// The full block's dense MLP on the 5th-generation tensor cores: bf16 weights
// x bf16 activations -> fp32, both operands staged in shared memory by TMA.
//
// The block ("Gemma 4 26B-A4B (MoE) - Core AI", the layer dataflow listing)
// runs a dense GELU-gated MLP, h = down(gelu_tanh(gate x) * up x) with
// intermediate 2112 ("Architecture" table), next to the sparse branch; its
// weights stay bf16 ("Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe").
//
// Two launches of one kernel:
//   gate_up: D[128 rows, NT tokens] = [Wg rows 64j..; Wu rows 64j..] x X^T
//            (a tile stacks 64 gate rows over the matching 64 up rows), K = H;
//   down:    D[128 rows, NT tokens] = Wd rows 128j.. x (Hd_hi + Hd_lo)^T,
//            K = 2112, the gated hidden split exactly into two bf16 parts
//            (two MMAs per K step against the same weight tile).
// K is walked in chunks of 64; a work tile is (row tile, token tile, K
// split), and with few tokens the K range is split so that every SM has a
// tile; each split writes its fp32 partial tile to its own slab of the
// output, and the consumer sums the slabs in split order (deterministic).
//
// Warp roles (8 warps): 0 TMA producer, 1 MMA issuer (the whole warp runs the
// loop so descriptors stay warp-uniform; one elected lane issues), 4-7
// epilogue (tensor memory -> registers -> global, one weight row per lane).
// The accumulator is double-buffered in tensor memory so a tile's epilogue
// overlaps the next tile's MMAs.  Every wait is bounded in wall time; a wait
// that gives up records a timeout, and the CTA drains its copies and MMAs,
// frees its tensor memory and exits.
#include "tc_common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kDRows = 128;   // weight rows per tile (MMA M)
constexpr int kDBK = 64;      // K per chunk (one 128-byte swizzle atom of bf16)
constexpr int kDThreads = 256;
constexpr int kDWarpProd = 0, kDWarpMma = 1, kDWarpEpi0 = 4;
constexpr int kDTmemCols = 512;

enum DMode { kDGateUp = 0, kDDown = 1 };

template <int MODE, int NT>
struct DCfg {
  static constexpr int K = MODE == kDGateUp ? kH : kDenseI;          // 2816 or 2112
  static constexpr int KC = K / kDBK;                                 // 44 or 33 chunks
  static constexpr int MROWS = MODE == kDGateUp ? 2 * kDenseI : kH;   // 4224 or 2816
  static constexpr int MT = MROWS / kDRows;                           // 33 or 22 row tiles
  static constexpr int NB = MODE == kDGateUp ? 1 : 2;                 // B tiles per chunk (hi, lo)
  static constexpr int A_BYTES = kDRows * 128;                        // 16 KB
  static constexpr int B_BYTES = NT * 128;
  static constexpr int STAGE = A_BYTES + NB * B_BYTES;
  static constexpr int NS_RAW = (220 * 1024) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
  static constexpr int ND = 2 * NT <= kDTmemCols ? 2 : 1;             // accumulator buffers
  static_assert(NS >= 2, "shared memory budget");
};

template <int MODE, int NT>
struct alignas(1024) DSmem {
  using C = DCfg<MODE, NT>;
  uint8_t stage[C::NS][C::STAGE];  // A tile then B tile(s), each 1024-aligned, 128B-swizzled
  uint64_t full[C::NS], empty[C::NS];
  uint64_t d_full[2], d_empty[2];
  uint64_t fin;
  uint32_t taddr;
  int abort_flag;
  int issued_chunks;
};

// Work tile t of the launch: row tile fastest, then K split, then token tile.
struct DTile {
  int m, ks, n, kc0, kc1;
};

template <int MODE, int NT>
__device__ __forceinline__ DTile dense_tile(int t, int splits) {
  using C = DCfg<MODE, NT>;
  DTile d;
  d.m = t % C::MT;
  d.ks = (t / C::MT) % splits;
  d.n = t / (C::MT * splits);
  d.kc0 = d.ks * C::KC / splits;
  d.kc1 = (d.ks + 1) * C::KC / splits;
  return d;
}

template <int MODE, int NT>
__device__ __forceinline__ bool dwait(DSmem<MODE, NT>& sm, uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_wait_bounded(bar, parity)) return true;
  atomicExch(&sm.abort_flag, 1);
  record_status(status, kStatusTimeout);
  return false;
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by the whole (converged) warp and
// performed by one elected lane (warp-uniform operands).
__device__ __forceinline__ void tc_mma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit_warp_d(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N) {
  return make_idesc_f16(M, N) | (1u << 7) | (1u << 10);
}

template <int MODE, int NT>
__global__ void __launch_bounds__(kDThreads, 1)
    dense_gemm_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                      const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                      DenseArgs p, int splits) {
  using C = DCfg<MODE, NT>;
  using Smem = DSmem<MODE, NT>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = C::MT * splits * ((p.T + NT - 1) / NT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.d_full[b], 1);
      mbar_init(&sm.d_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sm.fin, 1);
    sm.abort_flag = 0;
    sm.issued_chunks = 0;
    fence_mbar_init();
  }
  if (warp == kDWarpMma) {
    tmem_alloc(&sm.taddr, kDTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = sm.taddr;

  if (warp == kDWarpProd) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t kiter = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const DTile d = dense_tile<MODE, NT>(t, splits);
        for (int kc = d.kc0; kc < d.kc1; ++kc, ++kiter) {
          const int s = kiter % C::NS, use = kiter / C::NS;
          if (use > 0 && !dwait(sm, &sm.empty[s], (use - 1) & 1, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], C::STAGE);
          const uint32_t dst = smem_u32(sm.stage[s]);
          if (MODE == kDGateUp) {
            // 64 gate rows over the matching 64 up rows
            tma_load_2d(dst, &tm_a0, kc * kDBK, d.m * 64, &sm.full[s]);
            tma_load_2d(dst + C::A_BYTES / 2, &tm_a1, kc * kDBK, d.m * 64, &sm.full[s]);
          } else {
            tma_load_2d(dst, &tm_a0, kc * kDBK, d.m * kDRows, &sm.full[s]);
          }
          // token rows past T read as zero
          tma_load_2d(dst + C::A_BYTES, &tm_b0, kc * kDBK, d.n * NT, &sm.full[s]);
          if (C::NB == 2) tma_load_2d(dst + C::A_BYTES + C::B_BYTES, &tm_b1, kc * kDBK, d.n * NT, &sm.full[s]);
          sm.issued_chunks = kiter + 1;
        }
      }
    }
  } else if (warp == kDWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    uint32_t kiter = 0, titer = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++titer) {
      const DTile d = dense_tile<MODE, NT>(t, splits);
      const int db = titer % C::ND, duse = titer / C::ND;
      // only the columns of the tile's valid tokens (rounded up to 16)
      const int nvalid = min(NT, p.T - d.n * NT);
      const int nmma = (nvalid + 15) & ~15;
      const uint32_t idesc = make_idesc_bf16(kDRows, nmma);
      if (duse > 0) ok = dwait(sm, &sm.d_empty[db], (duse - 1) & 1, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t dcol = taddr + (uint32_t)(db * NT);
      for (int kc = d.kc0; kc < d.kc1; ++kc, ++kiter) {
        const int s = kiter % C::NS, use = kiter / C::NS;
        ok = __shfl_sync(0xffffffffu, dwait(sm, &sm.full[s], use & 1, p.status), 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = smem_u32(sm.stage[s]);
        const uint64_t ad = make_sw128_desc(base);
#pragma unroll
        for (int b = 0; b < C::NB; ++b) {
          const uint64_t bd = make_sw128_desc(base + C::A_BYTES + b * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kDBK / 16; ++kk)
            tc_mma_ss_warp(dcol, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                           kc != d.kc0 || kk > 0 || b > 0);
        }
        tc_commit_warp_d(&sm.empty[s]);
      }
      if (!ok) break;
      tc_commit_warp_d(&sm.d_full[db]);
    }
    // every MMA this warp issued has completed before the tear-down frees
    // tensor memory (also after an abort)
    tc_commit_warp_d(&sm.fin);
    mbar_wait_bounded(&sm.fin, 0);
    __syncwarp();
  } else if (warp >= kDWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp - kDWarpEpi0;
    const int row = quarter * 32 + lane;  // tile row = tensor-memory lane
    uint32_t titer = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++titer) {
      const DTile d = dense_tile<MODE, NT>(t, splits);
      const int db = titer % C::ND, duse = titer / C::ND;
      if (!dwait(sm, &sm.d_full[db], duse & 1, p.status)) break;
      tc_fence_after();
      const int nvalid = min(NT, p.T - d.n * NT);
      // output row of this lane: gate_up tiles hold gate rows 64m.. then up rows
      const int orow = MODE == kDGateUp ? (row < 64 ? d.m * 64 + row : kDenseI + d.m * 64 + row - 64)
                                        : d.m * kDRows + row;
      float* out = p.out + (size_t)d.ks * p.T * C::MROWS + orow;
      const uint32_t trow = taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(db * NT);
      for (int cc = 0; cc * 16 < nvalid; ++cc) {
        float v[16];
        tmem_ld16(trow + cc * 16, v);
        const int nmax = min(16, nvalid - cc * 16);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k < nmax) out[(size_t)(d.n * NT + cc * 16 + k) * C::MROWS] = v[k];
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
    for (int it = max(0, sm.issued_chunks - C::NS); it < sm.issued_chunks; ++it)
      mbar_wait_bounded(&sm.full[it % C::NS], (it / C::NS) & 1, kAbortDrainNs);
  }
  __syncthreads();
  if (warp == kDWarpMma) {
    tc_fence_after();
    tmem_dealloc(taddr, kDTmemCols);
  }
}

template <int MODE, int NT>
cudaError_t launch_dense(const DenseArgs& a, cudaStream_t st) {
  using C = DCfg<MODE, NT>;
  const int smem = (int)sizeof(DSmem<MODE, NT>) + 1024;
  cudaError_t err = configure_kernel_once((const void*)dense_gemm_kernel<MODE, NT>, smem);
  if (err != cudaSuccess) return err;
  int sms = 0;
  err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  const int nt = (a.T + NT - 1) / NT;
  const int splits = a.splits;
  CUtensorMap ta0, ta1, tb0, tb1;
  bool ok;
  if (MODE == kDGateUp) {
    ok = encode_tma_2d(&ta0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w0, kH, kDenseI, kH * 2, kDBK, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&ta1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w1, kH, kDenseI, kH * 2, kDBK, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&tb0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b0, kH, (uint64_t)a.T, kH * 2, kDBK, NT,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    tb1 = tb0;
  } else {
    ok = encode_tma_2d(&ta0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w0, kDenseI, kH, kDenseI * 2, kDBK, kDRows,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&tb0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b0, kDenseI, (uint64_t)a.T, kDenseI * 2, kDBK, NT,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tma_2d(&tb1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b1, kDenseI, (uint64_t)a.T, kDenseI * 2, kDBK, NT,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    ta1 = ta0;
  }
  if (!ok) return cudaErrorInvalidValue;
  const int tiles = C::MT * splits * nt;
  dense_gemm_kernel<MODE, NT><<<tiles < sms ? tiles : sms, kDThreads, smem, st>>>(ta0, ta1, tb0, tb1, a, splits);
  return cudaGetLastError();
}

static_assert(sizeof(DSmem<kDGateUp, 256>) + 1024 <= 232448, "shared memory budget (gate_up)");
static_assert(sizeof(DSmem<kDDown, 128>) + 1024 <= 232448, "shared memory budget (down)");

}  // namespace

// split K until every SM has a tile, each split keeping at least 4 chunks
int dense_splits(int mode, int T, int sms) {
  const int NT = T <= 64 ? 64 : (mode == kDGateUp ? 256 : 128);
  const int MT = mode == kDGateUp ? (2 * kDenseI) / kDRows : kH / kDRows;
  const int KC = (mode == kDGateUp ? kH : kDenseI) / kDBK;
  const int nt = (T + NT - 1) / NT;
  int splits = 1;
  while (MT * nt * splits * 2 <= sms && KC / (splits * 2) >= 4) splits *= 2;
  return splits;
}

cudaError_t launch_dense_gate_up(const DenseArgs& a, cudaStream_t st) {
  return a.T <= 64 ? launch_dense<kDGateUp, 64>(a, st) : launch_dense<kDGateUp, 256>(a, st);
}

cudaError_t launch_dense_down(const DenseArgs& a, cudaStream_t st) {
  return a.T <= 64 ? launch_dense<kDDown, 64>(a, st) : launch_dense<kDDown, 128>(a, st);
}

}  // namespace nvfp4moe
