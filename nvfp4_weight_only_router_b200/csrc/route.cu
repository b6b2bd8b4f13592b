// Router: scale-free RMSNorm -> x scale x H^-0.5 -> linear to 128 experts ->
// fp32 softmax -> top-8 -> renormalise -> x per_expert_scale ("Gemma 4
// 26B-A4B (MoE) - Core AI", router description under the layer dataflow
// listing).
//
// The linear map runs on the tensor cores without changing its fp32 meaning:
// logit_e = inv_rms * H^-0.5 * sum_k (x_k * scale_k) * proj_ek.  The product
// x_k * scale_k of two bf16 values has at most 16 significant bits, so it
// splits exactly into hi + lo with hi = bf16(p) and lo = bf16(p - hi); two
// bf16 MMAs (hi and lo against the same proj fragment) accumulate the exact
// products in fp32.
//
// Two kernels:
//   few tokens (T <= 256): a thread-block cluster per 16 tokens, one CTA per
//        256-wide K slice, partial logits summed through distributed shared
//        memory in rank order; the last CTA of the launch also groups the
//        slots by expert (the permutation step) when T*8 <= 1024;
//   many tokens: one CTA per 32 tokens over the whole K, streamed through a
//        TMA ring.
// Both run softmax / top-8 with one warp per token and write ids and weights.
//
// Within a K block, the MMA fragments follow the warp-level m16n8k16 layout
// (ldmatrix from 128B-swizzled shared-memory tiles).
#include "tc_common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kRouteThreads = 256;

// Top-8 of 128 logits held 4 per lane (expert lane + 32 i).  Ordered by
// descending logit (= descending probability); equal logits -> lower id first.
// pesv[i] = per_expert_scale of expert lane + 32 i (loaded by the caller ahead
// of time, so no global read sits on this token's critical path).
__device__ void finish_token(const RouteArgs& a, int t, const float (&lg)[4], const float (&pesv)[4]) {
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
  float sel_p = 0.f, sel_pes = 0.f, psum = 0.f;
  for (int r = 0; r < kTopK; ++r) {
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
    float pw = 0.f, pe = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane == owner && slot == i) {
        taken[i] = true;
        pw = p[i];
        pe = pesv[i];
      }
    pw = __shfl_sync(0xffffffffu, pw, owner);
    pe = __shfl_sync(0xffffffffu, pe, owner);
    psum += pw;
    if (lane == r) {
      sel_id = bi;
      sel_p = pw;
      sel_pes = pe;
    }
  }
  if (lane < kTopK) {
    a.ids[(size_t)t * kTopK + lane] = sel_id;
    a.wts[(size_t)t * kTopK + lane] = (sel_p / psum) * sel_pes;
  }
}

// per_expert_scale and logit bias of experts lane + 32 i
__device__ __forceinline__ void load_expert_consts(const RouteArgs& a, float (&pesv)[4], float (&bv)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pesv[i] = bf16_bits_to_f32(__ldg(a.pes + lane + 32 * i));
    bv[i] = a.bias ? __ldg(a.bias + lane + 32 * i) : 0.f;
  }
}

// Stable grouping of S <= 1024 slots by expert, by one CTA of 256 threads:
// a histogram gives the offsets, then slots are ranked in four rounds of 256
// (within-warp ranks by __match_any_sync, warp order, round order).
__device__ void block_permute_small(const RouteArgs& a) {
  __shared__ int s_cnt[kE];
  __shared__ int s_off[kE + 1];
  __shared__ int s_run[kE];
  __shared__ int s_wc[kRouteThreads / 32][kE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.T * kTopK;
  if (tid < kE) {
    s_cnt[tid] = 0;
    s_run[tid] = 0;
  }
  __syncthreads();
  for (int s = tid; s < S; s += kRouteThreads) {
    const int e = __ldcg(a.ids + s);
    if (e >= 0 && e < kE) atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  if (warp == 0) {
    int cnt[4], off[4], flag[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      cnt[i] = s_cnt[4 * lane + i];
      flag[i] = cnt[i] > 0;
    }
    int run = 0, frun = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      off[i] = run;
      run += cnt[i];
      const int f = flag[i];
      flag[i] = frun;
      frun += f;
    }
    int incl = run, fincl = frun;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      const int fn = __shfl_up_sync(0xffffffffu, fincl, o);
      if (lane >= o) {
        incl += n;
        fincl += fn;
      }
    }
    const int base = incl - run, fbase = fincl - frun;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ex = 4 * lane + i;
      s_off[ex] = base + off[i];
      a.meta[kMetaCounts + ex] = cnt[i];
      a.meta[kMetaOffsets + ex] = base + off[i];
      if (cnt[i] > 0) a.meta[kMetaAct + fbase + flag[i]] = ex;
    }
    if (lane == 31) {
      s_off[kE] = incl;
      a.meta[kMetaOffsets + kE] = incl;
      a.meta[kMetaNAct] = fincl;
    }
  }
  __syncthreads();
  for (int base = 0; base < S; base += kRouteThreads) {
    const int s = base + tid;
    int e = s < S ? __ldcg(a.ids + s) : -1;
    if (e >= kE || (e < 0 && s < S)) {
      record_status(a.status, kStatusDevice);
      e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    for (int i = tid; i < (kRouteThreads / 32) * kE; i += kRouteThreads) (&s_wc[0][0])[i] = 0;
    __syncthreads();
    if (e >= 0 && rank == 0) s_wc[warp][e] = __popc(peers);
    __syncthreads();
    if (tid < kE) {
      int run = s_run[tid];
      for (int w = 0; w < kRouteThreads / 32; ++w) {
        const int c = s_wc[w][tid];
        s_wc[w][tid] = run;
        run += c;
      }
      s_run[tid] = run;
    }
    __syncthreads();
    if (s < S) {
      if (e >= 0) {
        const int pos = s_off[e] + s_wc[warp][e] + rank;
        a.sorted_slot[pos] = s;
        a.slot_pos[s] = pos;
      } else {
        a.slot_pos[s] = -1;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------
// Cluster router.  A cluster of H/256 CTAs (11 for H = 2816) owns TOK tokens;
// CTA r owns the K slice [256 r, 256 r + 256) for all 128 experts, so the
// exact hi/lo split of x * scale is computed once per element.  Each CTA
// brings its proj slice (128 x 256 bf16, four 128B-swizzled TMA boxes) and
// its x slice (TOK x 256) into shared memory, splits x * scale into hi/lo
// bf16 tiles, runs the two bf16 MMAs per k-step and keeps its partial logits
// (TOK x 128 fp32) and partial sums of squares in shared memory.  After a
// cluster barrier each CTA finishes some of the tokens, reading the partials
// of all CTAs of the cluster in rank order (distributed shared memory, so
// the sum has a fixed order), then softmax / top-8.  A second cluster barrier
// keeps every CTA's shared memory alive until all reads are done.
constexpr int kRcK = 256;  // K per CTA
constexpr int kRcMaxRanks = 16;  // largest cluster (hidden size 4096)
constexpr int kRcMinRanks = 8;   // smallest cluster (hidden size 2048): at most TOK / 8 tokens per CTA

template <int TOK>
struct RcSmem {
  uint8_t proj[4][kE * 128];     // 4 K blocks of 64, rows = experts, 128B swizzle
  uint8_t x[4][TOK * 128];       // 4 K blocks of 64, rows = tokens, 128B swizzle
  uint16_t hi[TOK][kRcK];        // x * scale split, 16-byte chunks XOR (token & 7)
  uint16_t lo[TOK][kRcK];
  // partial logits and sums of squares pushed here by every CTA of the
  // cluster for the tokens this CTA finishes (token j -> CTA j % nr, slot j / nr)
  float red[(TOK + kRcMinRanks - 1) / kRcMinRanks][kRcMaxRanks][kE];
  float red_ss[(TOK + kRcMinRanks - 1) / kRcMinRanks][kRcMaxRanks];
  uint16_t scale[kRcK];
  uint64_t bar;
  int abort_flag;
  int last;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_shared(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float a0, float a1) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a0), "f"(a1) : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float a0) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(a0) : "memory");
}
// four 8x8 b16 matrices from shared memory, lane l giving the 16-byte row
// address of row l % 8 of matrix l / 8; register i holds matrix i in the
// warp-MMA fragment order (row l / 4, elements 2 (l % 4) and 2 (l % 4) + 1)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(addr)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_rc(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// byte offset of element k (0..255) of row r in a hi/lo tile
__device__ __forceinline__ uint32_t split_off(int r, int k) {
  return (uint32_t)(r * (kRcK * 2) + ((((k >> 3) ^ (r & 7)) << 4) | ((k & 7) << 1)));
}
// byte offset of element k (0..63) of row r in one 128B-swizzled K block
__device__ __forceinline__ uint32_t sw_off(int r, int k) {
  return (uint32_t)(r * 128 + ((((k >> 3) ^ (r & 7)) << 4) | ((k & 7) << 1)));
}

template <int TOK>
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_cluster_kernel(const __grid_constant__ CUtensorMap tm_proj, const __grid_constant__ CUtensorMap tm_x,
                         RouteArgs a) {
  extern __shared__ uint8_t smem_raw[];
  RcSmem<TOK>& sm = *reinterpret_cast<RcSmem<TOK>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int r = (int)cluster_ctarank(), nr = a.H / kRcK;
  const int tok0 = blockIdx.y * TOK;
  const int k0 = r * kRcK;
  float pesv[4], biasv[4];  // read now; used by the warps that finish tokens
  load_expert_consts(a, pesv, biasv);

  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&sm.bar, 4 * kE * 128 + 4 * TOK * 128 + kRcK * 2);
    for (int b = 0; b < 4; ++b) {
      tma_load_2d_rc(smem_u32(sm.proj[b]), &tm_proj, k0 + 64 * b, 0, &sm.bar);
      tma_load_2d_rc(smem_u32(sm.x[b]), &tm_x, k0 + 64 * b, tok0, &sm.bar);  // rows past T read as zero
    }
    bulk_g2s(sm.scale, a.scale + k0, kRcK * 2, &sm.bar);
    if (!mbar_wait_bounded(&sm.bar, 0)) {
      record_status(a.status, kStatusTimeout);
      sm.abort_flag = 1;
    }
  }
  __syncthreads();
  const bool ok = sm.abort_flag == 0;

  float acc[TOK / 16][2][4];
#pragma unroll
  for (int m = 0; m < TOK / 16; ++m)
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;

  if (ok) {
    // split: thread pair kp = tid % 128 of the slice (k = 2 kp, 2 kp + 1), tokens
    // tid / 128 + 2 i
    const int kp = tid & 127, k = 2 * kp, b = k >> 6, kk = k & 63;
    const float2 sc = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sm.scale[k]));
#pragma unroll 4
    for (int i = tid >> 7; i < TOK; i += 2) {
      const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sm.x[b] + sw_off(i, kk)));
      const float p0 = __fmul_rn(xv.x, sc.x), p1 = __fmul_rn(xv.y, sc.y);
      const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
      const float2 hf = __bfloat1622float2(h);
      const __nv_bfloat162 l = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<uint8_t*>(sm.hi) + split_off(i, k)) = h;
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<uint8_t*>(sm.lo) + split_off(i, k)) = l;
    }
    // sum of squares of x over the slice: warp w takes tokens w, w + 8, ...;
    // lane l sums k = 8l .. 8l + 7, then a butterfly over the warp
    for (int i = warp; i < TOK; i += kRouteThreads / 32) {
      float q2 = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int kk2 = 8 * lane + c;
        const float xv = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(sm.x[kk2 >> 6] + sw_off(i, kk2 & 63)));
        q2 = __fmaf_rn(xv, xv, q2);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) q2 += __shfl_xor_sync(0xffffffffu, q2, o);
      if (lane == 0) st_cluster_f32(map_shared(&sm.red_ss[i / nr][r], (uint32_t)(i % nr)), q2);
    }
  }
  __syncthreads();
  if (ok) {
    // MMAs: warp w owns experts [16w, 16w + 16) = two n-tiles, every m-tile;
    // even and odd k-steps accumulate separately (shorter dependency chains)
    float acc2[TOK / 16][2][4];
#pragma unroll
    for (int m = 0; m < TOK / 16; ++m)
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc2[m][n][i] = 0.f;
    // fragments by ldmatrix: lane l addresses row l % 8 of matrix l / 8
    const int mat = lane >> 3, rr = lane & 7;
    const uint32_t hbase = smem_u32(sm.hi), lbase = smem_u32(sm.lo);
#pragma unroll 2
    for (int ks = 0; ks < kRcK / 16; ++ks) {
      // B: matrices (n0, k lo), (n0, k hi), (n1, k lo), (n1, k hi) of this warp's 16 experts
      uint32_t bq[4];
      {
        const int e = 16 * warp + 8 * (mat >> 1) + rr, kc = (ks & 3) * 2 + (mat & 1);
        ldsm_x4(smem_u32(sm.proj[ks >> 2]) + (uint32_t)(e * 128 + ((kc ^ rr) << 4)), bq);
      }
#pragma unroll
      for (int m = 0; m < TOK / 16; ++m) {
        // A: matrices (rows lo, k lo), (rows hi, k lo), (rows lo, k hi), (rows hi, k hi)
        const int row = 16 * m + rr + 8 * (mat & 1), kc = ks * 2 + (mat >> 1);
        const uint32_t off = (uint32_t)(row * (kRcK * 2) + ((kc ^ rr) << 4));
        uint32_t ah[4], al[4];
        ldsm_x4(hbase + off, ah);
        ldsm_x4(lbase + off, al);
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          float (&d)[4] = (ks & 1) ? acc2[m][n] : acc[m][n];
          mma_bf16_16816(d, ah, bq[2 * n], bq[2 * n + 1]);
          mma_bf16_16816(d, al, bq[2 * n], bq[2 * n + 1]);
        }
      }
    }
    // push the partial logits to the CTA that finishes each token
#pragma unroll
    for (int m = 0; m < TOK / 16; ++m)
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const int e = 16 * warp + 8 * n + 2 * t4;
#pragma unroll
        for (int hrow = 0; hrow < 2; ++hrow) {
          const int j = 16 * m + g + 8 * hrow;
          st_cluster_f32x2(map_shared(&sm.red[j / nr][r][e], (uint32_t)(j % nr)),
                           acc[m][n][2 * hrow] + acc2[m][n][2 * hrow],
                           acc[m][n][2 * hrow + 1] + acc2[m][n][2 * hrow + 1]);
        }
      }
  }
  __syncthreads();
  cluster_sync_all();  // every CTA's partials have landed at their owners

  // finish: token j of the tile is done by CTA j % nr (slot j / nr), one
  // warp per slot; partials summed in rank order
  for (int sl = warp; sl * nr + r < TOK; sl += kRouteThreads / 32) {
    const int j = sl * nr + r, t = tok0 + j;
    if (t >= a.T) break;
    float lg[4] = {0.f, 0.f, 0.f, 0.f}, ssum = 0.f;
    for (int rr = 0; rr < nr; ++rr) {
#pragma unroll
      for (int i = 0; i < 4; ++i) lg[i] += sm.red[sl][rr][lane + 32 * i];
      ssum += sm.red_ss[sl][rr];
    }
    const float f = (1.0f / sqrtf(ssum / (float)a.H + a.eps)) * a.inv_sqrt_h;
#pragma unroll
    for (int i = 0; i < 4; ++i) lg[i] = lg[i] * f + biasv[i];
    finish_token(a, t, lg, pesv);
  }
  __syncthreads();
  cluster_sync_all();  // no CTA exits while peers may still store into it
  if (!ok && tid == 0) mbar_wait_bounded(&sm.bar, 0, kAbortDrainNs);  // copies of a failed wait land first

  if (a.meta == nullptr) return;
  // few tokens: the last CTA to finish groups the slots by expert
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(a.meta + kMetaRouteCounter, 1);
    sm.last = (prev == (int)(gridDim.x * gridDim.y) - 1);
    if (sm.last) a.meta[kMetaRouteCounter] = 0;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  block_permute_small(a);
}

// ------------------------------------------------------------------------
// Wide router (many tokens): a CTA owns 32 tokens and all 128 experts over
// the whole K, streamed in blocks of 64 through an 8-deep ring (proj block
// 128 x 64 and x block 32 x 64, both 128B-swizzled TMA boxes, and the
// scale block by a bulk copy).  16 warps: per block every thread splits two
// pairs of products x * scale into hi/lo bf16 (double-buffered tiles), one
// barrier, then warp w runs the hi and lo MMAs for experts [16 (w % 8), +16)
// and token tile w / 8.  Softmax / top-8 at the end from the logits in
// shared memory.
constexpr int kRwTok = 32;
constexpr int kRwNS = 8;
constexpr int kRwThreads = 512;

struct RwSmem {
  uint8_t proj[kRwNS][kE * 128];
  uint8_t x[kRwNS][kRwTok * 128];
  uint16_t scale[kRwNS][64];
  uint16_t hi[2][kRwTok * 64];   // 128-byte rows, 16-byte chunks XOR (token & 7)
  uint16_t lo[2][kRwTok * 64];
  float logits[kRwTok][kE];
  float ss[kRwTok];
  uint64_t full[kRwNS];
  int abort_flag;
};

__global__ void __launch_bounds__(kRwThreads, 1)
    route_wide_kernel(const __grid_constant__ CUtensorMap tm_proj, const __grid_constant__ CUtensorMap tm_x,
                      RouteArgs a) {
  extern __shared__ uint8_t smem_raw[];
  RwSmem& sm = *reinterpret_cast<RwSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int tok0 = blockIdx.x * kRwTok;
  const int nkb = a.H / 64;
  float pesv[4], biasv[4];  // read now; used by the warps that finish tokens
  load_expert_consts(a, pesv, biasv);
  constexpr uint32_t kStageTx = kE * 128 + kRwTok * 128 + 128;

  if (tid == 0) {
    for (int i = 0; i < kRwNS; ++i) mbar_init(&sm.full[i], 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int kb) {
    const int sl = kb % kRwNS;
    mbar_arrive_expect_tx(&sm.full[sl], kStageTx);
    tma_load_2d_rc(smem_u32(sm.proj[sl]), &tm_proj, kb * 64, 0, &sm.full[sl]);
    tma_load_2d_rc(smem_u32(sm.x[sl]), &tm_x, kb * 64, tok0, &sm.full[sl]);  // rows past T read as zero
    bulk_g2s(sm.scale[sl], a.scale + kb * 64, 128, &sm.full[sl]);
  };
  if (tid == 0)
    for (int kb = 0; kb < kRwNS - 1 && kb < nkb; ++kb) issue(kb);

  const int eg = warp & 7, mt = warp >> 3;  // expert group (16 experts), token tile
  float acc[2][4];
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
  // this thread's split elements: k pair kp = lane (k = 2 kp, 2 kp + 1), tokens warp, warp + 16
  const int kp = lane;
  float ssq[2] = {0.f, 0.f};
  int issued = min(kRwNS - 1, nkb);

  for (int kb = 0; kb < nkb; ++kb) {
    const int sl = kb % kRwNS, hb = kb & 1;
    if (!mbar_wait_bounded(&sm.full[sl], (kb / kRwNS) & 1)) {
      record_status(a.status, kStatusTimeout);
      atomicExch(&sm.abort_flag, 1);
    }
    const float2 sc = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sm.scale[sl][2 * kp]));
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = warp + 16 * i;
      const uint32_t off = sw_off(r, 2 * kp);
      const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sm.x[sl] + off));
      ssq[i] = __fmaf_rn(xv.x, xv.x, ssq[i]);
      ssq[i] = __fmaf_rn(xv.y, xv.y, ssq[i]);
      const float p0 = __fmul_rn(xv.x, sc.x), p1 = __fmul_rn(xv.y, sc.y);
      const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
      const float2 hf = __bfloat1622float2(h);
      const __nv_bfloat162 l = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<uint8_t*>(sm.hi[hb]) + off) = h;
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<uint8_t*>(sm.lo[hb]) + off) = l;
    }
    __syncthreads();  // split tiles ready; the MMAs of block kb - 1 are done everywhere
    if (sm.abort_flag) break;  // uniform: read after the barrier
    if (tid == 0 && issued < nkb) issue(issued++);  // refills the slot of block kb - 1
    // fragments by ldmatrix: lane l addresses row l % 8 of matrix l / 8
    const int mat = lane >> 3, rr = lane & 7;
    const uint32_t pb = smem_u32(sm.proj[sl]), hbase = smem_u32(sm.hi[hb]), lbase = smem_u32(sm.lo[hb]);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t bq[4];
      {
        const int e = 16 * eg + 8 * (mat >> 1) + rr, kc = ks * 2 + (mat & 1);
        ldsm_x4(pb + (uint32_t)(e * 128 + ((kc ^ rr) << 4)), bq);
      }
      const int row = 16 * mt + rr + 8 * (mat & 1), kc = ks * 2 + (mat >> 1);
      const uint32_t off = (uint32_t)(row * 128 + ((kc ^ rr) << 4));
      uint32_t ah[4], al[4];
      ldsm_x4(hbase + off, ah);
      ldsm_x4(lbase + off, al);
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        mma_bf16_16816(acc[n], ah, bq[2 * n], bq[2 * n + 1]);
        mma_bf16_16816(acc[n], al, bq[2 * n], bq[2 * n + 1]);
      }
    }
  }
  // sums of squares: warp w holds tokens w and w + 16 over all k (lane = k pair)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float q2 = ssq[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q2 += __shfl_xor_sync(0xffffffffu, q2, o);
    if (lane == 0) sm.ss[warp + 16 * i] = q2;
  }
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int e = 16 * eg + 8 * n + 2 * t4;
    sm.logits[16 * mt + g][e] = acc[n][0];
    sm.logits[16 * mt + g][e + 1] = acc[n][1];
    sm.logits[16 * mt + g + 8][e] = acc[n][2];
    sm.logits[16 * mt + g + 8][e + 1] = acc[n][3];
  }
  __syncthreads();
  if (!sm.abort_flag) {
    // softmax / top-8: warp w finishes tokens 2w, 2w + 1
    for (int j = 2 * warp; j < 2 * warp + 2; ++j) {
      const int t = tok0 + j;
      if (t >= a.T) break;
      const float f = (1.0f / sqrtf(sm.ss[j] / (float)a.H + a.eps)) * a.inv_sqrt_h;
      float lg[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) lg[i] = sm.logits[j][lane + 32 * i] * f + biasv[i];
      finish_token(a, t, lg, pesv);
    }
  } else if (tid == 0) {
    // let copies of a failed wait land before the CTA exits
    for (int kb = max(0, issued - kRwNS); kb < issued; ++kb)
      mbar_wait_bounded(&sm.full[kb % kRwNS], (kb / kRwNS) & 1, kAbortDrainNs);
  }
}

cudaError_t launch_route_wide(const RouteArgs& a, cudaStream_t st) {
  const int smem = (int)sizeof(RwSmem) + 1024;
  cudaError_t err = configure_kernel_once((const void*)route_wide_kernel, smem);
  if (err != cudaSuccess) return err;
  CUtensorMap tm_proj, tm_x;
  if (!encode_tma_2d(&tm_proj, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.proj, (uint64_t)a.H, kE, (uint64_t)a.H * 2, 64, kE,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.H, (uint64_t)a.T, (uint64_t)a.H * 2, 64,
                     kRwTok, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  route_wide_kernel<<<(a.T + kRwTok - 1) / kRwTok, kRwThreads, smem, st>>>(tm_proj, tm_x, a);
  return cudaGetLastError();
}

template <int TOK>
cudaError_t launch_route_cluster(const RouteArgs& a, cudaStream_t st) {
  const int smem = (int)sizeof(RcSmem<TOK>) + 1024;  // + alignment slack
  cudaError_t err = configure_kernel_once((const void*)route_cluster_kernel<TOK>, smem, true);
  if (err != cudaSuccess) return err;
  const int nr = a.H / kRcK;
  CUtensorMap tm_proj, tm_x;
  if (!encode_tma_2d(&tm_proj, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.proj, (uint64_t)a.H, kE, (uint64_t)a.H * 2, 64, kE,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tma_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.H, (uint64_t)a.T, (uint64_t)a.H * 2, 64,
                     TOK, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nr, (a.T + TOK - 1) / TOK, 1);
  cfg.blockDim = dim3(kRouteThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nr;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, route_cluster_kernel<TOK>, tm_proj, tm_x, a);
}

static_assert(sizeof(RcSmem<16>) + 1024 + 8192 <= 232448, "shared memory budget of the cluster router");

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  // the C ABI admits hidden sizes of 8 to 16 slices of 256 (clusters of 8 to 16 CTAs)
  if (a.H % kRcK != 0 || a.H / kRcK < kRcMinRanks || a.H / kRcK > kRcMaxRanks) return cudaErrorInvalidValue;
  // few tokens: one cluster per 16 tokens; many tokens: 32 tokens per CTA over the whole K
  return a.few_tokens ? launch_route_cluster<16>(a, st) : launch_route_wide(a, st);
}

}  // namespace nvfp4moe
