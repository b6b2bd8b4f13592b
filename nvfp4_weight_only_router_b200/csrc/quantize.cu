// NVFP4 quantise / dequantise kernels.
//
// Method ("Gemma-4-26B-A4B-it-NVFP4" page, block-scale formulas, in the
// two-level form of the "gemma-4-26B-A4B . NVFP4A16" card, "Quantization
// details"): per tensor G = amax / (6 * 448); per block of 16 along K
// s = E4M3_rne_satfinite((amax_b / 6) / G), d = s * G; per element the code is
// the E2M1 value nearest to w / d, ties to the even code, saturating at 6, with
// the sign bit of w.  Each step is one correctly rounded fp32 operation.
//
// Main path (quantize_fused_kernel): one cooperative launch, one CTA per SM,
// reads every weight from HBM once.  Each CTA owns a contiguous 1/n of every
// tensor and streams its pieces of tensors e .. e+3 into four shared-memory
// buffers (bulk asynchronous copies).  Per tensor it reduces |w| over its
// piece, publishes the maximum (atomicMax) and arrives on a counter; once all
// CTAs have arrived it encodes its piece from shared memory.  The compute
// warps reduce two tensors ahead of the one they encode, and a control warp
// does the global publishing and waiting, so neither the wait nor the copies
// of later tensors hold the compute warps up.  Every wait is bounded.
// Fallback (tensors too large for the buffers, too small to split, or no room
// for the counters): amax_kernel reduces |w| per tensor, then encode_kernel
// encodes one 16-element block per thread.
//
// The element step avoids a division per element: with r = 1/d (correctly
// rounded), the quotients w * r * (1 -+ 2^-20) bracket the correctly rounded
// w / d, and E2M1 rounding is monotone, so when both bracket ends give the
// same code that code is the one of w / d.  Blocks where they differ (a
// quotient within ~2^-20 of a rounding threshold) take the exact division.
#include "common.cuh"
#include "kernels.h"
#include "nvfp4_encode.cuh"

namespace nvfp4moe {

// |w| of a bf16 pattern as a monotone integer key (non-NaN inputs).
__device__ __forceinline__ uint32_t bf16_abs_key(uint32_t b) { return b & 0x7FFFu; }

// Per-tensor max |w|, tensors on grid rows blockIdx.y, blockIdx.y + gridDim.y, ...
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ w, int64_t E, int64_t per_expert,
                                                   uint32_t* __restrict__ amax_bits) {
  __shared__ uint32_t red[8];
  const int64_t n16 = per_expert / 8;  // 8 bf16 per 16-byte load
  for (int64_t e = blockIdx.y; e < E; e += gridDim.y) {
    const uint4* base = reinterpret_cast<const uint4*>(w + (size_t)e * per_expert);
    uint32_t m = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
      uint4 v = ldg_nc_v4(base + i);
      uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m = max(m, bf16_abs_key(a[j] & 0xFFFFu));
        m = max(m, bf16_abs_key(a[j] >> 16));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int j = 1; j < (int)(blockDim.x >> 5); ++j) m = max(m, red[j]);
      atomicMax(amax_bits + e, m << 16);  // fp32 bit pattern of the bf16 amax
    }
    __syncthreads();  // red[] is reused by the next tensor
  }
}

// max |w| of a block as a bf16 bit pattern (a monotone key for finite values)
__device__ __forceinline__ uint32_t block_key16(const uint32_t (&pair)[8]) {
  uint32_t key2 = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) key2 = __vmaxu2(key2, pair[j] & 0x7FFF7FFFu);
  return max(key2 & 0xFFFFu, key2 >> 16);
}

// encode_block16 with the block's max |w| key already known
__device__ __forceinline__ uint32_t encode_block16k(const uint32_t (&pair)[8], uint32_t key, const TensorScale& ts,
                                                    uint2& codes) {
  float x[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    x[2 * j] = bf16_bits_to_f32(pair[j] & 0xFFFFu);
    x[2 * j + 1] = __uint_as_float(pair[j] & 0xFFFF0000u);
  }
  return encode_block16f(x, __uint_as_float(key << 16), ts, codes);
}

__device__ __forceinline__ uint32_t encode_block16(const uint32_t (&pair)[8], const TensorScale& ts, uint2& codes) {
  return encode_block16k(pair, block_key16(pair), ts, codes);
}

__global__ void __launch_bounds__(256) encode_kernel(const uint16_t* __restrict__ w,
                                                     int64_t blocks_per_expert, int64_t n_blocks,
                                                     const uint32_t* __restrict__ amax_bits,
                                                     uint8_t* __restrict__ q, uint8_t* __restrict__ s,
                                                     float* __restrict__ g) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= n_blocks) return;
  const int64_t e = blk / blocks_per_expert;
  const TensorScale ts = tensor_scale(__uint_as_float(amax_bits[e]));
  if (blk == e * blocks_per_expert) g[e] = ts.G;

  const uint4* src = reinterpret_cast<const uint4*>(w) + blk * 2;
  uint4 v0 = ldg_nc_v4(src), v1 = ldg_nc_v4(src + 1);
  const uint32_t pair[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  uint2 codes;
  const uint32_t sc = encode_block16(pair, ts, codes);
  *reinterpret_cast<uint2*>(q + blk * 8) = codes;
  s[blk] = (uint8_t)sc;
}

// ------------------------------------------------------- single-pass path
constexpr int kQThreads = 1024;                // warp 0: control; warps 1..31: compute
constexpr int kQCompute = kQThreads - 32;
constexpr int kQBufs = 4;                      // tensors e (encoding), e+1, e+2 (reduced), e+3 (loading)
constexpr int kQHeader = 1024;                 // barriers, reduction slots, tensor constants, flags
constexpr int kQMaxPiece = 54400;              // bytes per buffer (1700 blocks)
constexpr int kQKeys = kQMaxPiece / 32;         // per-block max |w| keys (u16) per buffer

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// amax_ws: [E] amax bit patterns, then 3 arrival counters (tensor e counts on
// counter e % 3, which receives the arrivals of e, e+3, ...); all zero on
// entry.  Launched cooperatively (every CTA resident), one CTA per SM.
//
// Per CTA, tensor e lives in buffer e % 4.  The compute warps reduce |w| over
// tensor e+2's piece while the control thread (warp 0, lane 0) publishes
// tensor e's maximum, waits for every CTA's, and hands the tensor constants
// back; so the global round trips overlap the compute warps' work:
//   control: part(e+1) -> atomicMax, arrive on the counter of e+1 -> wait for
//            all CTAs' arrivals on e -> constants of e -> scale(e) ->
//            [free(e-1)] -> copy of e+3
//   compute: full(e+2) -> reduce -> part(e+2) -> scale(e) -> encode e -> free(e)
// A CTA publishes e+1 only after all CTAs published e-1, so counters modulo 3
// never mix tensors that are both in flight.
//
// extra_target (0 in normal use) raises the arrival count the control thread
// waits for, and wait_ns limits every wait: with extra_target > 0 the wait
// can never be met, which exercises the timeout path (every CTA gives up,
// records the timeout status, lets its copies land and exits).
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_fused_kernel(const uint16_t* __restrict__ w, int E, int64_t bpe, uint32_t* amax_ws,
                          uint8_t* __restrict__ q, uint8_t* __restrict__ s, float* __restrict__ g, int* status,
                          uint32_t extra_target, uint64_t wait_ns) {
  extern __shared__ __align__(128) uint8_t qsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(qsm);        // copy landed
  uint64_t* part = full + kQBufs;                           // compute warps' maxima written
  uint64_t* scl = part + kQBufs;                            // tensor constants published
  uint64_t* freeb = scl + kQBufs;                           // buffer fully read
  uint32_t (*red)[32] = reinterpret_cast<uint32_t(*)[32]>(qsm + 128);          // [kQBufs][31]
  TensorScale* ts_sh = reinterpret_cast<TensorScale*>(qsm + 128 + kQBufs * 128);  // [kQBufs]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(qsm + 960);
  uint8_t* buf0 = qsm + kQHeader;
  uint16_t* keys = reinterpret_cast<uint16_t*>(buf0 + (size_t)kQBufs * kQMaxPiece);  // [kQBufs][kQKeys]
  uint32_t* ctr = amax_ws + E;
  const int n = gridDim.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t b0 = (int64_t)blockIdx.x * bpe / n, b1 = (int64_t)(blockIdx.x + 1) * bpe / n;
  const int nb = (int)(b1 - b0);              // this CTA's blocks of every tensor
  const uint32_t piece = (uint32_t)nb * 32u;  // bytes

  if (tid == 0) {
    for (int b = 0; b < kQBufs; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&part[b], kQCompute / 32);
      mbar_init(&scl[b], 1);
      mbar_init(&freeb[b], kQCompute / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto fail = [&]() {
    *abort_flag = 1;
    record_status(status, kStatusTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ control
    if (lane == 0) {
      int issued = 0;
      auto issue = [&](int t) {  // tensor t's piece into buffer t % 4
        uint64_t* bar = &full[t % kQBufs];
        if (piece > 0) {
          mbar_arrive_expect_tx(bar, piece);
          bulk_g2s(buf0 + (size_t)(t % kQBufs) * kQMaxPiece, w + ((size_t)t * bpe + b0) * 16, piece, bar);
        } else {
          mbar_arrive(bar);
        }
        issued = t + 1;
      };
      for (int t = 0; t < kQBufs - 1 && t < E; ++t) issue(t);
      // publish tensor t's maximum once the compute warps have reduced it
      auto contribute = [&](int t) -> bool {
        const int b = t % kQBufs;
        if (*abort_flag || !mbar_wait_bounded(&part[b], (t / kQBufs) & 1, wait_ns)) return false;
        uint32_t m = 0;
        for (int j = 0; j < kQCompute / 32; ++j) m = max(m, red[b][j]);
        atomicMax(amax_ws + t, m << 16);  // fp32 bit pattern of the bf16 amax
        red_release_add(ctr + t % 3, 1u);
        return true;
      };
      if (!contribute(0)) fail();
      for (int e = 0; e < E && !*abort_flag; ++e) {
        const int b = e % kQBufs;
        const uint32_t target = (uint32_t)n * (uint32_t)(e / 3 + 1) + extra_target;
        uint32_t c = ld_acquire_u32(ctr + e % 3);  // in flight while tensor e+1 is published
        if (e + 1 < E && !contribute(e + 1)) {
          fail();
          break;
        }
        if (c < target) {
          const uint64_t t0 = globaltimer_ns();
          while ((c = ld_acquire_u32(ctr + e % 3)) < target)
            if (globaltimer_ns() - t0 > wait_ns) break;
        }
        if (c < target) {
          fail();
          break;
        }
        ts_sh[b] = tensor_scale(__uint_as_float(__ldcg(amax_ws + e)));
        if (blockIdx.x == 0) g[e] = ts_sh[b].G;
        mbar_arrive(&scl[b]);
        const int t = e + kQBufs - 1;
        if (t < E) {
          if (t >= kQBufs && !mbar_wait_bounded(&freeb[t % kQBufs], ((t - kQBufs) / kQBufs) & 1, wait_ns)) {
            fail();
            break;
          }
          issue(t);
        }
      }
      if (*abort_flag) {
        // let the copies still in flight land before exiting
        for (int t = issued - kQBufs < 0 ? 0 : issued - kQBufs; t < issued; ++t)
          mbar_wait_bounded(&full[t % kQBufs], (t / kQBufs) & 1, kAbortDrainNs);
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    const int ct = tid - 32, cw = warp - 1;
    // |w| over tensor t's piece -> red[t % 4][cw]; each block's own maximum
    // is kept in keys[] for the encoder
    auto reduce = [&](int t) -> bool {
      const int b = t % kQBufs;
      if (!mbar_wait_bounded(&full[b], (t / kQBufs) & 1, wait_ns)) return false;
      const uint4* v = reinterpret_cast<const uint4*>(buf0 + (size_t)b * kQMaxPiece);
      uint16_t* kb = keys + (size_t)b * kQKeys;
      uint32_t m = 0;
      for (int lb = ct; lb < nb; lb += kQCompute) {
        const uint4 v0 = v[2 * lb], v1 = v[2 * lb + 1];
        const uint32_t pair[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint32_t key = block_key16(pair);
        kb[lb] = (uint16_t)key;
        m = max(m, key);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) {
        red[b][cw] = m;
        mbar_arrive(&part[b]);
      }
      return true;
    };
    bool ok = reduce(0) && (E < 2 || reduce(1));
    for (int e = 0; e < E && ok; ++e) {
      if (e + 2 < E && !reduce(e + 2)) {
        ok = false;
        break;
      }
      const int b = e % kQBufs;
      if (!mbar_wait_bounded(&scl[b], (e / kQBufs) & 1, wait_ns)) {
        ok = false;
        break;
      }
      const TensorScale ts = ts_sh[b];
      const uint4* v = reinterpret_cast<const uint4*>(buf0 + (size_t)b * kQMaxPiece);
      const uint16_t* kb = keys + (size_t)b * kQKeys;
      const size_t gb0 = (size_t)e * bpe + b0;
      for (int lb = ct; lb < nb; lb += kQCompute) {
        const uint4 v0 = v[2 * lb], v1 = v[2 * lb + 1];
        const uint32_t pair[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint2 codes;
        const uint32_t sc = encode_block16k(pair, kb[lb], ts, codes);
        *reinterpret_cast<uint2*>(q + (gb0 + lb) * 8) = codes;
        s[gb0 + lb] = (uint8_t)sc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&freeb[b]);
    }
    if (!ok && lane == 0) fail();
  }
  __syncthreads();
}

// w = e2m1 * e4m3 * G rounded once to fp32: e2m1 * e4m3 is exact in f16/f32,
// so the only rounding is the final multiply by G.  One thread per 8 codes.
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ q,
                                                      const uint8_t* __restrict__ s,
                                                      const float* __restrict__ g,
                                                      int64_t groups_per_expert, int64_t n_groups,
                                                      float* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // group of 8 codes
  if (i >= n_groups) return;
  const int64_t e = i / groups_per_expert;
  const uint32_t w = *reinterpret_cast<const uint32_t*>(q + i * 4);
  const uint32_t sc = s[i >> 1];  // 16 codes per scale, 8 per group
  const float sv = e4m3_to_f32(sc);
  const float G = g[e];
  uint32_t h[4];
  e2m1x8_to_f16x2(w, h);
  float4 o0, o1;
  float v[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[j] & 0xFFFFu))) * sv, G);
    v[2 * j + 1] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[j] >> 16))) * sv, G);
  }
  o0 = make_float4(v[0], v[1], v[2], v[3]);
  o1 = make_float4(v[4], v[5], v[6], v[7]);
  float4* dst = reinterpret_cast<float4*>(out + i * 8);
  dst[0] = o0;
  dst[1] = o1;
}

namespace {

constexpr int kQSmem = kQHeader + kQBufs * kQMaxPiece + kQBufs * kQKeys * 2;
static_assert(kQSmem <= 232448, "shared memory budget of the single-pass quantiser");

// the single-pass kernel applies: the largest piece fits a buffer, every CTA
// gets a few blocks, and the workspace holds the arrival counters
bool single_pass_fits(int64_t E, int64_t bpe, int64_t ws_words, int sms) {
  return ws_words >= E + 3 && E <= (int64_t(1) << 24) && bpe >= 8 * (int64_t)sms &&
         (bpe + sms - 1) / sms * 32 <= kQMaxPiece;
}

cudaError_t launch_fused(const uint16_t* w, int64_t E, int64_t bpe, uint32_t* amax_ws, uint8_t* q, uint8_t* s,
                         float* g, int* status, int sms, uint32_t extra_target, uint64_t wait_ns,
                         cudaStream_t st) {
  cudaError_t err = configure_kernel_once((const void*)quantize_fused_kernel, kQSmem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sms);
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = (size_t)kQSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: the arrival waits end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_fused_kernel, w, (int)E, bpe, amax_ws, q, s, g, status, extra_target,
                            wait_ns);
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* q,
                            uint8_t* s, float* g, uint32_t* amax_ws, int64_t ws_words, int* status,
                            cudaStream_t st) {
  const int64_t per = N * K;
  const int64_t bpe = per / 16;
  int sms = 0;
  cudaError_t err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  const bool fused = single_pass_fits(E, bpe, ws_words, sms);
  err = cudaMemsetAsync(amax_ws, 0, sizeof(uint32_t) * (size_t)(fused ? E + 3 : E), st);
  if (err != cudaSuccess) return err;
  if (fused) {
    err = launch_fused(w, E, bpe, amax_ws, q, s, g, status, sms, 0u, kWaitTimeoutNs, st);
    // not every SM available to this context (a partitioned GPU): the two
    // passes below need no co-residency (their amax words are cleared too)
    if (err != cudaErrorCooperativeLaunchTooLarge) return err;
    (void)cudaGetLastError();
  }
  int gx = (int)((per / 8 + 255) / 256);
  if (gx > 64) gx = 64;
  const unsigned gy = (unsigned)(E < 65535 ? E : 65535);  // tensors beyond: grid-stride
  amax_kernel<<<dim3(gx, gy), 256, 0, st>>>(w, E, per, amax_ws);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t nb = E * bpe;
  encode_kernel<<<(unsigned)((nb + 255) / 256), 256, 0, st>>>(w, bpe, nb, amax_ws, q, s, g);
  return cudaGetLastError();
}

cudaError_t launch_quantize_timeout_selftest(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* q,
                                             uint8_t* s, float* g, uint32_t* amax_ws, int64_t ws_words,
                                             int* status, uint64_t wait_ns, cudaStream_t st) {
  const int64_t bpe = N * K / 16;
  int sms = 0;
  cudaError_t err = sm_count(&sms);
  if (err != cudaSuccess) return err;
  if (!single_pass_fits(E, bpe, ws_words, sms)) return cudaErrorNotSupported;
  err = cudaMemsetAsync(amax_ws, 0, sizeof(uint32_t) * (size_t)(E + 3), st);
  if (err != cudaSuccess) return err;
  return launch_fused(w, E, bpe, amax_ws, q, s, g, status, sms, 1u, wait_ns, st);
}

cudaError_t launch_dequantize(const uint8_t* q, const uint8_t* s, const float* g, int64_t E,
                              int64_t N, int64_t K, float* out, cudaStream_t st) {
  const int64_t gpe = N * K / 8, ng = E * gpe;
  dequant_kernel<<<(unsigned)((ng + 255) / 256), 256, 0, st>>>(q, s, g, gpe, ng, out);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
