// Shared device helpers of the NVFP4 MoE library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4moe {

// Layer constants of the Gemma-4-26B-A4B MoE branch ("Gemma 4 26B-A4B (MoE) -
// Core AI", "Architecture" table).
constexpr int kH = 2816;          // hidden size
constexpr int kI = 704;           // moe_intermediate_size
constexpr int kE = 128;           // routed experts
constexpr int kTopK = 8;          // experts per token
constexpr int kBlock = 16;        // elements per E4M3 block scale
constexpr int kDenseI = 2112;     // the full block's dense MLP intermediate_size

// Packed row geometry.
constexpr int kGuRowBytes = kH / 2;        // 1408: one gate_up row, two codes per byte
constexpr int kGuScaleRow = kH / kBlock;   // 176
constexpr int kDnRowBytes = kI / 2;        // 352
constexpr int kDnScaleRow = kI / kBlock;   // 44

// A "segment" is 128 consecutive K elements = 64 packed bytes: four lanes of a
// quad each hold one 16-byte chunk (32 elements) of it.
constexpr int kSegK = 128;
constexpr int kGuSegs = kH / kSegK;              // 22
constexpr int kDnSegs = (kI + kSegK - 1) / kSegK; // 6 (the last one half full)

// Expert weight codecs.
constexpr int kCodecNvfp4 = 0;  // E2M1 codes, E4M3 scale per 16, FP32 global per expert
constexpr int kCodecAff4 = 1;   // u4 codes, fp16 scale and bias per 32

// Device status codes (mirror nvfp4_status).
constexpr int kStatusTimeout = 5;
constexpr int kStatusDevice = 7;
constexpr int kStatusRange = 8;

// Layout of the small integer "meta" block at the start of a forward
// workspace.
constexpr int kMetaCounts = 0;      // [E] tokens routed to each expert
constexpr int kMetaOffsets = 128;   // [E+1] exclusive prefix of counts
constexpr int kMetaAct = 260;       // [E] ids of experts with count > 0, ascending
constexpr int kMetaNAct = 388;      // number of active experts
constexpr int kMetaRouteCounter = 396; // arrival counter of the router's token tiles
constexpr int kMetaInts = 512;

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------- conversions
// Four packed bytes (eight E2M1 codes) -> four f16x2 registers.  Register i
// holds byte i: its low nibble in the low half, its high nibble in the high
// half.  The conversion is exact (every E2M1 value is an f16).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// Four packed bytes (eight unsigned 4-bit aff4 codes q, element 2i in the low
// nibble of byte i) -> four f16x2 registers of q * scale + bias, register i
// holding elements 2i (low half) and 2i+1 (high half).  Each code first
// becomes the f16 1024 + q (q placed in the mantissa under the exponent of
// 1024), 1024 is subtracted exactly, and one f16x2 fma applies the block's
// scale and bias (s2, b2: each broadcast to both halves), so the weight is
// rounded once to f16.
__device__ __forceinline__ void u4x8_affine_f16x2(uint32_t w, uint32_t s2, uint32_t b2, uint32_t (&o)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t x01 = __byte_perm(lo, hi, 0x5140);  // elements 0, 1, 2, 3 as bytes
  const uint32_t x23 = __byte_perm(lo, hi, 0x7362);  // elements 4, 5, 6, 7
  const uint32_t e = 0x64646464u;                    // high byte of the f16 1024
  uint32_t q[4];
  q[0] = __byte_perm(x01, e, 0x4140);
  q[1] = __byte_perm(x01, e, 0x4342);
  q[2] = __byte_perm(x23, e, 0x4140);
  q[3] = __byte_perm(x23, e, 0x4342);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t t;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(q[i]), "r"(0x64006400u));  // exact: q
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(o[i]) : "r"(t), "r"(s2), "r"(b2));
  }
}

// Two E4M3 bytes (low byte first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t o;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(o) : "h"(v));
  return o;
}

// f16x2 multiply (used on exact products only: e2m1 * e4m3 fits in f16).
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t o;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o) : "r"(a), "r"(b));
  return o;
}

// Broadcast the low / high half of an f16x2 to both halves.
__device__ __forceinline__ uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, v, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, v, 0x3232); }

// fp32 -> f16 with saturation to +-65504 (finite inputs); `over` is set
// when the value lies beyond the f16 range (|v| >= 65520 would round to
// infinity), i.e. when the saturation changed the result.
__device__ __forceinline__ __half f32_to_f16_sat(float v, bool& over) {
  over |= fabsf(v) >= 65520.0f;
  v = fminf(fmaxf(v, -65504.0f), 65504.0f);
  return __float2half_rn(v);
}

// 2^k as an fp32 value, for -126 <= k <= 127 (exact).
__device__ __forceinline__ float exp2i(int k) { return __int_as_float((k + 127) << 23); }

// Power-of-two prescale of the expert GEMMs' f16 operands.  Token t's
// activation row enters the tensor cores as x * 2^(15 - e_t) and its gated
// hidden rows as h * 2^(-2 e_h), with e_t = floor(log2 max|x_t|) clamped to
// [kXExpMin, kXExpMax] and e_h = e_t clamped to [-kHExpLim, kHExpLim]; the
// epilogues multiply the fp32 accumulators back by the inverse powers of two,
// so the scaling is exact.  Scaled, every bf16 element of a row whose maximum
// lies in [2^-111, 2^113) is exact in f16 down to 2^-32 of the row maximum,
// and h keeps its f16 precision whatever the magnitude of x (h grows as x^2).
constexpr int kXExpMin = -111, kXExpMax = 112, kHExpLim = 63;
__device__ __forceinline__ int h_exp(int e) { return max(-kHExpLim, min(kHExpLim, e)); }

__device__ __forceinline__ uint32_t pack_f16x2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// ------------------------------------------------------------- tensor cores
// D += A * B, m16n8k16, f16 inputs, f32 accumulators (legacy warp-level MMA;
// used for the bandwidth-bound decode GEMVs where the MMA pipe is not the
// bottleneck).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------- memory
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ldg_nc_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// GELU, tanh form: 0.5 g (1 + tanh(a)), a = sqrt(2/pi) (g + 0.044715 g^3),
// evaluated through the identity 0.5 (1 + tanh(a)) = 1 / (1 + exp(-2a)).
// The exponential (__expf, relative error ~2^-21) keeps the result within a
// few fp32 ulps of the tanh expression; exp overflow for very negative g gives
// the correct limit 0.
__device__ __forceinline__ float gelu_tanh(float g) {
  const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
  const float k1 = 0.044715f;
  const float a = k0 * (g + k1 * g * g * g);
  return g / (1.0f + __expf(-2.0f * a));
}

}  // namespace nvfp4moe

namespace nvfp4moe {

// ------------------------------------------------------- async bulk copies
// Shared-memory mbarrier helpers and the 1-D bulk (TMA) global->shared copy.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// make barrier initialisation visible to the async proxy before first use
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wall-time limits of the bounded device-side waits.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s: a pipeline wait that never completes
constexpr uint64_t kAbortDrainNs = 200000000ull;    // 0.2 s: draining copies after an abort

// Bounded wait: returns false if the phase did not complete within
// `timeout_ns` of wall time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
}

__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory loads.  Not volatile, so the compiler may schedule them
// among register-only work; the "memory" clobber keeps them after the
// barrier waits (volatile, memory-clobbering asm) that publish the data.
__device__ __forceinline__ uint4 lds_v4(const void* p) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "r"(smem_u32(p))
      : "memory");
  return v;
}

}  // namespace nvfp4moe
