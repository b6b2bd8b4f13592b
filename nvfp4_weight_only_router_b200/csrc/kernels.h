// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4moe {

// amax_ws: ws_words zero-initialised-by-the-call words; E + 3 or more enables
// the single-pass kernel (E amax words + 3 arrival counters), else two passes
cudaError_t launch_quantize(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* q,
                            uint8_t* s, float* g, uint32_t* amax_ws, int64_t ws_words, int* status,
                            cudaStream_t st);
// The single-pass kernel of launch_quantize with a cross-CTA arrival count
// that cannot be met and every wait limited to wait_ns: the failure path of
// the bounded waits (cudaErrorNotSupported if the shape does not take the
// single-pass kernel).
cudaError_t launch_quantize_timeout_selftest(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* q,
                                             uint8_t* s, float* g, uint32_t* amax_ws, int64_t ws_words,
                                             int* status, uint64_t wait_ns, cudaStream_t st);
// the library's device status word of the current device (null on failure)
int* device_status_ptr();
// Record `e` as the calling thread's last CUDA error (what
// nvfp4_last_cuda_error reports) and return NVFP4_ERR_CUDA.
int fail_cuda(cudaError_t e);
// Raise a kernel's dynamic shared-memory limit to smem_bytes (and allow
// non-portable cluster sizes if asked) once per kernel and device; safe to
// call from several host threads.
cudaError_t configure_kernel_once(const void* fn, int smem_bytes, bool nonportable_cluster = false);
// Number of SMs of the current device.
cudaError_t sm_count(int* sms);
cudaError_t launch_dequantize(const uint8_t* q, const uint8_t* s, const float* g, int64_t E,
                              int64_t N, int64_t K, float* out, cudaStream_t st);

struct RouteArgs {
  const uint16_t* x;      // bf16 [T, H]
  const uint16_t* proj;   // bf16 [E, H]
  const uint16_t* scale;  // bf16 [H]
  const uint16_t* pes;    // bf16 [E]
  const float* bias;      // f32 [E] or null
  int T, H;               // H: 8 to 16 slices of 256
  bool few_tokens;        // T <= 256: clusters of H/256 CTAs per 16 tokens (else 32 tokens per CTA)
  float eps, inv_sqrt_h;
  int32_t* ids;           // [T, 8]
  float* wts;             // [T, 8]
  // optional fused permutation (few tokens, T*8 <= 1024): meta (route counter
  // zero on entry), sorted_slot [T*8], slot_pos [T*8]; meta == null -> not fused
  int* meta;
  int* sorted_slot;
  int* slot_pos;
  int* status;
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);

struct PermuteArgs {
  const int32_t* ids;  // [S]
  int S, nchunks;
  int* meta;           // kMetaInts ints (written: counts, offsets, active list)
  int* chunk_count;    // [nchunks, 128] per-chunk counts (scratch)
  int* sorted_slot;    // [S]
  int* slot_pos;       // [S]
  int* status;
};
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st);
// The dense over-read's permutation: every token t to every expert e, slot
// t*128 + e at sorted position e*T + t, with weight w_tj if e = ids[t, j] for
// some j and 0 otherwise.  meta gets counts T, offsets e*T and all experts
// active.
cudaError_t launch_dense_permute(const int32_t* ids, const float* wts, int T, int* meta, int* sorted_slot,
                                 int* slot_pos, float* wdense, int* status, cudaStream_t st);

struct ExpertArgs {
  int codec;                // kCodecNvfp4 or kCodecAff4
  const uint8_t* gu_q;
  const uint8_t* gu_s;      // NVFP4: e4m3 [E, 2I, H/16]; aff4: fp16 scales [E, 2I, H/32]
  const float* gu_g;        // NVFP4: FP32 global [E]; aff4: unused
  const uint16_t* gu_b;     // aff4: fp16 biases [E, 2I, H/32]
  const uint8_t* dn_q;
  const uint8_t* dn_s;
  const float* dn_g;
  const uint16_t* dn_b;
  // optional packed codes (moe_nvfp4_pack_codes); null: read gu_q / dn_q by TMA
  const uint8_t* gu_pk;
  const uint8_t* dn_pk;
  const uint16_t* x;        // bf16 [T, H] (the layer input)
  __half* xs;               // [S, H] activations in expert-sorted slot order
  const int* meta;
  // [S] per sorted slot: e_t of the slot's token (the f16 operand prescale:
  // x enters as x * 2^(15 - e_t), h as h * 2^(-2 h_exp(e_t)))
  int* xexp;
  const int* sorted_slot;   // [S]
  const int* slot_pos;      // [S]
  const float* wts;         // [S]
  __half* h;                // [S, I], rows in sorted order
  float* obuf;              // [S, H] per-slot weighted outputs, sorted order
  void* y;                  // bf16 [T, H]
  int T, max_active;
  int spt;                  // slots per token: 8 (top-8), or 128 (the dense over-read, every expert)
  int* status;
};
// y[t] = bf16(sum over the token's 8 slots of obuf, in slot order)
cudaError_t launch_finalize(const ExpertArgs& a, cudaStream_t st);
// persistent streaming GEMVs (few tokens per expert): register dequant + warp MMA
cudaError_t launch_gate_up_stream(const ExpertArgs& a, cudaStream_t st);
cudaError_t launch_down_stream(const ExpertArgs& a, cudaStream_t st);
// tcgen05 grouped GEMMs with the dequantised weights in tensor memory;
// nt = tokens per tile (16, 64 or 192)
cudaError_t launch_gather_sorted(const ExpertArgs& a, cudaStream_t st);
cudaError_t launch_moe_gate_up(const ExpertArgs& a, int nt, cudaStream_t st);
cudaError_t launch_moe_down(const ExpertArgs& a, int nt, cudaStream_t st);

// W4A4 experts on the block-scaled FP4 tensor cores (w4a4.cu).
// Tokens per tile for T tokens (16, 64 or 128).
int w4a4_tile_tokens(int T);
// Packed block scales / codes of one projection (kind 0 gate_up, 1 down) of E experts.
cudaError_t launch_w4a4_pack_scales(const uint8_t* s, int E, int kind, uint8_t* out, cudaStream_t st);
// Codes of one projection in 128-row x 256-element tiles, 128-byte swizzled
// (moe_nvfp4_pack_codes), and their size.
cudaError_t launch_pack_codes(const uint8_t* q, int E, int kind, uint8_t* out, cudaStream_t st);
size_t packed_code_bytes(int E, int kind);
// Each token's x -> E2M1 codes aq (tile-major, 128-byte swizzled) and scale
// chunks asf (static global gx) at the padded rows of its 8 slots, and each
// slot's routing weight at its padded row of roww [max_tiles*nt].
cudaError_t launch_w4a4_act_quant(const uint16_t* x, const int* meta, const int* slot_pos, const float* wts, int T,
                                  float gx, int nt, uint8_t* aq, uint8_t* asf, float* roww, int* status,
                                  cudaStream_t st);
struct W4A4Args {
  const uint8_t* wq;        // packed weight codes of this GEMM
  const uint8_t* wsf;       // its packed scales
  const float* wg;          // its FP32 globals [E]
  float gin;                // global of its input (Gx for gate_up, Gh for down)
  float gh;                 // gate_up: the global the hidden is quantised under
  const uint8_t* aq;        // input codes, tile-major [max_tiles][K/256][nt][128 B]
  const uint8_t* asf;       // input scale chunks
  uint8_t* hq;              // gate_up: hidden codes, tile-major [max_tiles][3][nt][128 B]
  uint8_t* hsf;             // gate_up: hidden scale chunks
  const int* meta;
  const float* roww;        // routing weight per padded row (0 for padding)
  float* obuf;              // down: per-slot rows [S, H] (x weight x G_d x Gh)
  int max_tiles;
  int* status;
};
// kind 0 gate_up (+ GELU gate + hidden quantisation), 1 down
cudaError_t launch_w4a4_gemm(const W4A4Args& a, int kind, int nt, cudaStream_t st);

// The full block's dense MLP GEMMs (bf16 x bf16 -> fp32 on tcgen05).
//   gate_up: w0 = gate [2112, H], w1 = up [2112, H], b0 = X [T, H] (bf16);
//            out [splits][T][2 * 2112]: gate rows 0..2111, then up rows
//   down:    w0 = down [H, 2112], b0 / b1 = the gated hidden's bf16 high and
//            low parts [T, 2112]; out [splits][T][H]
// Each K split writes its own slab of out (the consumer sums them in order).
struct DenseArgs {
  const void* w0;
  const void* w1;
  const void* b0;
  const void* b1;
  float* out;
  int T;
  int splits;               // K splits (dense_splits for this T, or fewer)
  int* status;
};
cudaError_t launch_dense_gate_up(const DenseArgs& a, cudaStream_t st);
cudaError_t launch_dense_down(const DenseArgs& a, cudaStream_t st);
// K splits that give every one of `sms` SMs a tile for T tokens (mode 0
// gate_up, 1 down); 1 when the row and token tiles already do.
int dense_splits(int mode, int T, int sms);

// The full block's per-token kernels.
cudaError_t launch_block_prenorm(const uint16_t* x, const uint16_t* g1, const uint16_t* g2, float eps, int T,
                                 uint16_t* x1, uint16_t* x2, cudaStream_t st);
cudaError_t launch_dense_act(const float* part, int splits, int T, uint16_t* hi, uint16_t* lo, cudaStream_t st);
struct BlockFinalArgs {
  const uint16_t* x;        // bf16 [T, H] the residual
  const float* obuf;        // [S, H] per-slot rows of the sparse branch (x w x G_d)
  const int* slot_pos;      // [T*8]
  const float* dense;       // [splits, T, H] dense-branch partials
  int splits, T;
  const uint16_t* post1;    // post_feedforward_layernorm_1 weight
  const uint16_t* post2;    // post_feedforward_layernorm_2 weight
  const uint16_t* post;     // post_feedforward_layernorm weight
  const uint16_t* layer_scalar;
  float eps;
  void* y;                  // bf16 [T, H]
};
cudaError_t launch_block_final(const BlockFinalArgs& a, cudaStream_t st);

// 2-D TMA tensor map: `inner` elements per row, `outer` rows, `pitch` bytes
// between rows, box of box_inner x box_outer; false if the driver refuses it.
bool encode_tma_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t pitch, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
// 3-D TMA tensor map: dims innermost first, pitch[i] = bytes between steps of dim i+1.
bool encode_tma_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, const uint64_t (&dims)[3],
                   const uint64_t (&pitch)[2], const uint32_t (&box)[3], CUtensorMapSwizzle sw);

cudaError_t launch_residual_rmsnorm(float* res, const uint16_t* y, uint16_t* x_out, int T, int H,
                                    float eps, cudaStream_t st);

}  // namespace nvfp4moe
