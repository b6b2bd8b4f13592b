/*
 * nvfp4moe.h -- C ABI of the NVFP4 weight-only (W4A16) sparse MoE branch for
 * NVIDIA B200 (sm_100a).
 *
 * The branch is the sparse half of a Gemma-4-26B-A4B decoder layer
 * ("Gemma 4 26B-A4B (MoE) - Core AI" card, "Architecture": hidden 2816,
 * 128 experts, top-8, moe_intermediate 704; the layer dataflow listing and the
 * router description under it).  Expert weights are NVFP4 ("gemma-4-26B-A4B .
 * NVFP4A16" release card, "Quantization details"; "Gemma-4-26B-A4B-NVFP4-mlx",
 * "Quantization recipe"): E2M1 codes packed two per byte, one E4M3 block scale
 * per 16 consecutive elements along K, one FP32 global scale per expert
 * projection; w = e2m1 * e4m3 * fp32.  Activations are bf16.
 *
 * Conventions for every entry point
 *   - Pointers named *_dev are device pointers; the caller owns all memory.
 *     The library never allocates device memory; calls that need scratch
 *     take a caller-allocated workspace whose size a *_workspace_bytes query
 *     returns (for the same arguments).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call is asynchronous on that stream; none synchronises
 *     except nvfp4_get_device_status.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns an error status and enqueues nothing.
 *   - Every device pointer must be 16-byte aligned (NVFP4_ERR_ALIGNMENT
 *     otherwise) and workspaces 256-byte aligned.
 *   - Errors are returned, never thrown or printed.  A failed CUDA runtime
 *     call or launch is reported as NVFP4_ERR_CUDA; nvfp4_last_cuda_error
 *     gives the CUDA error behind it.
 *   - Calls that share a workspace must not overlap on the GPU.
 *
 * Tensor layouts (row-major, innermost last)
 *   x            bf16 [T, H]
 *   y            bf16 [T, H]
 *   router.proj  bf16 [E, H]     router.scale bf16 [H]
 *   router.per_expert_scale bf16 [E]      router.logit_bias f32 [E] or NULL
 *   gate_up_q    u8   [E, 2I, H/2]   rows 0..I-1 = gate, I..2I-1 = up
 *   gate_up_s    u8   [E, 2I, H/16]  E4M3 block scales
 *   gate_up_g    f32  [E]
 *   down_q       u8   [E, H, I/2]
 *   down_s       u8   [E, H, I/16]
 *   down_g       f32  [E]
 * Byte j of a packed row holds element 2j in its low nibble and element 2j+1
 * in its high nibble.  The sign bit of an E2M1 code is bit 3.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVFP4MOE_ABI_VERSION 3

#if defined(__GNUC__)
#define NVFP4MOE_API __attribute__((visibility("default")))
#else
#define NVFP4MOE_API
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,   /* null pointer, non-positive or inconsistent size */
  NVFP4_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte (workspace: 256-byte) aligned */
  NVFP4_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the query returned */
  NVFP4_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  NVFP4_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (device status) */
  NVFP4_ERR_UNSUPPORTED = 6,   /* valid but not implemented shape (see each call) */
  NVFP4_ERR_DEVICE = 7,        /* a kernel detected bad input data (device status) */
  NVFP4_ERR_RANGE = 8          /* an activation left the f16 operand range and was
                                  saturated (device status; see moe_nvfp4_forward) */
} nvfp4_status;

/* Router parameters ("Gemma 4 26B-A4B (MoE) - Core AI", router description
 * under the layer dataflow listing).  All pointers are device pointers. */
typedef struct {
  const void* proj;              /* bf16 [E, H] */
  const void* scale;             /* bf16 [H] */
  const void* per_expert_scale;  /* bf16 [E] */
  const float* logit_bias;       /* f32 [E], added to the logits; NULL = none */
  int32_t E;                     /* number of experts: must be 128 */
  int32_t H;                     /* hidden size: a multiple of 256 in [2048, 4096] */
  int32_t top_k;                 /* must be 8 */
  float eps;                     /* RMSNorm epsilon (the pages are silent; 1e-6) */
} moe_router;

/* NVFP4 expert stacks.  All pointers are device pointers.  gate_up_pk and
 * down_pk are optional (NULL = absent): the same codes copied once by
 * moe_nvfp4_pack_codes into whole 16 KB tiles, which the decode kernels then
 * stream as contiguous blocks instead of gathering 128-byte row pieces;
 * moe_w4a4_forward requires them. */
typedef struct {
  const uint8_t* gate_up_q;  /* [E, 2I, H/2] */
  const uint8_t* gate_up_s;  /* [E, 2I, H/16] */
  const float* gate_up_g;    /* [E] */
  const uint8_t* down_q;     /* [E, H, I/2] */
  const uint8_t* down_s;     /* [E, H, I/16] */
  const float* down_g;       /* [E] */
  int32_t E;                 /* must be 128 */
  int32_t H;                 /* must be 2816 */
  int32_t I;                 /* must be 704 */
  const uint8_t* gate_up_pk; /* moe_pack_bytes(E, 0) bytes, or NULL */
  const uint8_t* down_pk;    /* moe_pack_bytes(E, 1) bytes, or NULL */
} moe_experts;

/* Bytes of the packed gate_up codes (which = 0), down codes (1), gate_up
 * block scales in the FP4 tensor core's order (2) or down block scales (3)
 * of E experts (0 for E < 1 or another `which`). */
NVFP4MOE_API size_t moe_pack_bytes(int32_t E, int32_t which);

/* moe_nvfp4_pack_codes: copies experts->gate_up_q / down_q into
 * gate_up_pk_dev / down_pk_dev (moe_pack_bytes(E, 0 / 1) bytes, device,
 * 16-byte aligned, caller-owned): per expert, per 128-row tile of the
 * projection and per 256 elements of K, the tile's codes as 128 rows of 128
 * bytes in the 128-byte swizzle (16-byte piece p of tile row r stored at
 * piece p ^ (r % 8)); bytes past a row's end are zero.  Gate_up tile j holds,
 * for each quarter q = 0..3, the gate rows of hidden units 64 j + 16 q ..
 * + 15 followed by their 16 up rows; down tile j holds rows 128 j .. + 127.
 * Run once per set of weights; asynchronous on `stream`.  Same shape
 * requirements as moe_nvfp4_forward (the packed pointers of `experts` are
 * ignored). */
NVFP4MOE_API nvfp4_status moe_nvfp4_pack_codes(const moe_experts* experts, uint8_t* gate_up_pk_dev,
                                               uint8_t* down_pk_dev, void* stream);

/* ---------------------------------------------------------------------------
 * nvfp4_quantize: bf16 weights -> NVFP4.
 * Source: "Gemma-4-26B-A4B-it-NVFP4" page, block-scale formulas (S_block =
 * max|w|/6, q = clip(round(w/S), -6, 6)), in the two-level form of the
 * NVFP4A16 card ("Quantization details").  For each tensor e (one per expert):
 *   G      = f32(amax_e) / 2688                    (2688 = 6 * 448)
 *   s_b    = E4M3_rne_satfinite((amax_b / 6) / G)  per block of 16 along K
 *   d_b    = f32(s_b) * G
 *   code_i = E2M1_rne(w_i / d_b), saturating at 6, sign bit = sign bit of w_i
 * each step one correctly rounded fp32 operation; ties go to the even code.
 * A block with d_b == 0 (all-zero block or tensor) gets scale 0 and codes that
 * carry only the sign bit.
 *   w_dev  bf16 [E, N, K] (in)      q_dev u8 [E, N, K/2] (out)
 *   s_dev  u8 [E, N, K/16] (out)    g_dev f32 [E] (out)
 * Requires E >= 1, N >= 1, K >= 16, K % 32 == 0, N * K < 2^31.  NaN/Inf
 * inputs are not supported (their codes are unspecified).
 * Workspace: nvfp4_quantize_workspace_bytes(E, N, K) bytes, 256-aligned
 * (E amax words and three arrival counters; the call clears what it uses).
 * Execution: when one tensor's share per SM fits on chip (N * K / 16 blocks
 * of 32 bytes split over all SMs, at most 1700 blocks each, and at least 8
 * blocks per SM) the call is one cooperative launch of one CTA per SM that reads
 * every weight once; it occupies the whole GPU while it runs (if the
 * context cannot hold one CTA on every SM at once, the call takes the two
 * passes instead).  Other shapes take two passes (amax, then encode).  Both
 * give the same bytes.
 * ------------------------------------------------------------------------- */
NVFP4MOE_API size_t nvfp4_quantize_workspace_bytes(int64_t E, int64_t N, int64_t K);
NVFP4MOE_API nvfp4_status nvfp4_quantize(const void* w_dev, int64_t E, int64_t N, int64_t K,
                            uint8_t* q_dev, uint8_t* s_dev, float* g_dev,
                            void* ws_dev, size_t ws_bytes, void* stream);

/* nvfp4_quantize_noalloc: nvfp4_quantize for callers that cannot allocate
 * device memory when they quantise -- for instance a plugin whose host
 * framework owns all device memory and forbids allocation inside its execute
 * callback, or a latency-critical path that must not enter an allocator.  It
 * takes no workspace: the per-tensor amax scratch lives in a fixed 16 KiB
 * device array inside the library (held on every GPU that loads the library
 * until the process exits), and the call allocates nothing (no cudaMalloc,
 * no allocating library routine).  The pages have no counterpart of this
 * entry point; it exists for such callers only.
 * Same arguments, layouts, results and limits as nvfp4_quantize, plus
 * E <= 4096 (NVFP4_ERR_UNSUPPORTED beyond).  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress, with that device
 * current); make that first call before any stream capture.  With CUDA's
 * default lazy module loading, that first call on each device (or loading the
 * library, with CUDA_MODULE_LOADING=EAGER) is also when the driver places the
 * array and the library's code on the device: callers with a strict
 * no-allocation window make one call before the window opens.  All calls on a
 * device share the array, which keeps the last call's contents (each call
 * clears what it needs): calls that overlap on the GPU race. */
NVFP4MOE_API nvfp4_status nvfp4_quantize_noalloc(const void* w_dev, int64_t E, int64_t N, int64_t K,
                                                 uint8_t* q_dev, uint8_t* s_dev, float* g_dev,
                                                 void* stream);

/* nvfp4_dequantize: w = e2m1 * e4m3 * G rounded once to fp32 ("Gemma-4-26B-A4B-
 * NVFP4-mlx", "Quantization recipe": E2M1 x per-16 E4M3 x per-tensor F32).
 * Same layouts and limits as nvfp4_quantize; out_dev f32 [E, N, K].  No
 * workspace. */
NVFP4MOE_API nvfp4_status nvfp4_dequantize(const uint8_t* q_dev, const uint8_t* s_dev, const float* g_dev,
                              int64_t E, int64_t N, int64_t K, float* out_dev, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route: the router ("Gemma 4 26B-A4B (MoE) - Core AI", router
 * description): r = x / sqrt(mean(x^2) + eps) * scale * H^-0.5;
 * logits = proj r (+ logit_bias); p = softmax(logits) in fp32 over all E;
 * the top_k largest p; weights = p_sel / sum(p_sel) * per_expert_scale[ids].
 * fp32 arithmetic throughout (the x*scale products are carried exactly).
 *   x_dev    bf16 [T, H] (in)
 *   ids_dev  int32 [T, top_k] (out), by descending p; the selection compares
 *            the fp32 logits (softmax is monotone), equal logits -> lower id first
 *   w_dev    f32 [T, top_k] (out)
 * Requires 1 <= T <= 65536, E == 128, top_k == 8, H % 256 == 0 and
 * 2048 <= H <= 4096 (NVFP4_ERR_UNSUPPORTED otherwise).
 * Workspace: moe_route_workspace_bytes(T, router) bytes (the kernels keep
 * their scratch on chip; the query returns 256).
 * ------------------------------------------------------------------------- */
NVFP4MOE_API size_t moe_route_workspace_bytes(int32_t T, const moe_router* router);
NVFP4MOE_API nvfp4_status moe_route(const void* x_dev, int32_t T, const moe_router* router,
                       int32_t* ids_dev, float* w_dev,
                       void* ws_dev, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_nvfp4_forward: y = sum_j w_j * expert_{id_j}(x) for every token
 * ("Gemma 4 26B-A4B (MoE) - Core AI", layer dataflow listing: the experts'
 * outputs combined as sum_k w_k h2_k; experts GELU-tanh gated).  Both the
 * router and the experts read x.  Per expert e and routed token x:
 *   gate = G_gu[e] * (Wq_gate[e] x),  up = G_gu[e] * (Wq_up[e] x)
 *   h    = gelu_tanh(gate) * up
 *   out  = G_d[e] * (Wq_down[e] h)
 * where Wq = e2m1 * e4m3 is exact in f16.  x and h enter the tensor cores as
 * f16 under an exact power-of-two prescale per token: with e_t = floor(log2
 * max|x_t|), x_t enters as x_t * 2^(15 - e_t) (every bf16 element down to
 * 2^-32 of the row maximum is exact) and h as h * 2^(-2 e_t) rounded to f16
 * (h grows as x^2, so its f16 precision does not depend on the size of x);
 * the fp32 epilogues undo both scalings.  Products are accumulated in fp32,
 * the combine is fp32, y is rounded once to bf16.  A row maximum outside
 * [2^-111, 2^113), or a scaled h beyond the f16 range (|h| >= 65520 *
 * 2^(2 e_t): weights whose gated outputs exceed ~65000 for an input of unit
 * maximum), saturates and records NVFP4_ERR_RANGE in the device status.
 * x must be finite.
 *   x_dev bf16 [T, H] (in), y_dev bf16 [T, H] (out)
 * When experts->gate_up_pk / down_pk are set (moe_nvfp4_pack_codes), the
 * decode kernels (T <= 256) read the codes from them; the result is the same
 * bit for bit.  Both or neither must be set (NVFP4_ERR_INVALID_ARG).
 * Requires 1 <= T <= 65536, E == 128, H == 2816, I == 704, top_k == 8.
 * Workspace: moe_forward_workspace_bytes(T, experts, router) bytes.
 * ------------------------------------------------------------------------- */
NVFP4MOE_API size_t moe_forward_workspace_bytes(int32_t T, const moe_experts* experts, const moe_router* router);
NVFP4MOE_API nvfp4_status moe_nvfp4_forward(const void* x_dev, int32_t T, const moe_experts* experts,
                               const moe_router* router, void* y_dev,
                               void* ws_dev, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_aff4_forward: moe_nvfp4_forward with the experts in the aff4 codec
 * ("Gemma 4 26B-A4B (MoE) - Core AI", "Compression recipe": affine int4 with
 * an fp16 scale and bias per (output row, K-block of 32); a q4_0 grid
 * w = (q - 8) d is the block with scale = d, bias = -8 d):
 *   w = q * scale + bias,  q the unsigned 4-bit code.
 * The same router, permutation, grouped kernels, combine and output; each
 * weight is formed in f16 by one fma (rounded once) before the MMA.
 *   gate_up_q u8 [E, 2I, H/2]  (rows 0..I-1 gate, I..2I-1 up; element 2j in
 *             the low nibble of byte j)
 *   gate_up_s, gate_up_b fp16 [E, 2I, H/32]
 *   down_q u8 [E, H, I/2];  down_s, down_b fp16 [E, H, I/32]
 * Same requirements and workspace size as moe_nvfp4_forward
 * (moe_aff4_forward_workspace_bytes). */
typedef struct {
  const uint8_t* gate_up_q;
  const void* gate_up_s;   /* fp16 */
  const void* gate_up_b;   /* fp16 */
  const uint8_t* down_q;
  const void* down_s;      /* fp16 */
  const void* down_b;      /* fp16 */
  int32_t E;               /* must be 128 */
  int32_t H;               /* must be 2816 */
  int32_t I;               /* must be 704 */
} moe_experts_aff4;
NVFP4MOE_API size_t moe_aff4_forward_workspace_bytes(int32_t T, const moe_experts_aff4* experts,
                                                     const moe_router* router);
NVFP4MOE_API nvfp4_status moe_aff4_forward(const void* x_dev, int32_t T, const moe_experts_aff4* experts,
                                           const moe_router* router, void* y_dev, void* ws_dev, size_t ws_bytes,
                                           void* stream);

/* moe_nvfp4_forward_dense: the same output as moe_nvfp4_forward computed the
 * way a runtime without a gather kernel does it ("Gemma 4 26B-A4B (MoE) -
 * Core AI", "Compression recipe": without the gather kernel the sparse
 * branch becomes a dense matmul that reads all 128 experts every token, a 16x
 * over-read; "Performance": 140 vs 39 tok/s for another MoE through its
 * gather kernel and as the dense over-read).  Every token goes through every
 * expert, each expert's output weighted by the token's routing weight for it
 * (0 for the 120 experts the router did not select), so all 128 experts'
 * weights are read for any T.  An ablation for measuring the gather's
 * advantage, not a path to deploy.  Same arguments and layouts as
 * moe_nvfp4_forward; requires 1 <= T <= 256.  Workspace:
 * moe_forward_dense_workspace_bytes(T, experts, router) bytes. */
NVFP4MOE_API size_t moe_forward_dense_workspace_bytes(int32_t T, const moe_experts* experts,
                                                      const moe_router* router);
NVFP4MOE_API nvfp4_status moe_nvfp4_forward_dense(const void* x_dev, int32_t T, const moe_experts* experts,
                                                  const moe_router* router, void* y_dev,
                                                  void* ws_dev, size_t ws_bytes, void* stream);

/* moe_nvfp4_forward_profiled: moe_nvfp4_forward that also records CUDA
 * events between its phases on `stream`.  phase_events points to 6 cudaEvent_t
 * (passed as void*; a NULL entry is skipped): [0] before the first kernel,
 * [1] after the router, [2] after the permutation, [3] after gate_up + GELU,
 * [4] after down, [5] after the combine.  Results are identical to
 * moe_nvfp4_forward. */
NVFP4MOE_API nvfp4_status moe_nvfp4_forward_profiled(const void* x_dev, int32_t T,
                                                     const moe_experts* experts,
                                                     const moe_router* router, void* y_dev,
                                                     void* ws_dev, size_t ws_bytes, void* stream,
                                                     void* const* phase_events);

/* Byte offsets, inside a forward workspace, of the intermediate results a
 * finished moe_nvfp4_forward leaves behind (for inspection and tests):
 *   ids int32 [T, 8], weights f32 [T, 8] (the router's outputs),
 *   counts int32 [E], offsets int32 [E+1] (exclusive prefix of counts),
 *   sorted_slot int32 [T*8] (slots t*8+j grouped by expert, stable),
 *   slot_pos int32 [T*8] (inverse permutation),
 *   xexp int32 [T*8] (e_t of each sorted slot's token: the prescale exponent),
 *   h f16 [T*8, I] (gated hidden, rows in sorted_slot order, row p holding
 *     h * 2^(-2 e) with e = xexp[p] clamped to [-63, 63]). */
typedef struct {
  size_t ids, weights, counts, offsets, sorted_slot, slot_pos, xexp, h;
} moe_forward_views;
NVFP4MOE_API nvfp4_status moe_forward_workspace_views(int32_t T, const moe_experts* experts,
                                         const moe_router* router, moe_forward_views* out);

/* ---------------------------------------------------------------------------
 * moe_block_forward: the full feed-forward half of a Gemma-4-26B-A4B decoder
 * layer ("Gemma 4 26B-A4B (MoE) - Core AI", the layer dataflow listing): a
 * dense GELU-gated MLP (intermediate 2112, "Architecture" table; bf16
 * weights, "Gemma-4-26B-A4B-NVFP4-mlx", "Quantization recipe") in parallel
 * with the NVFP4 sparse branch,
 *   h   = mlp(pre_ff_norm(x))                 h1 = post_ff_norm_1(h)
 *   ids, w = router(x)                        (the RAW residual)
 *   h2  = post_ff_norm_2(sum_k w_k expert_{ids_k}(pre_ff_norm_2(x)))
 *   y   = (x + post_ff_norm(h1 + h2)) * layer_scalar
 * Each norm is x / sqrt(mean(x^2) + eps) * weight (fp32).  The two MLP inputs
 * are rounded to bf16 (the modules' bf16 activations); the dense MLP runs on
 * the tensor cores with bf16 operands and fp32 accumulation, its gated
 * hidden entering the down projection as an exact bf16 high + low pair; the
 * experts as in moe_nvfp4_forward; all later steps in fp32; y is rounded
 * once to bf16.
 *   x_dev bf16 [T, H] (in: the post-attention hidden), y_dev bf16 [T, H] (out)
 * Requires 1 <= T <= 8192, the experts and router of moe_nvfp4_forward,
 * dense_I == 2112.  Workspace: moe_block_workspace_bytes(T, block) bytes.
 * ------------------------------------------------------------------------- */
typedef struct {
  moe_experts experts;
  moe_router router;
  const void* dense_gate;      /* bf16 [dense_I, H] */
  const void* dense_up;        /* bf16 [dense_I, H] */
  const void* dense_down;      /* bf16 [H, dense_I] */
  const void* pre_ff_norm;     /* bf16 [H] pre_feedforward_layernorm */
  const void* post_ff_norm_1;  /* bf16 [H] post_feedforward_layernorm_1 */
  const void* pre_ff_norm_2;   /* bf16 [H] pre_feedforward_layernorm_2 */
  const void* post_ff_norm_2;  /* bf16 [H] post_feedforward_layernorm_2 */
  const void* post_ff_norm;    /* bf16 [H] post_feedforward_layernorm */
  const void* layer_scalar;    /* bf16 [1] */
  int32_t dense_I;             /* must be 2112 */
  float eps;                   /* the five norms' epsilon (the pages are silent; 1e-6) */
} moe_block;
NVFP4MOE_API size_t moe_block_workspace_bytes(int32_t T, const moe_block* block);
NVFP4MOE_API nvfp4_status moe_block_forward(const void* x_dev, int32_t T, const moe_block* block, void* y_dev,
                                            void* ws_dev, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * W4A4: the routed experts with NVFP4 activations on the block-scaled FP4
 * tensor cores ("Gemma-4-26B-A4B-it-NVFP4": built for native FP4 tensor-core
 * execution, block-scale formulas; "Gemma-4-26B-A4B-NVFP4-mlx": the
 * checkpoint's `input_scale` sidecar, a static FP32 global per projection
 * input; "gemma-4-26B-A4B . NVFP4A16": W4A16 keeps BF16 activations and
 * forgoes this form's activation speed-up).
 * Each token's x is quantised once as a weight row is (blocks of 16 along H,
 * E4M3 scale s = e4m3_rn_satfinite((amax_b / 6) / Gx), E2M1 codes of x / (s Gx),
 * every step one correctly rounded fp32 operation) under the static global
 * Gx = input_scale_gate_up; per expert the gate_up GEMM multiplies the E2M1
 * codes of both operands with their E4M3 scales in the tensor core (fp32
 * accumulation), h = gelu_tanh(Gx G_gu g) * (Gx G_gu u) in fp32 is quantised
 * the same way per 16 hidden units under Gh = input_scale_down, the down GEMM
 * multiplies those codes with the down weights', o = w G_d Gh acc per slot,
 * and y[t] = bf16(sum over the token's 8 slots in slot order).
 *
 * The weights are those of moe_experts with their packed codes
 * (moe_nvfp4_pack_codes), plus their block scales copied once into the FP4
 * tensor core's order (moe_w4a4_pack_scales): per expert, per 128-row tile
 * (the packed codes' row order) and per 64 elements of K, one 512-byte chunk,
 * the scale of tile row r = r0 + 32 r1 and block i of the 64 at byte
 * 16 r0 + 4 r1 + i.
 * ------------------------------------------------------------------------- */
typedef struct {
  moe_experts experts;           /* moe_nvfp4_forward's, with gate_up_pk and down_pk set */
  const uint8_t* gate_up_sf;     /* moe_pack_bytes(E, 2) bytes from moe_w4a4_pack_scales */
  const uint8_t* down_sf;        /* moe_pack_bytes(E, 3) bytes */
  float input_scale_gate_up;     /* Gx > 0, finite */
  float input_scale_down;        /* Gh > 0, finite */
} moe_experts_w4a4;

/* moe_w4a4_pack_scales: copies experts->gate_up_s / down_s into
 * gate_up_sf_dev / down_sf_dev (moe_pack_bytes(E, 2 / 3) bytes, device,
 * 16-byte aligned, caller-owned) in the order above.  Run once per set of
 * weights; asynchronous on `stream`. */
NVFP4MOE_API nvfp4_status moe_w4a4_pack_scales(const moe_experts* experts, uint8_t* gate_up_sf_dev,
                                               uint8_t* down_sf_dev, void* stream);

/* moe_w4a4_forward: y_dev bf16 [T, H] from x_dev bf16 [T, H] as described
 * above; 1 <= T <= 65536, router and experts as for moe_nvfp4_forward.
 * Workspace: moe_w4a4_workspace_bytes(T, experts, router) bytes, 256-byte
 * aligned, caller-owned.  Errors as for moe_nvfp4_forward. */
NVFP4MOE_API size_t moe_w4a4_workspace_bytes(int32_t T, const moe_experts_w4a4* experts, const moe_router* router);
NVFP4MOE_API nvfp4_status moe_w4a4_forward(const void* x_dev, int32_t T, const moe_experts_w4a4* experts,
                                           const moe_router* router, void* y_dev, void* ws_dev, size_t ws_bytes,
                                           void* stream);

/* moe_w4a4_forward_profiled: moe_w4a4_forward that also records CUDA events
 * between its phases on `stream` (phase_events: 6 cudaEvent_t passed as
 * void*, NULL entries skipped): [0] before the first kernel, [1] after the
 * router, [2] after the permutation and the quantisation of x, [3] after
 * gate_up + GELU + the quantisation of h, [4] after down, [5] after the
 * combine.  Results are identical to moe_w4a4_forward. */
NVFP4MOE_API nvfp4_status moe_w4a4_forward_profiled(const void* x_dev, int32_t T, const moe_experts_w4a4* experts,
                                                    const moe_router* router, void* y_dev, void* ws_dev,
                                                    size_t ws_bytes, void* stream, void* const* phase_events);

/* Byte offsets inside a W4A4 workspace of what a finished moe_w4a4_forward
 * leaves behind.  Each expert's slots are padded to whole tiles of
 * tile_tokens rows: expert e's tiles start at tile p_e = sum over e' < e of
 * ceil(counts[e'] / tile_tokens), and its sorted slot offsets[e] + n is row
 * n' = (n mod tile_tokens) of tile p_e + n / tile_tokens.  Padding rows of x
 * are unspecified; those of h hold zero codes and scales.
 *   ids, weights, counts, offsets, sorted_slot, slot_pos: as moe_forward_views
 *   x_codes, h_codes: E2M1 codes (element 2k in the low nibble of byte k) per
 *     tile p and 256-element K chunk c, a block of tile_tokens rows of 128
 *     bytes at (p * C + c) * tile_tokens * 128 (C = 11 for x, 3 for h, whose
 *     rows end at byte 352 of 384), row r's byte k of the chunk at
 *     128 r + 16 ((k / 16) ^ (r % 8)) + k % 16
 *   x_scales, h_scales: per tile p and 64-element group g of the row, a
 *     512-byte chunk at (p * (H/64 or I/64) + g) * 512; the E4M3 scale of
 *     tile row r and block 4 g + i at byte 16 (r % 32) + 4 (r / 32) + i.
 * tile_tokens is 16 for T <= 256, 64 for T <= 1024, else 128. */
typedef struct {
  size_t ids, weights, counts, offsets, sorted_slot, slot_pos;
  size_t x_codes, x_scales, h_codes, h_scales;
  int32_t tile_tokens, max_tiles;
} moe_w4a4_views;
NVFP4MOE_API nvfp4_status moe_w4a4_workspace_views(int32_t T, const moe_experts_w4a4* experts,
                                                   const moe_router* router, moe_w4a4_views* out);

/* ---------------------------------------------------------------------------
 * moe_permute: the token permutation of moe_nvfp4_forward on its own -- the
 * T*8 routing slots s = t*8 + j grouped by expert with a stable counting sort
 * (the sort-by-expert step of the batched expert kernel, "Gemma 4 26B-A4B
 * (MoE) - Core AI", "Decode only ...").
 *   ids_dev         int32 [T, 8] (in), expert ids in [0, 128)
 *   counts_dev      int32 [128] (out), slots per expert
 *   offsets_dev     int32 [129] (out), exclusive prefix of counts
 *   sorted_slot_dev int32 [T*8] (out), slots grouped by expert, increasing
 *                   slot order within an expert
 *   slot_pos_dev    int32 [T*8] (out), inverse: sorted_slot[slot_pos[s]] == s
 * An id outside [0, 128) records NVFP4_ERR_DEVICE in the device status; that
 * slot is left out of every expert (slot_pos -1, not counted) and the entries
 * of sorted_slot past offsets[128] are unspecified.
 * Requires 1 <= T <= 65536.  Workspace: moe_permute_workspace_bytes(T).
 * ------------------------------------------------------------------------- */
NVFP4MOE_API size_t moe_permute_workspace_bytes(int32_t T);
NVFP4MOE_API nvfp4_status moe_permute(const int32_t* ids_dev, int32_t T, int32_t* counts_dev,
                                      int32_t* offsets_dev, int32_t* sorted_slot_dev,
                                      int32_t* slot_pos_dev, void* ws_dev, size_t ws_bytes,
                                      void* stream);

/* ---------------------------------------------------------------------------
 * moe_residual_rmsnorm: one link of a chained layer stack,
 *   res += y (if y_dev != NULL);  x_out = bf16(res / sqrt(mean(res^2) + eps))
 * (scale-free RMSNorm as in the router description).  Used to chain layers as
 * x_{l+1} = x_l + moe_l(rmsnorm(x_l)) with an fp32 residual.
 *   res_dev f32 [T, H] (in/out), y_dev bf16 [T, H] or NULL, x_out_dev bf16 [T, H]
 * Requires 1 <= T <= 65536, H % 8 == 0, H <= 16384.  No workspace.
 * ------------------------------------------------------------------------- */
NVFP4MOE_API nvfp4_status moe_residual_rmsnorm(float* res_dev, const void* y_dev, void* x_out_dev,
                                  int32_t T, int32_t H, float eps, void* stream);

/* ---------------------------------------------------------------------------
 * Device status: kernels record data errors (an expert id out of range) and
 * bounded waits that gave up in a per-device status word instead of faulting.
 * nvfp4_get_device_status synchronises `stream`, returns the first recorded
 * error (NVFP4_OK if none) and clears the word.
 * ------------------------------------------------------------------------- */
NVFP4MOE_API nvfp4_status nvfp4_get_device_status(void* stream);

/* nvfp4_selftest_wait_timeout: exercises the device-side failure path of the
 * bounded waits, so a deployment can check it on its driver without harming
 * the GPU.  It runs nvfp4_quantize's single-pass kernel on the given tensors
 * with a cross-CTA arrival count that can never be reached and every wait
 * limited to limit_us microseconds: each CTA gives up, records
 * NVFP4_ERR_TIMEOUT in the device status word, lets its own copies land and
 * exits, so the context stays usable (the next nvfp4_get_device_status
 * returns NVFP4_ERR_TIMEOUT).  The outputs are left unspecified.  Same
 * arguments and limits as nvfp4_quantize plus 1 <= limit_us <= 1000000;
 * NVFP4_ERR_UNSUPPORTED for a shape that does not take the single-pass
 * kernel.  The pages have no counterpart of this entry point. */
NVFP4MOE_API nvfp4_status nvfp4_selftest_wait_timeout(const void* w_dev, int64_t E, int64_t N, int64_t K,
                                                      uint8_t* q_dev, uint8_t* s_dev, float* g_dev,
                                                      void* ws_dev, size_t ws_bytes, uint32_t limit_us,
                                                      void* stream);

NVFP4MOE_API const char* nvfp4_status_string(nvfp4_status status);
NVFP4MOE_API int nvfp4_abi_version(void);

/* The CUDA runtime's text for the error behind the last NVFP4_ERR_CUDA that a
 * call of this library returned on the calling thread ("no error" if none).
 * A static string owned by the CUDA runtime; never NULL. */
NVFP4MOE_API const char* nvfp4_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4MOE_H */
