// C ABI of the NVFP4 MoE library: argument validation, workspace layout and
// launch sequencing on the caller's stream.  See include/nvfp4moe.h.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "../../include/nvfp4moe.h"
#include "common.cuh"
#include "kernels.h"

using namespace nvfp4moe;

namespace {

// Per-device status word (see nvfp4_get_device_status).
__device__ int g_device_status;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

}  // namespace

int* nvfp4moe::device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A named range on the calling host thread for profilers (NVTX): kernels
// launched inside it carry its name in an nsys or ncu timeline.  Without a
// tool attached the calls do nothing.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// ------------------------------------------------------------------ layouts
struct Region {
  size_t off = 0, bytes = 0;
};

struct Alloc {
  size_t cur = 0;
  Region take(size_t bytes) {
    Region r;
    r.off = cur;
    r.bytes = bytes;
    cur = round_up(cur + bytes, 256);
    return r;
  }
};

constexpr int kFusedPermuteMaxSlots = 1024;  // the router's last CTA groups the slots

// Largest token count that takes the streaming GEMV path; above it the
// tensor-core grouped GEMMs run.
constexpr int kStreamMaxTokens = 256;
// Largest token count of the dense over-read variant (128 slots per token).
constexpr int kDenseMaxTokens = 256;

struct FwdLayout {
  Region meta;
  Region ids, wts, wdense, chunk_count, sorted, pos, xexp, xs, h, obuf;
  int S = 0, nchunks = 0, spt = kTopK;
  size_t total = 0;
};

// dense: the over-read variant (every token through all 128 experts)
FwdLayout fwd_layout(int T, bool dense = false) {
  FwdLayout L;
  Alloc al;
  L.spt = dense ? kE : kTopK;
  L.S = T * L.spt;
  L.nchunks = (L.S + 1023) / 1024;
  // zeroed on entry: meta (includes the router's arrival counter)
  L.meta = al.take(sizeof(int) * kMetaInts);
  L.ids = al.take(sizeof(int) * T * kTopK);
  L.wts = al.take(sizeof(float) * T * kTopK);
  if (dense) L.wdense = al.take(sizeof(float) * L.S);
  L.chunk_count = al.take(sizeof(int) * (size_t)L.nchunks * kE);
  L.sorted = al.take(sizeof(int) * L.S);
  L.pos = al.take(sizeof(int) * L.S);
  L.xexp = al.take(sizeof(int) * L.S);
  L.xs = al.take(sizeof(__half) * (size_t)L.S * kH);
  L.h = al.take(sizeof(__half) * (size_t)L.S * kI);
  // per-slot outputs, summed in slot order by the combine: deterministic
  L.obuf = al.take(sizeof(float) * (size_t)L.S * kH);
  L.total = al.cur;
  return L;
}

// Permutation workspace of moe_permute: the meta block and the per-chunk counts.
struct PermLayout {
  Region meta, chunk_count;
  int S = 0, nchunks = 0;
  size_t total = 0;
};

PermLayout perm_layout(int T) {
  PermLayout L;
  Alloc al;
  L.S = T * kTopK;
  L.nchunks = (L.S + 1023) / 1024;
  L.meta = al.take(sizeof(int) * kMetaInts);
  L.chunk_count = al.take(sizeof(int) * (size_t)L.nchunks * kE);
  L.total = al.cur;
  return L;
}

template <typename T>
T* at(void* ws, const Region& r) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + r.off);
}

// the last CUDA error behind an NVFP4_ERR_CUDA status, per calling thread
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

nvfp4_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = e != cudaSuccess ? e : cudaErrorUnknown;
  return NVFP4_ERR_CUDA;
}

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : cuda_fail(e); }

// hidden sizes the router kernels take: 8 to 16 slices of 256
bool router_hidden_ok(int H) { return H % 256 == 0 && H >= 2048 && H <= 4096; }

nvfp4_status check_router(const moe_router* r, bool forward) {
  if (!r || !r->proj || !r->scale || !r->per_expert_scale) return NVFP4_ERR_INVALID_ARG;
  if (r->E <= 0 || r->H <= 0 || r->top_k <= 0 || !(r->eps >= 0.f) || !std::isfinite(r->eps))
    return NVFP4_ERR_INVALID_ARG;
  if (r->E != kE || r->top_k != kTopK) return NVFP4_ERR_UNSUPPORTED;
  if (forward ? (r->H != kH) : !router_hidden_ok(r->H)) return NVFP4_ERR_UNSUPPORTED;
  if (!aligned(r->proj, 16) || !aligned(r->scale, 16) || !aligned(r->per_expert_scale, 16) ||
      (r->logit_bias && !aligned(r->logit_bias, 16)))
    return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

nvfp4_status check_experts(const moe_experts* x) {
  if (!x || !x->gate_up_q || !x->gate_up_s || !x->gate_up_g || !x->down_q || !x->down_s ||
      !x->down_g)
    return NVFP4_ERR_INVALID_ARG;
  if (x->E <= 0 || x->H <= 0 || x->I <= 0) return NVFP4_ERR_INVALID_ARG;
  if (x->E != kE || x->H != kH || x->I != kI) return NVFP4_ERR_UNSUPPORTED;
  const void* ps[] = {x->gate_up_q, x->gate_up_s, x->gate_up_g, x->down_q, x->down_s, x->down_g};
  for (const void* p : ps)
    if (!aligned(p, 16)) return NVFP4_ERR_ALIGNMENT;
  // the packed copies are optional, but both or neither
  if ((x->gate_up_pk == nullptr) != (x->down_pk == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(x->gate_up_pk, 16) || !aligned(x->down_pk, 16)) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

// The expert stacks of either codec, as the kernels take them.
struct ExpertPtrs {
  int codec = kCodecNvfp4;
  const uint8_t *gu_q = nullptr, *gu_s = nullptr, *dn_q = nullptr, *dn_s = nullptr;
  const uint8_t *gu_pk = nullptr, *dn_pk = nullptr;
  const float *gu_g = nullptr, *dn_g = nullptr;
  const uint16_t *gu_b = nullptr, *dn_b = nullptr;
};

ExpertPtrs nvfp4_ptrs(const moe_experts* x) {
  ExpertPtrs e;
  e.codec = kCodecNvfp4;
  e.gu_q = x->gate_up_q;
  e.gu_s = x->gate_up_s;
  e.gu_g = x->gate_up_g;
  e.dn_q = x->down_q;
  e.dn_s = x->down_s;
  e.dn_g = x->down_g;
  e.gu_pk = x->gate_up_pk;
  e.dn_pk = x->down_pk;
  return e;
}

nvfp4_status check_experts_aff4(const moe_experts_aff4* x) {
  if (!x || !x->gate_up_q || !x->gate_up_s || !x->gate_up_b || !x->down_q || !x->down_s || !x->down_b)
    return NVFP4_ERR_INVALID_ARG;
  if (x->E <= 0 || x->H <= 0 || x->I <= 0) return NVFP4_ERR_INVALID_ARG;
  if (x->E != kE || x->H != kH || x->I != kI) return NVFP4_ERR_UNSUPPORTED;
  const void* ps[] = {x->gate_up_q, x->gate_up_s, x->gate_up_b, x->down_q, x->down_s, x->down_b};
  for (const void* p : ps)
    if (!aligned(p, 16)) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

ExpertPtrs aff4_ptrs(const moe_experts_aff4* x) {
  ExpertPtrs e;
  e.codec = kCodecAff4;
  e.gu_q = x->gate_up_q;
  e.gu_s = static_cast<const uint8_t*>(x->gate_up_s);
  e.gu_b = static_cast<const uint16_t*>(x->gate_up_b);
  e.dn_q = x->down_q;
  e.dn_s = static_cast<const uint8_t*>(x->down_s);
  e.dn_b = static_cast<const uint16_t*>(x->down_b);
  return e;
}

RouteArgs make_route_args(const void* x, int T, const moe_router* r, int32_t* ids, float* wts, int* status) {
  RouteArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.proj = static_cast<const uint16_t*>(r->proj);
  a.scale = static_cast<const uint16_t*>(r->scale);
  a.pes = static_cast<const uint16_t*>(r->per_expert_scale);
  a.bias = r->logit_bias;
  a.T = T;
  a.H = r->H;
  a.few_tokens = T <= 256;
  a.eps = r->eps;
  a.inv_sqrt_h = (float)(1.0 / std::sqrt((double)r->H));
  a.ids = ids;
  a.wts = wts;
  a.meta = nullptr;
  a.sorted_slot = nullptr;
  a.slot_pos = nullptr;
  a.status = status;
  return a;
}

}  // namespace

int nvfp4moe::fail_cuda(cudaError_t e) { return cuda_fail(e); }

extern "C" {

int nvfp4_abi_version(void) { return NVFP4MOE_ABI_VERSION; }

const char* nvfp4_last_cuda_error(void) { return cudaGetErrorString(t_last_cuda_error); }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_ALIGNMENT: return "misaligned pointer";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported shape";
    case NVFP4_ERR_DEVICE: return "invalid data detected on the device";
    case NVFP4_ERR_RANGE: return "an activation left the range of the f16 tensor-core operands";
  }
  return "unknown status";
}

// ---------------------------------------------------------------- quantize
static nvfp4_status check_quant_dims(int64_t E, int64_t N, int64_t K) {
  if (E < 1 || N < 1 || K < 16) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (N * K >= (int64_t(1) << 31) || E > (int64_t(1) << 20)) return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

size_t nvfp4_quantize_workspace_bytes(int64_t E, int64_t N, int64_t K) {
  if (check_quant_dims(E, N, K) != NVFP4_OK) return 0;
  // E amax words + 3 arrival counters of the single-pass kernel
  return round_up(sizeof(uint32_t) * (size_t)(E + 3), 256);
}

nvfp4_status nvfp4_quantize(const void* w, int64_t E, int64_t N, int64_t K, uint8_t* q, uint8_t* s,
                            float* g, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nv("nvfp4_quantize");
  nvfp4_status st = check_quant_dims(E, N, K);
  if (st != NVFP4_OK) return st;
  if (!w || !q || !s || !g) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(s, 16) || !aligned(g, 16))
    return NVFP4_ERR_ALIGNMENT;
  if (!ws || ws_bytes < nvfp4_quantize_workspace_bytes(E, N, K)) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  return cuda_status(launch_quantize(static_cast<const uint16_t*>(w), E, N, K, q, s, g,
                                     static_cast<uint32_t*>(ws), (int64_t)(ws_bytes / sizeof(uint32_t)),
                                     device_status_ptr(), as_stream(stream)));
}

nvfp4_status nvfp4_dequantize(const uint8_t* q, const uint8_t* s, const float* g, int64_t E,
                              int64_t N, int64_t K, float* out, void* stream) {
  nvfp4_status st = check_quant_dims(E, N, K);
  if (st != NVFP4_OK) return st;
  if (!q || !s || !g || !out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(s, 16) || !aligned(g, 16) || !aligned(out, 16))
    return NVFP4_ERR_ALIGNMENT;
  return cuda_status(launch_dequantize(q, s, g, E, N, K, out, as_stream(stream)));
}

// ------------------------------------------------------------------- route
size_t moe_route_workspace_bytes(int32_t T, const moe_router* r) {
  if (T < 1 || T > 65536 || check_router(r, false) != NVFP4_OK) return 0;
  return 256;  // the router kernels keep their scratch on chip
}

nvfp4_status moe_route(const void* x, int32_t T, const moe_router* r, int32_t* ids, float* w,
                       void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nv("moe_route");
  if (T < 1 || T > 65536 || !x || !ids || !w) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_router(r, false);
  if (st != NVFP4_OK) return st;
  if (!aligned(x, 16) || !aligned(ids, 16) || !aligned(w, 16)) return NVFP4_ERR_ALIGNMENT;
  if (!ws || ws_bytes < moe_route_workspace_bytes(T, r)) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  RouteArgs a = make_route_args(x, T, r, ids, w, device_status_ptr());
  return cuda_status(launch_route(a, as_stream(stream)));
}

// ---------------------------------------------------------------- permute
size_t moe_permute_workspace_bytes(int32_t T) {
  if (T < 1 || T > 65536) return 0;
  return perm_layout(T).total;
}

nvfp4_status moe_permute(const int32_t* ids, int32_t T, int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                         int32_t* slot_pos, void* ws, size_t ws_bytes, void* stream) {
  if (T < 1 || T > 65536 || !ids || !counts || !offsets || !sorted_slot || !slot_pos) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ids, 16) || !aligned(counts, 16) || !aligned(offsets, 16) || !aligned(sorted_slot, 16) ||
      !aligned(slot_pos, 16))
    return NVFP4_ERR_ALIGNMENT;
  const PermLayout L = perm_layout(T);
  if (!ws || ws_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  PermuteArgs pa;
  pa.ids = ids;
  pa.S = L.S;
  pa.nchunks = L.nchunks;
  pa.meta = at<int>(ws, L.meta);
  pa.chunk_count = at<int>(ws, L.chunk_count);
  pa.sorted_slot = sorted_slot;
  pa.slot_pos = slot_pos;
  pa.status = device_status_ptr();
  cudaError_t e = launch_permute(pa, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(counts, pa.meta + kMetaCounts, sizeof(int) * kE, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(offsets, pa.meta + kMetaOffsets, sizeof(int) * (kE + 1), cudaMemcpyDeviceToDevice, s);
  return cuda_status(e);
}

// ----------------------------------------------------------------- forward
size_t moe_forward_workspace_bytes(int32_t T, const moe_experts* ex, const moe_router* r) {
  if (T < 1 || T > 65536 || check_experts(ex) != NVFP4_OK || check_router(r, true) != NVFP4_OK)
    return 0;
  return fwd_layout(T).total;
}

nvfp4_status moe_forward_workspace_views(int32_t T, const moe_experts* ex, const moe_router* r,
                                         moe_forward_views* out) {
  if (!out || T < 1 || T > 65536) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_experts(ex);
  if (st == NVFP4_OK) st = check_router(r, true);
  if (st != NVFP4_OK) return st;
  FwdLayout L = fwd_layout(T);
  out->ids = L.ids.off;
  out->weights = L.wts.off;
  out->counts = L.meta.off + sizeof(int) * kMetaCounts;
  out->offsets = L.meta.off + sizeof(int) * kMetaOffsets;
  out->sorted_slot = L.sorted.off;
  out->slot_pos = L.pos.off;
  out->xexp = L.xexp.off;
  out->h = L.h.off;
  return NVFP4_OK;
}

// The routed forward.  x_route (null: x) is the router's input, x the
// experts'; with finalize false the per-slot rows are left in the workspace
// (for the full block's final kernel) and y is not written.
static nvfp4_status forward_impl(const void* x, int32_t T, const ExpertPtrs& ex,
                                 const moe_router* r, void* y, void* ws, size_t ws_bytes,
                                 void* stream, void* const* ev, bool dense = false,
                                 const void* x_route = nullptr, bool finalize = true) {
  if (T < 1 || T > (dense ? kDenseMaxTokens : 65536) || !x || (finalize && !y)) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_router(r, true);
  if (st != NVFP4_OK) return st;
  if (!aligned(x, 16) || (y && !aligned(y, 16)) || (x_route && !aligned(x_route, 16))) return NVFP4_ERR_ALIGNMENT;
  const FwdLayout L = fwd_layout(T, dense);
  if (!ws || ws_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  int* status = device_status_ptr();
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (ev && cudaStreamIsCapturing(s, &cap) != cudaSuccess) return cuda_fail(cudaGetLastError());
  auto mark = [&](int i) -> bool {
    if (!ev || !ev[i]) return true;
    cudaEvent_t e = static_cast<cudaEvent_t>(ev[i]);
    // inside a stream capture, an external record becomes an event-record node
    // of the graph (a plain record would only order the capture)
    if (cap == cudaStreamCaptureStatusActive)
      return cudaEventRecordWithFlags(e, s, cudaEventRecordExternal) == cudaSuccess;
    return cudaEventRecord(e, s) == cudaSuccess;
  };
  if (!mark(0)) return cuda_fail(cudaGetLastError());
  NvtxRange nv(dense ? "moe_forward_dense" : "moe_forward");

  cudaError_t e = cudaMemsetAsync(at<int>(ws, L.meta), 0, L.meta.bytes, s);
  if (e != cudaSuccess) return cuda_fail(e);

  int32_t* ids = at<int32_t>(ws, L.ids);
  float* wts = at<float>(ws, L.wts);
  RouteArgs ra = make_route_args(x_route ? x_route : x, T, r, ids, wts, status);
  const bool fused_permute = !dense && ra.few_tokens && L.S <= kFusedPermuteMaxSlots;
  if (fused_permute) {
    ra.meta = at<int>(ws, L.meta);
    ra.sorted_slot = at<int>(ws, L.sorted);
    ra.slot_pos = at<int>(ws, L.pos);
  }
  {
    NvtxRange r("route");
    if ((e = launch_route(ra, s)) != cudaSuccess || !mark(1)) return cuda_fail(e);
  }

  PermuteArgs pa;
  pa.ids = ids;
  pa.S = L.S;
  pa.nchunks = L.nchunks;
  pa.meta = at<int>(ws, L.meta);
  pa.chunk_count = at<int>(ws, L.chunk_count);
  pa.sorted_slot = at<int>(ws, L.sorted);
  pa.slot_pos = at<int>(ws, L.pos);
  pa.status = status;
  if (dense) {
    e = launch_dense_permute(ids, wts, T, pa.meta, pa.sorted_slot, pa.slot_pos, at<float>(ws, L.wdense), status, s);
    if (e != cudaSuccess) return cuda_fail(e);
  } else if (!fused_permute && (e = launch_permute(pa, s)) != cudaSuccess) {
    return cuda_fail(e);
  }

  ExpertArgs xa;
  xa.codec = ex.codec;
  xa.gu_q = ex.gu_q;
  xa.gu_s = ex.gu_s;
  xa.gu_g = ex.gu_g;
  xa.gu_b = ex.gu_b;
  xa.dn_q = ex.dn_q;
  xa.dn_s = ex.dn_s;
  xa.dn_g = ex.dn_g;
  xa.dn_b = ex.dn_b;
  xa.gu_pk = ex.gu_pk;
  xa.dn_pk = ex.dn_pk;
  xa.x = static_cast<const uint16_t*>(x);
  xa.meta = pa.meta;
  xa.sorted_slot = pa.sorted_slot;
  xa.slot_pos = pa.slot_pos;
  xa.wts = dense ? at<float>(ws, L.wdense) : wts;
  xa.spt = L.spt;
  xa.xexp = at<int>(ws, L.xexp);
  xa.h = at<__half>(ws, L.h);
  xa.obuf = at<float>(ws, L.obuf);
  xa.y = y;
  xa.T = T;
  xa.max_active = L.S < kE ? L.S : kE;  // (the kernels read the active count from meta)
  xa.status = status;
  xa.xs = at<__half>(ws, L.xs);
  // the activations follow their slots into expert order (f16 for the MMAs)
  {
    NvtxRange r("gather");
    if ((e = launch_gather_sorted(xa, s)) != cudaSuccess) return cuda_fail(e);
    if (!mark(2)) return cuda_fail(cudaGetLastError());
  }
  if (T <= kStreamMaxTokens) {
    // few tokens per expert: the weight stream bounds the step (streaming
    // GEMV with register dequantisation)
    NvtxRange r("experts (streaming GEMV)");
    e = launch_gate_up_stream(xa, s);
    if (e != cudaSuccess || !mark(3)) return cuda_fail(e);
    e = launch_down_stream(xa, s);
    if (e != cudaSuccess || !mark(4)) return cuda_fail(e);
  } else {
    // many tokens per expert: tensor-core grouped GEMMs on expert-sorted rows
    NvtxRange r("experts (tensor-core GEMMs)");
    const int nt = T <= 512 ? 64 : 192;  // about the tokens an expert gets
    e = launch_moe_gate_up(xa, nt, s);
    if (e != cudaSuccess || !mark(3)) return cuda_fail(e);
    e = launch_moe_down(xa, nt, s);
    if (e != cudaSuccess || !mark(4)) return cuda_fail(e);
  }
  if (finalize) {
    NvtxRange r("combine");
    if ((e = launch_finalize(xa, s)) != cudaSuccess || !mark(5)) return cuda_fail(e);
  }
  return NVFP4_OK;
}

// ------------------------------------------------------------- full block
namespace {

constexpr int kBlockMaxTokens = 8192;
constexpr int kMaxSms = 148;  // the workspace holds the dense K splits for up to this many SMs

struct BlockLayout {
  FwdLayout moe;
  Region x1, x2, gu_part, hd_hi, hd_lo, dn_part;
  int sp_gu = 1, sp_dn = 1;
  size_t total = 0;
};

BlockLayout block_layout(int T) {
  BlockLayout L;
  L.moe = fwd_layout(T);
  Alloc al;
  al.cur = L.moe.total;
  L.sp_gu = dense_splits(0, T, kMaxSms);
  L.sp_dn = dense_splits(1, T, kMaxSms);
  L.x1 = al.take(sizeof(uint16_t) * (size_t)T * kH);
  L.x2 = al.take(sizeof(uint16_t) * (size_t)T * kH);
  L.gu_part = al.take(sizeof(float) * (size_t)L.sp_gu * T * 2 * kDenseI);
  L.hd_hi = al.take(sizeof(uint16_t) * (size_t)T * kDenseI);
  L.hd_lo = al.take(sizeof(uint16_t) * (size_t)T * kDenseI);
  L.dn_part = al.take(sizeof(float) * (size_t)L.sp_dn * T * kH);
  L.total = al.cur;
  return L;
}

nvfp4_status check_block(const moe_block* b) {
  if (!b) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_experts(&b->experts);
  if (st == NVFP4_OK) st = check_router(&b->router, true);
  if (st != NVFP4_OK) return st;
  const void* ps[] = {b->dense_gate, b->dense_up, b->dense_down, b->pre_ff_norm, b->post_ff_norm_1,
                      b->pre_ff_norm_2, b->post_ff_norm_2, b->post_ff_norm, b->layer_scalar};
  for (const void* q : ps)
    if (!q) return NVFP4_ERR_INVALID_ARG;
  if (b->dense_I <= 0 || !(b->eps >= 0.f) || !std::isfinite(b->eps)) return NVFP4_ERR_INVALID_ARG;
  if (b->dense_I != kDenseI) return NVFP4_ERR_UNSUPPORTED;
  for (const void* q : ps)
    if (!aligned(q, 16)) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

}  // namespace

size_t moe_block_workspace_bytes(int32_t T, const moe_block* b) {
  if (T < 1 || T > kBlockMaxTokens || check_block(b) != NVFP4_OK) return 0;
  return block_layout(T).total;
}

nvfp4_status moe_block_forward(const void* x, int32_t T, const moe_block* b, void* y, void* ws, size_t ws_bytes,
                               void* stream) {
  NvtxRange nv("moe_block_forward");
  if (T < 1 || T > kBlockMaxTokens || !x || !y) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_block(b);
  if (st != NVFP4_OK) return st;
  if (!aligned(x, 16) || !aligned(y, 16)) return NVFP4_ERR_ALIGNMENT;
  const BlockLayout L = block_layout(T);
  if (!ws || ws_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return cuda_fail(e);
  const int sp_gu = std::min(L.sp_gu, dense_splits(0, T, sms));
  const int sp_dn = std::min(L.sp_dn, dense_splits(1, T, sms));
  uint16_t* x1 = at<uint16_t>(ws, L.x1);
  uint16_t* x2 = at<uint16_t>(ws, L.x2);
  // the two pre-feedforward norms (the MLPs' bf16 inputs)
  e = launch_block_prenorm(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(b->pre_ff_norm),
                           static_cast<const uint16_t*>(b->pre_ff_norm_2), b->eps, T, x1, x2, s);
  if (e != cudaSuccess) return cuda_fail(e);
  // the sparse branch: router on the raw residual, experts on x2; per-slot rows stay in ws
  st = forward_impl(x2, T, nvfp4_ptrs(&b->experts), &b->router, nullptr, ws, ws_bytes, stream, nullptr, false, x,
                    false);
  if (st != NVFP4_OK) return st;
  // the dense branch
  DenseArgs da;
  da.w0 = b->dense_gate;
  da.w1 = b->dense_up;
  da.b0 = x1;
  da.b1 = nullptr;
  da.out = at<float>(ws, L.gu_part);
  da.T = T;
  da.splits = sp_gu;
  da.status = device_status_ptr();
  if ((e = launch_dense_gate_up(da, s)) != cudaSuccess) return cuda_fail(e);
  uint16_t* hi = at<uint16_t>(ws, L.hd_hi);
  uint16_t* lo = at<uint16_t>(ws, L.hd_lo);
  if ((e = launch_dense_act(da.out, sp_gu, T, hi, lo, s)) != cudaSuccess) return cuda_fail(e);
  da.w0 = b->dense_down;
  da.w1 = nullptr;
  da.b0 = hi;
  da.b1 = lo;
  da.out = at<float>(ws, L.dn_part);
  da.splits = sp_dn;
  if ((e = launch_dense_down(da, s)) != cudaSuccess) return cuda_fail(e);
  // the post norms, the residual and the layer scalar
  BlockFinalArgs fa;
  fa.x = static_cast<const uint16_t*>(x);
  fa.obuf = at<float>(ws, L.moe.obuf);
  fa.slot_pos = at<int>(ws, L.moe.pos);
  fa.dense = da.out;
  fa.splits = sp_dn;
  fa.T = T;
  fa.post1 = static_cast<const uint16_t*>(b->post_ff_norm_1);
  fa.post2 = static_cast<const uint16_t*>(b->post_ff_norm_2);
  fa.post = static_cast<const uint16_t*>(b->post_ff_norm);
  fa.layer_scalar = static_cast<const uint16_t*>(b->layer_scalar);
  fa.eps = b->eps;
  fa.y = y;
  return cuda_status(launch_block_final(fa, s));
}

// ------------------------------------------------------------------- W4A4
namespace {

struct W4A4Layout {
  Region meta, ids, wts, chunk_count, sorted, pos, aq, asf, roww, hq, hsf, obuf;
  int S = 0, nchunks = 0, nt = 16, max_tiles = 0;
  size_t total = 0;
};

W4A4Layout w4a4_layout(int T) {
  W4A4Layout L;
  Alloc al;
  L.S = T * kTopK;
  L.nchunks = (L.S + 1023) / 1024;
  L.nt = w4a4_tile_tokens(T);
  // every expert's slots padded to whole tiles: at most one partial tile each
  L.max_tiles = (L.S + L.nt - 1) / L.nt + kE;
  const size_t rows = (size_t)L.max_tiles * L.nt;
  L.meta = al.take(sizeof(int) * kMetaInts);
  L.ids = al.take(sizeof(int) * T * kTopK);
  L.wts = al.take(sizeof(float) * T * kTopK);
  L.chunk_count = al.take(sizeof(int) * (size_t)L.nchunks * kE);
  L.sorted = al.take(sizeof(int) * L.S);
  L.pos = al.take(sizeof(int) * L.S);
  L.aq = al.take(rows * (kH / 2));
  L.asf = al.take((size_t)L.max_tiles * (kH / 64) * 512);
  L.roww = al.take(sizeof(float) * rows);
  L.hq = al.take(rows * 384);  // 3 chunks of 128 bytes per row
  L.hsf = al.take((size_t)L.max_tiles * (kI / 64) * 512);
  L.obuf = al.take(sizeof(float) * (size_t)L.S * kH);
  L.total = al.cur;
  return L;
}

nvfp4_status check_experts_w4a4(const moe_experts_w4a4* x) {
  if (!x) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_experts(&x->experts);
  if (st != NVFP4_OK) return st;
  if (!x->experts.gate_up_pk || !x->gate_up_sf || !x->down_sf) return NVFP4_ERR_INVALID_ARG;
  const float gs[2] = {x->input_scale_gate_up, x->input_scale_down};
  for (float g : gs)
    if (!(g > 0.f) || !std::isfinite(g)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(x->gate_up_sf, 16) || !aligned(x->down_sf, 16)) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

}  // namespace

size_t moe_pack_bytes(int32_t E, int32_t which) {
  if (E < 1 || E > (1 << 20)) return 0;
  switch (which) {
    case 0: return packed_code_bytes(E, 0);
    case 1: return packed_code_bytes(E, 1);
    case 2: return (size_t)E * (2 * kI) * (kH / kBlock);
    case 3: return (size_t)E * kH * (kI / kBlock);
  }
  return 0;
}

nvfp4_status moe_nvfp4_pack_codes(const moe_experts* ex, uint8_t* gu_pk, uint8_t* dn_pk, void* stream) {
  nvfp4_status st = check_experts(ex);
  if (st != NVFP4_OK) return st;
  if (!gu_pk || !dn_pk) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(gu_pk, 16) || !aligned(dn_pk, 16)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_pack_codes(ex->gate_up_q, ex->E, 0, gu_pk, s);
  if (e == cudaSuccess) e = launch_pack_codes(ex->down_q, ex->E, 1, dn_pk, s);
  return cuda_status(e);
}

nvfp4_status moe_w4a4_pack_scales(const moe_experts* ex, uint8_t* gu_sf, uint8_t* dn_sf, void* stream) {
  nvfp4_status st = check_experts(ex);
  if (st != NVFP4_OK) return st;
  if (!gu_sf || !dn_sf) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(gu_sf, 16) || !aligned(dn_sf, 16)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_w4a4_pack_scales(ex->gate_up_s, ex->E, 0, gu_sf, s);
  if (e == cudaSuccess) e = launch_w4a4_pack_scales(ex->down_s, ex->E, 1, dn_sf, s);
  return cuda_status(e);
}

size_t moe_w4a4_workspace_bytes(int32_t T, const moe_experts_w4a4* ex, const moe_router* r) {
  if (T < 1 || T > 65536 || check_experts_w4a4(ex) != NVFP4_OK || check_router(r, true) != NVFP4_OK) return 0;
  return w4a4_layout(T).total;
}

nvfp4_status moe_w4a4_workspace_views(int32_t T, const moe_experts_w4a4* ex, const moe_router* r,
                                      moe_w4a4_views* out) {
  if (!out || T < 1 || T > 65536) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_experts_w4a4(ex);
  if (st == NVFP4_OK) st = check_router(r, true);
  if (st != NVFP4_OK) return st;
  const W4A4Layout L = w4a4_layout(T);
  out->ids = L.ids.off;
  out->weights = L.wts.off;
  out->counts = L.meta.off + sizeof(int) * kMetaCounts;
  out->offsets = L.meta.off + sizeof(int) * kMetaOffsets;
  out->sorted_slot = L.sorted.off;
  out->slot_pos = L.pos.off;
  out->x_codes = L.aq.off;
  out->x_scales = L.asf.off;
  out->h_codes = L.hq.off;
  out->h_scales = L.hsf.off;
  out->tile_tokens = L.nt;
  out->max_tiles = L.max_tiles;
  return NVFP4_OK;
}

static nvfp4_status w4a4_forward_impl(const void* x, int32_t T, const moe_experts_w4a4* ex, const moe_router* r,
                                      void* y, void* ws, size_t ws_bytes, void* stream, void* const* ev) {
  if (T < 1 || T > 65536 || !x || !y) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_experts_w4a4(ex);
  if (st == NVFP4_OK) st = check_router(r, true);
  if (st != NVFP4_OK) return st;
  if (!aligned(x, 16) || !aligned(y, 16)) return NVFP4_ERR_ALIGNMENT;
  const W4A4Layout L = w4a4_layout(T);
  if (!ws || ws_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  int* status = device_status_ptr();
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (ev && cudaStreamIsCapturing(s, &cap) != cudaSuccess) return cuda_fail(cudaGetLastError());
  auto mark = [&](int i) -> bool {
    if (!ev || !ev[i]) return true;
    cudaEvent_t evt = static_cast<cudaEvent_t>(ev[i]);
    if (cap == cudaStreamCaptureStatusActive)
      return cudaEventRecordWithFlags(evt, s, cudaEventRecordExternal) == cudaSuccess;
    return cudaEventRecord(evt, s) == cudaSuccess;
  };
  if (!mark(0)) return cuda_fail(cudaGetLastError());
  NvtxRange nv("moe_w4a4_forward");
  cudaError_t e = cudaMemsetAsync(at<int>(ws, L.meta), 0, L.meta.bytes, s);
  if (e != cudaSuccess) return cuda_fail(e);
  int32_t* ids = at<int32_t>(ws, L.ids);
  float* wts = at<float>(ws, L.wts);
  RouteArgs ra = make_route_args(x, T, r, ids, wts, status);
  const bool fused_permute = ra.few_tokens && L.S <= kFusedPermuteMaxSlots;
  PermuteArgs pa;
  pa.ids = ids;
  pa.S = L.S;
  pa.nchunks = L.nchunks;
  pa.meta = at<int>(ws, L.meta);
  pa.chunk_count = at<int>(ws, L.chunk_count);
  pa.sorted_slot = at<int>(ws, L.sorted);
  pa.slot_pos = at<int>(ws, L.pos);
  pa.status = status;
  if (fused_permute) {
    ra.meta = pa.meta;
    ra.sorted_slot = pa.sorted_slot;
    ra.slot_pos = pa.slot_pos;
  }
  if ((e = launch_route(ra, s)) != cudaSuccess || !mark(1)) return cuda_fail(e);
  if (!fused_permute && (e = launch_permute(pa, s)) != cudaSuccess) return cuda_fail(e);

  const moe_experts& w = ex->experts;
  uint8_t* aq = at<uint8_t>(ws, L.aq);
  uint8_t* asf = at<uint8_t>(ws, L.asf);
  uint8_t* hq = at<uint8_t>(ws, L.hq);
  uint8_t* hsf = at<uint8_t>(ws, L.hsf);
  float* roww = at<float>(ws, L.roww);
  e = launch_w4a4_act_quant(static_cast<const uint16_t*>(x), pa.meta, pa.slot_pos, wts, T, ex->input_scale_gate_up,
                            L.nt, aq, asf, roww, status, s);
  if (e != cudaSuccess || !mark(2)) return cuda_fail(e);
  W4A4Args ga;
  ga.wq = w.gate_up_pk;
  ga.wsf = ex->gate_up_sf;
  ga.wg = w.gate_up_g;
  ga.gin = ex->input_scale_gate_up;
  ga.gh = ex->input_scale_down;
  ga.aq = aq;
  ga.asf = asf;
  ga.hq = hq;
  ga.hsf = hsf;
  ga.meta = pa.meta;
  ga.roww = roww;
  ga.obuf = at<float>(ws, L.obuf);
  ga.max_tiles = L.max_tiles;
  ga.status = status;
  if ((e = launch_w4a4_gemm(ga, 0, L.nt, s)) != cudaSuccess || !mark(3)) return cuda_fail(e);
  W4A4Args da = ga;
  da.wq = w.down_pk;
  da.wsf = ex->down_sf;
  da.wg = w.down_g;
  da.gin = ex->input_scale_down;
  da.aq = hq;
  da.asf = hsf;
  if ((e = launch_w4a4_gemm(da, 1, L.nt, s)) != cudaSuccess || !mark(4)) return cuda_fail(e);
  ExpertArgs xa{};
  xa.T = T;
  xa.spt = kTopK;
  xa.slot_pos = pa.slot_pos;
  xa.obuf = ga.obuf;
  xa.y = y;
  if ((e = launch_finalize(xa, s)) != cudaSuccess || !mark(5)) return cuda_fail(e);
  return NVFP4_OK;
}

nvfp4_status moe_w4a4_forward(const void* x, int32_t T, const moe_experts_w4a4* ex, const moe_router* r, void* y,
                              void* ws, size_t ws_bytes, void* stream) {
  return w4a4_forward_impl(x, T, ex, r, y, ws, ws_bytes, stream, nullptr);
}

nvfp4_status moe_w4a4_forward_profiled(const void* x, int32_t T, const moe_experts_w4a4* ex, const moe_router* r,
                                       void* y, void* ws, size_t ws_bytes, void* stream, void* const* phase_events) {
  return w4a4_forward_impl(x, T, ex, r, y, ws, ws_bytes, stream, phase_events);
}

nvfp4_status moe_nvfp4_forward(const void* x, int32_t T, const moe_experts* ex, const moe_router* r,
                               void* y, void* ws, size_t ws_bytes, void* stream) {
  const nvfp4_status st = check_experts(ex);
  if (st != NVFP4_OK) return st;
  return forward_impl(x, T, nvfp4_ptrs(ex), r, y, ws, ws_bytes, stream, nullptr);
}

size_t moe_aff4_forward_workspace_bytes(int32_t T, const moe_experts_aff4* ex, const moe_router* r) {
  if (T < 1 || T > 65536 || check_experts_aff4(ex) != NVFP4_OK || check_router(r, true) != NVFP4_OK) return 0;
  return fwd_layout(T).total;
}

nvfp4_status moe_aff4_forward(const void* x, int32_t T, const moe_experts_aff4* ex, const moe_router* r, void* y,
                              void* ws, size_t ws_bytes, void* stream) {
  const nvfp4_status st = check_experts_aff4(ex);
  if (st != NVFP4_OK) return st;
  return forward_impl(x, T, aff4_ptrs(ex), r, y, ws, ws_bytes, stream, nullptr);
}

size_t moe_forward_dense_workspace_bytes(int32_t T, const moe_experts* ex, const moe_router* r) {
  if (T < 1 || T > kDenseMaxTokens || check_experts(ex) != NVFP4_OK || check_router(r, true) != NVFP4_OK)
    return 0;
  return fwd_layout(T, true).total;
}

nvfp4_status moe_nvfp4_forward_dense(const void* x, int32_t T, const moe_experts* ex, const moe_router* r,
                                     void* y, void* ws, size_t ws_bytes, void* stream) {
  const nvfp4_status st = check_experts(ex);
  if (st != NVFP4_OK) return st;
  return forward_impl(x, T, nvfp4_ptrs(ex), r, y, ws, ws_bytes, stream, nullptr, true);
}

nvfp4_status moe_nvfp4_forward_profiled(const void* x, int32_t T, const moe_experts* ex,
                                        const moe_router* r, void* y, void* ws, size_t ws_bytes,
                                        void* stream, void* const* phase_events) {
  const nvfp4_status st = check_experts(ex);
  if (st != NVFP4_OK) return st;
  return forward_impl(x, T, nvfp4_ptrs(ex), r, y, ws, ws_bytes, stream, phase_events);
}

nvfp4_status nvfp4_selftest_wait_timeout(const void* w, int64_t E, int64_t N, int64_t K, uint8_t* q, uint8_t* s,
                                         float* g, void* ws, size_t ws_bytes, uint32_t limit_us, void* stream) {
  nvfp4_status st = check_quant_dims(E, N, K);
  if (st != NVFP4_OK) return st;
  if (!w || !q || !s || !g || limit_us < 1 || limit_us > 1000000) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(s, 16) || !aligned(g, 16)) return NVFP4_ERR_ALIGNMENT;
  if (!ws || ws_bytes < nvfp4_quantize_workspace_bytes(E, N, K)) return NVFP4_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return NVFP4_ERR_ALIGNMENT;
  const cudaError_t e = launch_quantize_timeout_selftest(
      static_cast<const uint16_t*>(w), E, N, K, q, s, g, static_cast<uint32_t*>(ws),
      (int64_t)(ws_bytes / sizeof(uint32_t)), device_status_ptr(), (uint64_t)limit_us * 1000ull, as_stream(stream));
  if (e == cudaErrorNotSupported) return NVFP4_ERR_UNSUPPORTED;
  return cuda_status(e);
}

// ------------------------------------------------------------ chain helper
nvfp4_status moe_residual_rmsnorm(float* res, const void* y, void* x_out, int32_t T, int32_t H,
                                  float eps, void* stream) {
  if (!res || !x_out || T < 1 || T > 65536 || H < 8 || H % 8 != 0 || H > 16384 ||
      !(eps >= 0.f) || !std::isfinite(eps))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(res, 16) || !aligned(x_out, 16) || (y && !aligned(y, 16))) return NVFP4_ERR_ALIGNMENT;
  return cuda_status(launch_residual_rmsnorm(res, static_cast<const uint16_t*>(y),
                                             static_cast<uint16_t*>(x_out), T, H, eps,
                                             as_stream(stream)));
}

// ----------------------------------------------------------- device status
nvfp4_status nvfp4_get_device_status(void* stream) {
  int* p = device_status_ptr();
  if (!p) return cuda_fail(cudaGetLastError());
  cudaStream_t s = as_stream(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_fail(cudaGetLastError());
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_fail(cudaGetLastError());
  if (v != 0 && cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return cuda_fail(cudaGetLastError());
  return static_cast<nvfp4_status>(v);
}

}  // extern "C"
