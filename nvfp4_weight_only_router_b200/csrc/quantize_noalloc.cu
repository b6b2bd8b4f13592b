// nvfp4_quantize_noalloc: nvfp4_quantize without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the moment they quantise: a
// plugin whose host framework owns all device memory and forbids allocation
// inside its execute callback, or a latency-critical path that must never
// enter an allocator.  For them this entry point keeps the quantiser's only
// scratch -- one amax word per tensor -- in a fixed file-scope device array
// instead of a workspace.  It calls no cudaMalloc/cudaFree and no allocating
// library routine; the caller still passes the input and output buffers.
//
// The array is shared by every call on a device and keeps the last call's
// contents; each call clears the words it uses (one amax word per tensor,
// plus three arrival counters when the tensors take the single-pass kernel)
// before it reads them.  Calls
// that overlap on the GPU race on the array.  Every GPU that loads the
// library holds the array (16 KiB) until the process exits; with CUDA's lazy
// module loading the driver places it (with the module's code) at the first
// call on each device, so callers with a strict no-allocation window make one
// call before it opens.
#include <mutex>

#include "../../include/nvfp4moe.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int64_t kNoAllocMaxTensors = 4096;

// Per-tensor amax scratch of the no-allocation quantiser.  In host code this
// name is only a host-side stand-in for the symbol: kernels must be given the
// device address returned by cudaGetSymbolAddress below.
static __device__ __align__(256) uint32_t g_noalloc_amax[kNoAllocMaxTensors];

constexpr int kMaxDevices = 64;
uint32_t* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Set-up, once per device, with that device current: the device address of
// the scratch array, or the error of the runtime call that failed.
cudaError_t noalloc_scratch(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    uint32_t* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_noalloc_amax);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* w, int64_t E, int64_t N, int64_t K,
                                               uint8_t* q, uint8_t* s, float* g, void* stream) {
  if (E < 1 || N < 1 || K < 16) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || N * K >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (E > kNoAllocMaxTensors) return NVFP4_ERR_UNSUPPORTED;  // beyond the fixed scratch
  if (!w || !q || !s || !g) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || !aligned16(g)) return NVFP4_ERR_ALIGNMENT;
  uint32_t* scratch = nullptr;
  const cudaError_t se = noalloc_scratch(&scratch);
  if (se != cudaSuccess) return static_cast<nvfp4_status>(nvfp4moe::fail_cuda(se));
  // launch_quantize clears the scratch words it uses before the amax pass
  const cudaError_t e = nvfp4moe::launch_quantize(static_cast<const uint16_t*>(w), E, N, K, q, s, g,
                                                  scratch, kNoAllocMaxTensors, nvfp4moe::device_status_ptr(),
                                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : static_cast<nvfp4_status>(nvfp4moe::fail_cuda(e));
}
