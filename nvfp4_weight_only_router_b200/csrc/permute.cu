// Token permutation by expert (the "sort-by-expert" step of the batched expert
// kernel described on the "Gemma 4 26B-A4B (MoE) - Core AI" card, "Decode
// only ...").  Slots s = t*8 + j are grouped by expert id with a stable
// counting sort, so each expert's slots stay in token order.
//
// Each CTA takes a chunk of 1024 slots (one per thread):
//   phase A: within-warp ranks by __match_any_sync, per-warp per-expert
//            counts in shared memory, a scan over the 32 warps -> each slot's
//            rank inside its chunk and the chunk's per-expert counts;
//   the last CTA to arrive (arrival counter) then runs
//   phase B: per-expert prefix over chunks, exclusive scan over experts
//            (offsets), the list of active experts;
//   phase C: scatter: pos = offsets[e] + chunk_base[chunk][e] + local rank.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kChunk = 1024;

// Exclusive scan of 128 values held 4 per lane (v[i] = value of index 4*lane+i)
// by one warp.  Returns the total.
__device__ __forceinline__ int warp_exclusive_scan128(int (&v)[4]) {
  const int lane = threadIdx.x & 31;
  int local = v[0] + v[1] + v[2] + v[3];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int run = incl - local;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = v[i];
    v[i] = run;
    run += c;
  }
  return total;
}

__global__ void __launch_bounds__(kChunk) permute_kernel(PermuteArgs a) {
  __shared__ int wcount[32][kE];
  __shared__ int s_last;
  __shared__ int s_off[kE + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;

  for (int i = tid; i < 32 * kE; i += kChunk) (&wcount[0][0])[i] = 0;
  __syncthreads();

  const int s = chunk * kChunk + tid;
  int e = -1;
  if (s < a.S) {
    e = a.ids[s];
    if (e < 0 || e >= kE) {
      record_status(a.status, kStatusDevice);
      e = -1;
    }
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) wcount[warp][e] = __popc(peers);
  __syncthreads();
  if (tid < kE) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcount[w][tid];
      wcount[w][tid] = run;
      run += c;
    }
    a.chunk_count[(size_t)chunk * kE + tid] = run;
  }
  __syncthreads();
  if (s < a.S) a.local_rank[s] = (e >= 0) ? wcount[warp][e] + rank : 0;

  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(a.meta + kMetaPermCounter, 1);
    s_last = (prev == (int)gridDim.x - 1);
    if (s_last) a.meta[kMetaPermCounter] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // phase B: per-expert prefix over chunks
  if (tid < kE) {
    int run = 0;
    for (int c = 0; c < a.nchunks; ++c) {
      const int v = __ldcg(a.chunk_count + (size_t)c * kE + tid);
      a.chunk_base[(size_t)c * kE + tid] = run;
      run += v;
    }
    s_off[tid] = run;  // count of expert tid (scanned below)
  }
  __syncthreads();
  if (warp == 0) {
    int cnt[4], flag[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      cnt[i] = s_off[4 * lane + i];
      flag[i] = cnt[i] > 0;
      a.meta[kMetaCounts + 4 * lane + i] = cnt[i];
    }
    int off[4] = {cnt[0], cnt[1], cnt[2], cnt[3]};
    const int total = warp_exclusive_scan128(off);
    const int nact = warp_exclusive_scan128(flag);  // flag[] now holds the act-list position
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ex = 4 * lane + i;
      s_off[ex] = off[i];
      a.meta[kMetaOffsets + ex] = off[i];
      if (cnt[i] > 0) a.meta[kMetaAct + flag[i]] = ex;
    }
    if (lane == 0) {
      s_off[kE] = total;
      a.meta[kMetaOffsets + kE] = total;
      a.meta[kMetaNAct] = nact;
    }
  }
  __syncthreads();

  // phase C: scatter
  for (int ss = tid; ss < a.S; ss += kChunk) {
    const int ee = a.ids[ss];
    if (ee < 0 || ee >= kE) {
      a.slot_pos[ss] = -1;
      continue;
    }
    const int pos = s_off[ee] + a.chunk_base[(size_t)(ss / kChunk) * kE + ee] + __ldcg(a.local_rank + ss);
    a.sorted_slot[pos] = ss;
    a.slot_pos[ss] = pos;
  }
}

}  // namespace

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
  permute_kernel<<<a.nchunks, kChunk, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
