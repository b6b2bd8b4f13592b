// Token permutation by expert (the "sort-by-expert" step of the batched expert
// kernel described on the "Gemma 4 26B-A4B (MoE) - Core AI" card, "Decode
// only ...").  Slots s = t*8 + j are grouped by expert id with a stable
// counting sort, so each expert's slots stay in token order.
//
// Two launches over chunks of 1024 slots (one per thread):
//   count:   each CTA writes its chunk's per-expert counts;
//   scatter: each CTA recomputes its slots' ranks inside the chunk (within-
//            warp ranks by __match_any_sync, a scan over the 32 warps), reads
//            the count table to get its chunk's base per expert and every
//            expert's offset, and places its slots: pos = offset[e] +
//            base[chunk][e] + rank.  CTA 0 also writes the counts, offsets
//            and the active-expert list.
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

// ranks of the chunk's slots inside the chunk: per-warp per-expert counts in
// wcount (then their exclusive scan over warps); returns the slot's expert
// (-1 if none or invalid) and its rank
__device__ __forceinline__ int chunk_rank(const PermuteArgs& a, int (*wcount)[kE], int& e_out, bool write_counts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 32 * kE; i += kChunk) (&wcount[0][0])[i] = 0;
  __syncthreads();
  const int s = blockIdx.x * kChunk + tid;
  int e = -1;
  if (s < a.S) {
    e = a.ids[s];
    if (e < 0 || e >= kE) {
      if (write_counts) record_status(a.status, kStatusDevice);
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
    if (write_counts) a.chunk_count[(size_t)blockIdx.x * kE + tid] = run;
  }
  __syncthreads();
  e_out = e;
  return e >= 0 ? wcount[warp][e] + rank : 0;
}

__global__ void __launch_bounds__(kChunk) permute_count_kernel(PermuteArgs a) {
  __shared__ int wcount[32][kE];
  int e;
  chunk_rank(a, wcount, e, true);
}

__global__ void __launch_bounds__(kChunk) permute_scatter_kernel(PermuteArgs a) {
  __shared__ int wcount[32][kE];
  __shared__ int part_tot[8][kE], part_base[8][kE];
  __shared__ int s_off[kE + 1], s_base[kE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;
  int e;
  const int rank = chunk_rank(a, wcount, e, false);

  // per expert: its total over all chunks and its base in this chunk (the
  // counts of the chunks before it); thread (expert ex, part p) takes chunks
  // c = p, p + 8, ...
  {
    const int ex = tid & (kE - 1), part = tid >> 7;
    int tot = 0, base = 0;
    for (int c = part; c < a.nchunks; c += 8) {
      const int v = a.chunk_count[(size_t)c * kE + ex];
      tot += v;
      if (c < chunk) base += v;
    }
    part_tot[part][ex] = tot;
    part_base[part][ex] = base;
  }
  __syncthreads();
  if (tid < kE) {
    int tot = 0, base = 0;
#pragma unroll
    for (int pt = 0; pt < 8; ++pt) {
      tot += part_tot[pt][tid];
      base += part_base[pt][tid];
    }
    s_off[tid] = tot;
    s_base[tid] = base;
  }
  __syncthreads();
  if (warp == 0) {
    int cnt[4], flag[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      cnt[i] = s_off[4 * lane + i];
      flag[i] = cnt[i] > 0;
    }
    int off[4] = {cnt[0], cnt[1], cnt[2], cnt[3]};
    const int total = warp_exclusive_scan128(off);
    const int nact = warp_exclusive_scan128(flag);  // flag[] now holds the act-list position
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ex = 4 * lane + i;
      s_off[ex] = off[i];
      if (chunk == 0) {
        a.meta[kMetaCounts + ex] = cnt[i];
        a.meta[kMetaOffsets + ex] = off[i];
        if (cnt[i] > 0) a.meta[kMetaAct + flag[i]] = ex;
      }
    }
    if (lane == 0) {
      s_off[kE] = total;
      if (chunk == 0) {
        a.meta[kMetaOffsets + kE] = total;
        a.meta[kMetaNAct] = nact;
      }
    }
  }
  __syncthreads();
  const int s = chunk * kChunk + tid;
  if (s < a.S) {
    if (e < 0) {
      a.slot_pos[s] = -1;
    } else {
      const int pos = s_off[e] + s_base[e] + rank;
      a.sorted_slot[pos] = s;
      a.slot_pos[s] = pos;
    }
  }
}

// One thread per dense slot s = t*128 + e: its sorted position e*T + t, and
// its weight (the token's routing weight for e, 0 if e is not among its
// ids).  Block 0 also writes the meta block.
__global__ void __launch_bounds__(256) dense_permute_kernel(const int32_t* __restrict__ ids,
                                                            const float* __restrict__ wts, int T,
                                                            int* __restrict__ meta, int* __restrict__ sorted_slot,
                                                            int* __restrict__ slot_pos, float* __restrict__ wdense,
                                                            int* status) {
  const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && threadIdx.x <= kE) {
    const int e = threadIdx.x;
    if (e < kE) {
      meta[kMetaCounts + e] = T;
      meta[kMetaAct + e] = e;
    }
    meta[kMetaOffsets + e] = e * T;
    if (e == 0) meta[kMetaNAct] = kE;
  }
  if (s >= (int64_t)T * kE) return;
  const int t = (int)(s / kE), e = (int)(s % kE);
  float w = 0.f;
#pragma unroll
  for (int j = 0; j < kTopK; ++j) {
    const int id = ids[t * kTopK + j];
    if (id < 0 || id >= kE) record_status(status, kStatusDevice);
    if (id == e) w = wts[t * kTopK + j];
  }
  const int pos = e * T + t;
  sorted_slot[pos] = (int)s;
  slot_pos[s] = pos;
  wdense[s] = w;
}

}  // namespace

cudaError_t launch_dense_permute(const int32_t* ids, const float* wts, int T, int* meta, int* sorted_slot,
                                 int* slot_pos, float* wdense, int* status, cudaStream_t st) {
  const int64_t n = (int64_t)T * kE;
  dense_permute_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(ids, wts, T, meta, sorted_slot, slot_pos, wdense,
                                                                      status);
  return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
  permute_count_kernel<<<a.nchunks, kChunk, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  permute_scatter_kernel<<<a.nchunks, kChunk, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
