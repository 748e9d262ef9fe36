// Device cache of group summaries ("Long-Context Fine-Tuning with Limited VRAM", gist.science
// Technical Summary 2.1 "Group Selection": the group summaries are cached in device memory and the
// missing ones are fetched from host memory; 2.2 "Tiered Memory Hierarchy": the chunk summaries stay
// resident).  The unit of the cache is a chunk: its 8 group summaries (8 x 128 float32 = 4 KB, one
// contiguous piece of the group-summary table) occupy one slot.
//
// gcache_plan_kernel: one CTA per (batch, KV head).  Marks in a shared-memory bitmap every chunk any
//   query block chose this step; a chosen chunk already in a slot is a hit (its slot's stamp is set
//   to the step); the chosen chunks without a slot (the misses, in ascending chunk order) take the
//   slots holding no chosen chunk, least recently used first (ordered by stamp, then slot; empty
//   slots carry stamp -1), whose old chunks lose their slot.  Writes the miss list (chunk, slot) and
//   the (hits, misses) counts.  More misses than such slots (a cache smaller than the step's chunk
//   set) records HGA_ERR_ARG and leaves the extra misses without a slot.
// gcache_fetch_kernel: one warp per miss copies the chunk's 8 group summaries from the table in host
//   memory (read by the SMs over the host link; device memory works too) into its slot, all of a
//   lane's 16-byte loads in flight together.
#include <cuda_runtime.h>

#include "common.cuh"

namespace hga {

constexpr int kPlanThreadsG = 1024;
constexpr int kMaxCacheSlots = 4096;

// Exclusive prefix sum of one int per thread over the CTA; *total gets the sum.  wt: >= 32 ints.
__device__ int gc_block_scan(int v, int* wt, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wt[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? wt[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) wt[lane] = s;
  }
  __syncthreads();
  const int before = (warp ? wt[warp - 1] : 0) + x - v;
  *total = wt[nw - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kPlanThreadsG) gcache_plan_kernel(const int32_t* __restrict__ chunk_idx, int nidx,
                                                                   int nchs, int cap, int step, int32_t* slot_of,
                                                                   int32_t* chunk_of, int32_t* stamp,
                                                                   int32_t* __restrict__ miss_chunk,
                                                                   int32_t* __restrict__ miss_slot,
                                                                   int32_t* __restrict__ counts, int* status) {
  extern __shared__ uint32_t gsm[];
  const int nwords = (nchs + 31) >> 5;
  uint32_t* need = gsm;                                       // [nwords] chunks chosen this step
  int* misses = reinterpret_cast<int*>(need + nwords);        // [cap] missed chunks, ascending
  int* victim = misses + cap;                                 // [cap] free slot of LRU rank r
  int* wt = victim + cap;                                     // [32]
  const int64_t bkh = blockIdx.x;
  const int32_t* ci = chunk_idx + bkh * nidx;
  int32_t* so = slot_of + bkh * nchs;
  int32_t* co = chunk_of + bkh * cap;
  int32_t* st = stamp + bkh * cap;
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();                                                 // the chunk indices come from the router

  for (int w = threadIdx.x; w < nwords; w += blockDim.x) need[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < nidx; i += blockDim.x) {
    const int32_t c = ci[i];
    if (c < 0 || c >= nchs) {
      set_status(status, -1);
      continue;
    }
    atomicOr(&need[c >> 5], 1u << (c & 31));
  }
  __syncthreads();

  // hits refresh their stamps; misses are counted, then listed in ascending chunk order (each thread
  // takes a contiguous run of bitmap words)
  const int per = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = min(nwords, (int)threadIdx.x * per), w1 = min(nwords, w0 + per);
  int hit = 0, miss = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = need[w];
    while (m) {
      const int c = (w << 5) + __ffs(m) - 1;
      m &= m - 1u;
      const int32_t s = so[c];
      if (s >= 0 && s < cap) {
        st[s] = step;
        ++hit;
      } else {
        ++miss;
      }
    }
  }
  int nhit, nmiss;
  gc_block_scan(hit, wt, &nhit);
  int pos = gc_block_scan(miss, wt, &nmiss);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = need[w];
    while (m) {
      const int c = (w << 5) + __ffs(m) - 1;
      m &= m - 1u;
      const int32_t s = so[c];
      if (!(s >= 0 && s < cap) && pos < cap) misses[pos++] = c;
    }
  }
  __syncthreads();

  // free slots: those whose chunk (if any) was not chosen; LRU rank by (stamp, slot)
  auto is_free = [&](int s) {
    const int32_t c = co[s];
    return c < 0 || c >= nchs || !((need[c >> 5] >> (c & 31)) & 1u);
  };
  int nfree_part = 0;
  for (int s = threadIdx.x; s < cap; s += blockDim.x) {
    if (!is_free(s)) continue;
    ++nfree_part;
    const int32_t ks = st[s];
    int rank = 0;
    for (int s2 = 0; s2 < cap; ++s2) {
      if (s2 == s || !is_free(s2)) continue;
      const int32_t k2 = st[s2];
      rank += (k2 < ks) || (k2 == ks && s2 < s);
    }
    if (rank < cap) victim[rank] = s;
  }
  int nfree;
  gc_block_scan(nfree_part, wt, &nfree);
  const int placed = min(nmiss, nfree);
  if (threadIdx.x == 0 && nmiss > nfree) set_status(status, -1);   // the cache is smaller than this step's chunk set

  // the i-th miss goes to the free slot of LRU rank i, whose old chunk loses its slot (old chunks are
  // not chosen this step, the missed ones are: the two sets of writes never meet)
  for (int i = threadIdx.x; i < placed; i += blockDim.x) {
    const int s = victim[i];
    const int32_t old = co[s];
    if (old >= 0 && old < nchs) so[old] = -1;
    co[s] = misses[i];
    so[misses[i]] = s;
    st[s] = step;
    miss_chunk[bkh * cap + i] = misses[i];
    miss_slot[bkh * cap + i] = s;
  }
  if (threadIdx.x == 0) {
    counts[2 * bkh] = nhit;
    counts[2 * bkh + 1] = placed;
  }
}

size_t gcache_plan_smem_bytes(int nchs, int cap) {
  return ((size_t)((nchs + 31) / 32) + 2 * (size_t)cap + 32) * sizeof(uint32_t);
}

cudaError_t launch_gcache_plan(const int32_t* chunk_idx, int BHkv, int nidx, int nchs, int cap, int step,
                               int32_t* slot_of, int32_t* chunk_of, int32_t* stamp, int32_t* miss_chunk,
                               int32_t* miss_slot, int32_t* counts, int* status, cudaStream_t st) {
  if (BHkv == 0) return cudaSuccess;
  const size_t smem = gcache_plan_smem_bytes(nchs, cap);
  cudaError_t e = cudaFuncSetAttribute(gcache_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(gcache_plan_kernel, dim3((unsigned)BHkv), dim3(kPlanThreadsG), smem, st, 1, chunk_idx, nidx,
                       nchs, cap, step, slot_of, chunk_of, stamp, miss_chunk, miss_slot, counts, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One warp per miss: the 8 group summaries of chunk miss_chunk[i] (4 KB) into slot miss_slot[i].
__global__ void __launch_bounds__(256) gcache_fetch_kernel(const float4* __restrict__ gsum, int64_t ngrs,
                                                           const int32_t* __restrict__ miss_chunk,
                                                           const int32_t* __restrict__ miss_slot,
                                                           const int32_t* __restrict__ counts, int cap,
                                                           float4* __restrict__ gcache) {
  constexpr int kVec = kGroup * kD / 4;          // float4 per chunk: 256, 8 per lane
  const int lane = threadIdx.x & 31;
  const int64_t bkh = blockIdx.x;
  const int i = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();                                    // the miss list comes from the plan kernel
  if (i >= counts[2 * bkh + 1]) return;
  const int64_t c = miss_chunk[bkh * cap + i];
  const int64_t s = miss_slot[bkh * cap + i];
  const float4* src = gsum + (bkh * ngrs + c * kGroup) * (kD / 4);
  float4* dst = gcache + (bkh * cap + s) * kVec;
  float4 v[kVec / 32];
#pragma unroll
  for (int k = 0; k < kVec / 32; ++k) v[k] = src[k * 32 + lane];
#pragma unroll
  for (int k = 0; k < kVec / 32; ++k) dst[k * 32 + lane] = v[k];
}

cudaError_t launch_gcache_fetch(const float* gsum, int64_t ngrs, const int32_t* miss_chunk, const int32_t* miss_slot,
                                const int32_t* counts, int BHkv, int cap, float* gcache, cudaStream_t st) {
  if (BHkv == 0) return cudaSuccess;
  const dim3 grid((unsigned)BHkv, (unsigned)((cap + 7) / 8));
  cudaError_t e = launch_dependent(gcache_fetch_kernel, grid, dim3(256), 0, st, 1,
                                   reinterpret_cast<const float4*>(gsum), ngrs, miss_chunk, miss_slot, counts, cap,
                                   reinterpret_cast<float4*>(gcache));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hga
