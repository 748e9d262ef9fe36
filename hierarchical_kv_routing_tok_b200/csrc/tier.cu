// Tiered history storage ("Long-Context Fine-Tuning with Limited VRAM", gist.science Technical
// Summary 2.2 "Tiered Memory Hierarchy"; pith.science review, Figure 2 caption): the detached
// history K/V live in host memory, the summaries stay in device memory, and a layer step brings
// into device memory only the exact K/V of the groups its routing selected.
//
// tier_plan_kernel: one CTA per (batch, KV head) marks, in a shared-memory bitmap over the H/8
//   history groups, every group any query block of the step routed to (plus the sink groups),
//   turns the bitmap into the ascending list of used groups and rewrites each block's group
//   indices as positions in that list.  Positions keep the order of the group indices, so
//   attention over the compact cache visits the same keys in the same order as attention over
//   the full history and gives the same result bit for bit.
// tier_gather_kernel: one warp per used group copies its 8 K rows and 8 V rows from the history
//   (pinned host memory read over the host link by the SMs, or device memory) into the compact
//   cache, all 16-byte loads of a group in flight together.
#include <cuda_runtime.h>

#include "common.cuh"

namespace hga {

constexpr int kPlanThreads = 1024;

// Exclusive prefix sum over the block of one int per thread; returns this thread's prefix and the
// block total in *total.  `warp_tot` holds >= 32 ints of shared memory.
__device__ int plan_block_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) warp_tot[lane] = t;             // inclusive warp prefix
  }
  __syncthreads();
  const int before = (warp ? warp_tot[warp - 1] : 0) + x - v;
  *total = warp_tot[nw - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kPlanThreads) tier_plan_kernel(const int32_t* __restrict__ group_idx, int nblk,
                                                                 int kg, int nsg, int ngr, int cap,
                                                                 int32_t* __restrict__ used_groups,
                                                                 int32_t* __restrict__ n_used,
                                                                 int32_t* __restrict__ compact_idx, int* status) {
  extern __shared__ uint32_t plan_smem[];
  const int nwords = (ngr + 31) >> 5;
  uint32_t* bits = plan_smem;                                    // [nwords]
  int* wpre = reinterpret_cast<int*>(bits + nwords);             // [nwords] used groups before word w
  int* warp_tot = wpre + nwords;                                 // [32]
  const int64_t bkh = blockIdx.x;
  const int nidx = nblk * kg;
  const int32_t* gi = group_idx + bkh * nidx;

  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bits[w] = 0u;
  __syncthreads();
  for (int g = threadIdx.x; g < nsg; g += blockDim.x) atomicOr(&bits[g >> 5], 1u << (g & 31));
  for (int i = threadIdx.x; i < nidx; i += blockDim.x) {
    const int32_t g = gi[i];
    if (g < nsg || g >= ngr) {
      set_status(status, -1);
      continue;
    }
    atomicOr(&bits[g >> 5], 1u << (g & 31));
  }
  __syncthreads();

  // prefix of the per-word counts: each thread takes a contiguous run of words
  const int per = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = min(nwords, (int)threadIdx.x * per), w1 = min(nwords, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
  int total;
  int run = plan_block_scan(cnt, warp_tot, &total);
  for (int w = w0; w < w1; ++w) {
    wpre[w] = run;
    run += __popc(bits[w]);
  }
  __syncthreads();
  if (threadIdx.x == 0) n_used[bkh] = total;

  // the used groups, ascending
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
    uint32_t m = bits[w];
    int s = wpre[w];
    while (m) {
      const int b = __ffs(m) - 1;
      if (s < cap) used_groups[bkh * cap + s] = (w << 5) + b;
      ++s;
      m &= m - 1u;
    }
  }
  // every block's routed indices as positions in that list (an invalid index maps to 0)
  for (int i = threadIdx.x; i < nidx; i += blockDim.x) {
    const int32_t g = gi[i];
    int32_t pos = 0;
    if (g >= nsg && g < ngr) pos = wpre[g >> 5] + __popc(bits[g >> 5] & ((1u << (g & 31)) - 1u));
    compact_idx[bkh * nidx + i] = pos;
  }
}

size_t tier_plan_smem_bytes(int ngr) {
  const size_t nwords = ((size_t)ngr + 31) / 32;
  return (2 * nwords + 32) * sizeof(uint32_t);
}

cudaError_t launch_tier_plan(const int32_t* group_idx, int BHkv, int nblk, int kg, int nsg, int ngr, int cap,
                             int32_t* used_groups, int32_t* n_used, int32_t* compact_idx, int* status,
                             cudaStream_t st) {
  if (BHkv == 0) return cudaSuccess;
  const size_t smem = tier_plan_smem_bytes(ngr);
  cudaError_t e = cudaFuncSetAttribute(tier_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  tier_plan_kernel<<<(unsigned)BHkv, kPlanThreads, smem, st>>>(group_idx, nblk, kg, nsg, ngr, cap, used_groups,
                                                              n_used, compact_idx, status);
  return cudaGetLastError();
}

// One warp per cache slot: group used[bkh][slot] of the history (8 rows of row_bytes) -> slot.
template <int NV>     // 16-byte vectors per lane per tensor (8 rows x row_bytes / 16 / 32)
__global__ void __launch_bounds__(256) tier_gather_kernel(const uint4* __restrict__ kh, const uint4* __restrict__ vh,
                                                          const int32_t* __restrict__ used_groups,
                                                          const int32_t* __restrict__ n_used, int64_t Hs, int cap,
                                                          uint4* __restrict__ kc, uint4* __restrict__ vc) {
  const int lane = threadIdx.x & 31;
  const int64_t bkh = blockIdx.x;
  const int slot = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (slot >= cap || slot >= n_used[bkh]) return;
  const int64_t g = used_groups[bkh * cap + slot];
  constexpr int kVecPerGroup = 32 * NV;
  const uint4* ks = kh + (bkh * Hs + g * kGroup) * (kVecPerGroup / kGroup);
  const uint4* vs = vh + (bkh * Hs + g * kGroup) * (kVecPerGroup / kGroup);
  uint4* kd = kc + (bkh * cap + slot) * (int64_t)kVecPerGroup;
  uint4* vd = vc + (bkh * cap + slot) * (int64_t)kVecPerGroup;
  uint4 a[NV], b[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    a[i] = ks[i * 32 + lane];
    b[i] = vs[i * 32 + lane];
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    kd[i * 32 + lane] = a[i];
    vd[i * 32 + lane] = b[i];
  }
}

cudaError_t launch_tier_gather(bool bf16, const void* kh, const void* vh, const int32_t* used_groups,
                               const int32_t* n_used, int BHkv, int64_t Hs, int cap, void* kc, void* vc,
                               cudaStream_t st) {
  if (BHkv == 0 || cap == 0) return cudaSuccess;
  const dim3 grid((unsigned)BHkv, (unsigned)((cap + 7) / 8));
  const auto* k4 = static_cast<const uint4*>(kh);
  const auto* v4 = static_cast<const uint4*>(vh);
  if (bf16)   // 8 rows x 256 bytes = 128 vectors per group: 4 per lane
    tier_gather_kernel<4><<<grid, 256, 0, st>>>(k4, v4, used_groups, n_used, Hs, cap, static_cast<uint4*>(kc),
                                                static_cast<uint4*>(vc));
  else        // 8 rows x 512 bytes: 8 per lane
    tier_gather_kernel<8><<<grid, 256, 0, st>>>(k4, v4, used_groups, n_used, Hs, cap, static_cast<uint4*>(kc),
                                                static_cast<uint4*>(vc));
  return cudaGetLastError();
}

}  // namespace hga
