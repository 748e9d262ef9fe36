// Key summaries for HGA routing: one mean vector per 8-token group and per
// 64-token chunk of the detached history ("Long-Context Fine-Tuning with
// Limited VRAM", gist.science Technical Summary 2.1 "Chunk Selection" and
// "Group Selection"; pith.science review, Figure 1 caption).
//
// HBM-bound streaming reduction: one CTA per chunk, one warp per 8-row group, every
// lane's 16-byte loads (8 bf16 or 4 f32) in flight together; the group mean takes
// one shuffle between the row-halves of the warp, the chunk mean is the mean of
// the eight group means.  Each byte of k_hist is read exactly once.
#include "common.cuh"

namespace hga {

// One CTA per 64-key chunk; warp w reduces group w (8 rows) with all of its 16-byte loads in flight
// at once, writes the group mean, and the chunk mean is the mean of the eight group means (shared
// memory).  Every byte of k_hist is read exactly once.
// Chunks [c0, c0 + nc) of every (batch, KV head): history rows bkh * Hs + ..., summary rows
// bkh * Hs / 8 + ... and bkh * Hs / 64 + ... (Hs = rows per (batch, KV head) of the buffers).
template <typename T>
__global__ void __launch_bounds__(256) summaries_kernel(const T* __restrict__ k_hist,
                                                        float* __restrict__ group_sum,
                                                        float* __restrict__ chunk_sum, int64_t Hs,
                                                        int64_t c0, int64_t nc) {
  constexpr int N = Vec16<T>::N;              // elements per 16-byte load
  constexpr int LPR = kD / N;                 // lanes per row (16 bf16, 32 f32)
  constexpr int RPL = 32 / LPR;               // rows per warp-wide load (2 or 1)
  constexpr int LOADS = kGroup / RPL;         // loads per lane
  __shared__ float gmean[kChunk / kGroup][kD];
  if (threadIdx.x == 0) pdl_trigger();          // the router may start its block-query means
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t bkh = blockIdx.x / nc;
  const int64_t c = c0 + blockIdx.x % nc;
  const int64_t chunk = bkh * (Hs / kChunk) + c;        // chunk row in the chunk-summary buffer
  const int col = (lane % LPR) * N;
  const int rsub = lane / LPR;
  const T* base = k_hist + (bkh * Hs + c * kChunk + (int64_t)g * kGroup + rsub) * kD + col;
  // streaming loads (evict first): the history is read once here, and its lines would otherwise push
  // the summaries this kernel writes, which the router reads next, out of L2 (131K: 47 against 51 us)
  float v[LOADS][N];
  {
    uint4 raw[LOADS];
#pragma unroll
    for (int i = 0; i < LOADS; ++i) raw[i] = __ldcs(reinterpret_cast<const uint4*>(base + (int64_t)i * RPL * kD));
#pragma unroll
    for (int i = 0; i < LOADS; ++i) Vec16<T>::load(reinterpret_cast<const T*>(&raw[i]), v[i]);
  }
  float acc[N];
#pragma unroll
  for (int e = 0; e < N; ++e) {
    acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < LOADS; ++i) acc[e] += v[i][e];
    if (RPL == 2) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    acc[e] *= (1.0f / kGroup);
  }
  if (rsub == 0) {
    float* dst = group_sum + (chunk * (kChunk / kGroup) + g) * kD + col;
#pragma unroll
    for (int e = 0; e < N; e += 4) {
      store4(dst + e, make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
      *reinterpret_cast<float4*>(&gmean[g][col + e]) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    }
  }
  __syncthreads();
  if (threadIdx.x < kD) {
    float cs = 0.f;
#pragma unroll
    for (int j = 0; j < kChunk / kGroup; ++j) cs += gmean[j][threadIdx.x];
    chunk_sum[chunk * kD + threadIdx.x] = cs * (1.0f / (kChunk / kGroup));
  }
}

cudaError_t launch_summaries(bool bf16, const void* k_hist, float* group_sum, float* chunk_sum, int64_t BHkv,
                             int64_t Hs, int64_t c0, int64_t c1, cudaStream_t stream) {
  const int64_t nc = c1 - c0;
  if (BHkv == 0 || nc <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)(BHkv * nc);
  if (bf16)
    summaries_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(k_hist), group_sum,
                                                              chunk_sum, Hs, c0, nc);
  else
    summaries_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(k_hist), group_sum, chunk_sum, Hs,
                                                      c0, nc);
  return cudaGetLastError();
}

}  // namespace hga
