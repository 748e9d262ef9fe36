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
template <typename T>
__global__ void __launch_bounds__(256) summaries_kernel(const T* __restrict__ k_hist,
                                                        float* __restrict__ group_sum,
                                                        float* __restrict__ chunk_sum,
                                                        int64_t n_chunks_total) {
  constexpr int N = Vec16<T>::N;              // elements per 16-byte load
  constexpr int LPR = kD / N;                 // lanes per row (16 bf16, 32 f32)
  constexpr int RPL = 32 / LPR;               // rows per warp-wide load (2 or 1)
  constexpr int LOADS = kGroup / RPL;         // loads per lane
  __shared__ float gmean[kChunk / kGroup][kD];
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t chunk = blockIdx.x;
  if (chunk >= n_chunks_total) return;
  const int col = (lane % LPR) * N;
  const int rsub = lane / LPR;
  const T* base = k_hist + (chunk * kChunk + (int64_t)g * kGroup + rsub) * kD + col;
  float v[LOADS][N];
#pragma unroll
  for (int i = 0; i < LOADS; ++i) Vec16<T>::load(base + (int64_t)i * RPL * kD, v[i]);
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

cudaError_t launch_summaries(bool bf16, const void* k_hist, float* group_sum, float* chunk_sum,
                             int64_t n_chunks_total, cudaStream_t stream) {
  if (n_chunks_total == 0) return cudaSuccess;
  if (bf16)
    summaries_kernel<__nv_bfloat16><<<(unsigned)n_chunks_total, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_hist), group_sum, chunk_sum, n_chunks_total);
  else
    summaries_kernel<float><<<(unsigned)n_chunks_total, 256, 0, stream>>>(
        static_cast<const float*>(k_hist), group_sum, chunk_sum, n_chunks_total);
  return cudaGetLastError();
}

}  // namespace hga
