// Key summaries for HGA routing: one mean vector per 8-token group and per
// 64-token chunk of the detached history ("Long-Context Fine-Tuning with
// Limited VRAM", gist.science Technical Summary 2.1 "Chunk Selection" and
// "Group Selection"; pith.science review, Figure 1 caption).
//
// HBM-bound streaming reduction.  One warp owns one chunk (64 rows x 128 dims):
// every lane issues 16-byte loads covering 8 bf16 (or 4 f32) of a row, two
// groups' worth of loads are kept in flight, the group mean is formed with one
// shuffle between the row-halves of the warp, and the chunk mean is the mean
// of its eight group means.  Each byte of k_hist is read exactly once.
#include "common.cuh"

namespace hga {

template <typename T>
__global__ void __launch_bounds__(256) summaries_kernel(const T* __restrict__ k_hist,
                                                        float* __restrict__ group_sum,
                                                        float* __restrict__ chunk_sum,
                                                        int64_t n_chunks_total) {
  constexpr int N = Vec16<T>::N;              // elements per 16-byte load
  constexpr int LPR = kD / N;                 // lanes per row (16 bf16, 32 f32)
  constexpr int RPL = 32 / LPR;               // rows per warp-wide load (2 or 1)
  constexpr int LOADS = kGroup / RPL;         // loads per lane per group
  const int lane = threadIdx.x & 31;
  const int64_t chunk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (chunk >= n_chunks_total) return;
  const int col = (lane % LPR) * N;
  const int rsub = lane / LPR;
  const T* base = k_hist + chunk * (int64_t)kChunk * kD + (int64_t)rsub * kD + col;
  float csum[N];
#pragma unroll
  for (int e = 0; e < N; ++e) csum[e] = 0.f;

#pragma unroll
  for (int g0 = 0; g0 < kChunk / kGroup; g0 += 2) {
    float v[2][LOADS][N];
#pragma unroll
    for (int gg = 0; gg < 2; ++gg)
#pragma unroll
      for (int i = 0; i < LOADS; ++i)
        Vec16<T>::load(base + (int64_t)((g0 + gg) * kGroup + i * RPL) * kD, v[gg][i]);
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      float acc[N];
#pragma unroll
      for (int e = 0; e < N; ++e) {
        acc[e] = 0.f;
#pragma unroll
        for (int i = 0; i < LOADS; ++i) acc[e] += v[gg][i][e];
        if (RPL == 2) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
        acc[e] *= (1.0f / kGroup);
        csum[e] += acc[e];
      }
      if (rsub == 0) {
        float* dst = group_sum + (chunk * (kChunk / kGroup) + g0 + gg) * kD + col;
#pragma unroll
        for (int e = 0; e < N; e += 4) store4(dst + e, make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
      }
    }
  }
  if (rsub == 0) {
    float* dst = chunk_sum + chunk * kD + col;
#pragma unroll
    for (int e = 0; e < N; e += 4)
      store4(dst + e, make_float4(csum[e] * (1.0f / 8), csum[e + 1] * (1.0f / 8), csum[e + 2] * (1.0f / 8),
                                  csum[e + 3] * (1.0f / 8)));
  }
}

cudaError_t launch_summaries(bool bf16, const void* k_hist, float* group_sum, float* chunk_sum,
                             int64_t n_chunks_total, cudaStream_t stream) {
  if (n_chunks_total == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (n_chunks_total + warps - 1) / warps;
  if (bf16)
    summaries_kernel<__nv_bfloat16><<<(unsigned)blocks, warps * 32, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_hist), group_sum, chunk_sum, n_chunks_total);
  else
    summaries_kernel<float><<<(unsigned)blocks, warps * 32, 0, stream>>>(
        static_cast<const float*>(k_hist), group_sum, chunk_sum, n_chunks_total);
  return cudaGetLastError();
}

}  // namespace hga
