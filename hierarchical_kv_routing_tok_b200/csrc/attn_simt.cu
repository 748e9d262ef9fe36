// Routed + causal-local attention, forward and backward, on the CUDA cores with
// float32 arithmetic ("Long-Context Fine-Tuning with Limited VRAM",
// gist.science Technical Summary 2.1 "Exact-Token Attention" and 2.2 detached
// history; softmax-attention backward in the FlashAttention form cited there).
//
// This is the float32 path (tolerance 1e-4 against the float64 oracle) and the
// reference-grade path for any element type.  One CTA owns 64 query rows of one
// head; the key sequence of a row is [8*k_g routed history tokens | segment
// tokens 0..t], processed in 64-key tiles staged in shared memory with an
// online softmax (exp2 domain).
//
// Backward: a preprocess kernel forms delta = rowsum(dO * O); a dQ kernel per
// (head, query block) walks routed + local keys; a dK/dV kernel per (KV head,
// key block) walks the G query heads and the query blocks at or after the key
// block (local causal pairs only: history is detached, so routed keys get no
// gradient).  No atomics: every output element has one owner.
#include <math.h>

#include "common.cuh"

namespace hga {

namespace simt {

constexpr int BM = 64;            // query rows per CTA
constexpr int BN = 64;            // keys per tile
constexpr int LD = kD + 4;        // padded row stride of [64][128] tiles (floats)
constexpr int LP = BN + 4;        // padded row stride of [64][64] tiles
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

// Load a [64][128] tile of rows given by row_ptr(r) (nullptr = zero row) into smem, scaled.
template <typename T, typename RowPtr>
__device__ __forceinline__ void load_tile(float* dst, RowPtr row_ptr, float mul) {
  constexpr int N = Vec16<T>::N;
  constexpr int LPR = kD / N;                    // threads per row
  constexpr int RPI = kThreads / LPR;            // rows per iteration
  const int col = (threadIdx.x % LPR) * N;
  for (int r = threadIdx.x / LPR; r < BN; r += RPI) {
    const T* src = row_ptr(r);
    float v[N];
    if (src) {
      Vec16<T>::load(src + col, v);
    } else {
#pragma unroll
      for (int e = 0; e < N; ++e) v[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < N; e += 4)
      store4(dst + r * LD + col + e, make_float4(v[e] * mul, v[e + 1] * mul, v[e + 2] * mul, v[e + 3] * mul));
  }
}

// acc[i][j] += A[4ty+i] . B[tx+16j] over 128 dims (A, B: [64][LD] smem tiles).
__device__ __forceinline__ void mm_rows_cols(const float* A, const float* Bt, float acc[4][4]) {
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
#pragma unroll 4
  for (int d = 0; d < kD; d += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(A + (4 * ty + i) * LD + d);
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = *reinterpret_cast<const float4*>(Bt + (tx + 16 * j) * LD + d);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        acc[i][j] += a[i].x * b[j].x + a[i].y * b[j].y + a[i].z * b[j].z + a[i].w * b[j].w;
  }
}

// out[i][0..7] += sum_k P[4ty+i][k] * V[k][cols], cols = 4tx..4tx+3, 64+4tx..64+4tx+3.
__device__ __forceinline__ void mm_p_v(const float* P, const float* V, float out[4][8]) {
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
#pragma unroll 4
  for (int k = 0; k < BN; ++k) {
    const float4 v0 = *reinterpret_cast<const float4*>(V + k * LD + 4 * tx);
    const float4 v1 = *reinterpret_cast<const float4*>(V + k * LD + 64 + 4 * tx);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = P[(4 * ty + i) * LP + k];
      out[i][0] += p * v0.x; out[i][1] += p * v0.y; out[i][2] += p * v0.z; out[i][3] += p * v0.w;
      out[i][4] += p * v1.x; out[i][5] += p * v1.y; out[i][6] += p * v1.z; out[i][7] += p * v1.w;
    }
  }
}

__device__ __forceinline__ float half_warp_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct Dims {
  int Hq, Hkv, G, kg, nblk;
  int nsg;              // sink groups at the start of every block's history key list
  int64_t H, S;
  int64_t Hs;           // history rows per (batch, KV head) in k_hist / v_hist (>= H)
  float scale;
  int* status;          // workspace status word (HGA_ERR_ARG recorded for an out-of-range group index)
};

// Source row of key r of the key list of block n of KV head (b, kh): the first 8*(nsg + kg) keys
// are history tokens (the sink window, then the routed groups), then segment tokens 0.. (the
// caller masks u > t).  A routed group index outside [nsg, H/8) is never dereferenced: the key
// reads as zeros and the status word records HGA_ERR_ARG (-1).
template <typename T>
__device__ __forceinline__ const T* key_row(const T* hist, const T* seg, const int32_t* gi, const Dims& dm,
                                            int64_t r, int64_t n_keys) {
  if (r >= n_keys) return nullptr;
  const int64_t n_hist = 8LL * (dm.nsg + dm.kg);
  if (r < n_hist) {
    const int32_t g = routed_group(gi, (int)(r >> 3), dm.nsg, dm.kg, dm.H / kGroup, dm.status);
    if (g < 0) return nullptr;
    return hist + ((int64_t)g * kGroup + (r & 7)) * kD;
  }
  return seg + (r - n_hist) * kD;
}

// ------------------------------------------------------------------------------------ forward
template <typename T>
__global__ void __launch_bounds__(kThreads) fwd_kernel(const T* __restrict__ q, const T* __restrict__ k_hist,
                                                       const T* __restrict__ v_hist,
                                                       const T* __restrict__ k_seg,
                                                       const T* __restrict__ v_seg,
                                                       const int32_t* __restrict__ group_idx,
                                                       T* __restrict__ o, float* __restrict__ lse, Dims dm) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = Qs + BM * LD;
  float* Vs = Ks + BN * LD;
  float* Ps = Vs + BN * LD;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  // heavy blocks (late n) first
  const int n = dm.nblk - 1 - (int)(blockIdx.x % dm.nblk);
  const int bh = blockIdx.x / dm.nblk;             // b*Hq + h
  const int h = bh % dm.Hq, b = bh / dm.Hq;
  const int kh = h / dm.G;
  const int64_t bkh = (int64_t)b * dm.Hkv + kh;
  const T* qrow = q + ((int64_t)bh * dm.S + (int64_t)n * BM) * kD;
  const T* kh_base = k_hist + bkh * dm.Hs * kD;
  const T* vh_base = v_hist + bkh * dm.Hs * kD;
  const T* ks_base = k_seg + bkh * dm.S * kD;
  const T* vs_base = v_seg + bkh * dm.S * kD;
  const int32_t* gi = group_idx + (bkh * dm.nblk + n) * dm.kg;
  const int64_t n_route = 8LL * (dm.nsg + dm.kg);
  const int64_t n_keys = n_route + (int64_t)(n + 1) * BM;
  const float qmul = dm.scale * kLog2e;

  load_tile<T>(Qs, [&](int r) { return qrow + (int64_t)r * kD; }, qmul);

  float m[4], l[4], acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY; l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
  }
  for (int64_t k0 = 0; k0 < n_keys; k0 += BN) {
    __syncthreads();
    load_tile<T>(Ks, [&](int r) { return key_row(kh_base, ks_base, gi, dm, k0 + r, n_keys); }, 1.f);
    load_tile<T>(Vs, [&](int r) { return key_row(vh_base, vs_base, gi, dm, k0 + r, n_keys); }, 1.f);
    __syncthreads();
    float s[4][4] = {};
    mm_rows_cols(Qs, Ks, s);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t t = (int64_t)n * BM + 4 * ty + i;
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t r = k0 + tx + 16 * j;
        const bool ok = r < n_keys && (r < n_route || r - n_route <= t);
        s[i][j] = ok ? s[i][j] : -INFINITY;
        mx = fmaxf(mx, s[i][j]);
      }
      mx = half_warp_max(mx);
      const float mnew = fmaxf(m[i], mx);
      const float ref = (mnew == -INFINITY) ? 0.f : mnew;
      const float alpha = exp2f(m[i] - ref);           // 0 when m = -inf
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = exp2f(s[i][j] - ref);
        Ps[(4 * ty + i) * LP + tx + 16 * j] = p;
        rs += p;
      }
      rs = half_warp_sum(rs);
      l[i] = l[i] * alpha + rs;
      m[i] = mnew;
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[i][c] *= alpha;
    }
    __syncthreads();
    mm_p_v(Ps, Vs, acc);
  }
  // epilogue
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = 4 * ty + i;
    const float inv = 1.f / l[i];
    T* dst = o + ((int64_t)bh * dm.S + (int64_t)n * BM + row) * kD;
    store4(dst + 4 * tx, make_float4(acc[i][0] * inv, acc[i][1] * inv, acc[i][2] * inv, acc[i][3] * inv));
    store4(dst + 64 + 4 * tx, make_float4(acc[i][4] * inv, acc[i][5] * inv, acc[i][6] * inv, acc[i][7] * inv));
    if (tx == 0) lse[(int64_t)bh * dm.S + (int64_t)n * BM + row] = (m[i] + log2f(l[i])) * 0.6931471805599453f;
  }
}

// ------------------------------------------------------------------------------------ backward
// delta[row] = sum_d dO[row, d] * O[row, d].  Each warp owns 8 rows and keeps all of their
// 16-byte loads in flight at once (HBM-bound streaming kernel).
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_delta_kernel(const T* __restrict__ o, const T* __restrict__ d_o,
                                                             float* __restrict__ delta, int64_t rows) {
  constexpr int N = Vec16<T>::N;          // elements per 16-byte load
  constexpr int LPR = kD / N;             // lanes per row
  constexpr int RPW = 32 / LPR;           // rows per warp-wide load
  constexpr int ROWS = 8;                 // rows per warp
  constexpr int IT = ROWS / RPW;
  const int lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * ROWS;
  const int sub = lane / LPR, col = (lane % LPR) * N;
  float a[IT][N], c[IT][N];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int64_t row = row0 + it * RPW + sub;
    if (row < rows) {
      Vec16<T>::load(o + row * kD + col, a[it]);
      Vec16<T>::load(d_o + row * kD + col, c[it]);
    } else {
#pragma unroll
      for (int e = 0; e < N; ++e) a[it][e] = c[it][e] = 0.f;
    }
  }
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < N; ++e) sum = fmaf(a[it][e], c[it][e], sum);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const int64_t row = row0 + it * RPW + sub;
    if ((lane % LPR) == 0 && row < rows) delta[row] = sum;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k_hist,
                                                          const T* __restrict__ v_hist,
                                                          const T* __restrict__ k_seg,
                                                          const T* __restrict__ v_seg,
                                                          const int32_t* __restrict__ group_idx,
                                                          const T* __restrict__ d_o,
                                                          const float* __restrict__ lse,
                                                          const float* __restrict__ delta, T* __restrict__ dq,
                                                          Dims dm) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* dOs = Qs + BM * LD;
  float* Ks = dOs + BM * LD;
  float* Vs = Ks + BN * LD;
  float* dSs = Vs + BN * LD;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int n = dm.nblk - 1 - (int)(blockIdx.x % dm.nblk);
  const int bh = blockIdx.x / dm.nblk;
  const int h = bh % dm.Hq, b = bh / dm.Hq;
  const int kh = h / dm.G;
  const int64_t bkh = (int64_t)b * dm.Hkv + kh;
  const int64_t row0 = (int64_t)bh * dm.S + (int64_t)n * BM;
  const T* kh_base = k_hist + bkh * dm.Hs * kD;
  const T* vh_base = v_hist + bkh * dm.Hs * kD;
  const T* ks_base = k_seg + bkh * dm.S * kD;
  const T* vs_base = v_seg + bkh * dm.S * kD;
  const int32_t* gi = group_idx + (bkh * dm.nblk + n) * dm.kg;
  const int64_t n_route = 8LL * (dm.nsg + dm.kg);
  const int64_t n_keys = n_route + (int64_t)(n + 1) * BM;

  load_tile<T>(Qs, [&](int r) { return q + (row0 + r) * kD; }, dm.scale * kLog2e);
  load_tile<T>(dOs, [&](int r) { return d_o + (row0 + r) * kD; }, 1.f);
  float lse2[4], dl[4], acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lse2[i] = lse[row0 + 4 * ty + i] * kLog2e;
    dl[i] = delta[row0 + 4 * ty + i];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
  }
  for (int64_t k0 = 0; k0 < n_keys; k0 += BN) {
    __syncthreads();
    load_tile<T>(Ks, [&](int r) { return key_row(kh_base, ks_base, gi, dm, k0 + r, n_keys); }, 1.f);
    load_tile<T>(Vs, [&](int r) { return key_row(vh_base, vs_base, gi, dm, k0 + r, n_keys); }, 1.f);
    __syncthreads();
    float s[4][4] = {}, dp[4][4] = {};
    mm_rows_cols(Qs, Ks, s);
    mm_rows_cols(dOs, Vs, dp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t t = (int64_t)n * BM + 4 * ty + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t r = k0 + tx + 16 * j;
        const bool ok = r < n_keys && (r < n_route || r - n_route <= t);
        const float p = ok ? exp2f(s[i][j] - lse2[i]) : 0.f;
        dSs[(4 * ty + i) * LP + tx + 16 * j] = p * (dp[i][j] - dl[i]);
      }
    }
    __syncthreads();
    mm_p_v(dSs, Ks, acc);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    T* dst = dq + (row0 + 4 * ty + i) * kD;
    const float sc = dm.scale;
    store4(dst + 4 * tx, make_float4(acc[i][0] * sc, acc[i][1] * sc, acc[i][2] * sc, acc[i][3] * sc));
    store4(dst + 64 + 4 * tx, make_float4(acc[i][4] * sc, acc[i][5] * sc, acc[i][6] * sc, acc[i][7] * sc));
  }
}

// P^T-side products: out[i][c] += sum_q A[4ty+i][q] * B[q][cols] with A a [64][LP] tile.
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k_seg,
                                                            const T* __restrict__ v_seg,
                                                            const T* __restrict__ d_o,
                                                            const float* __restrict__ lse,
                                                            const float* __restrict__ delta,
                                                            T* __restrict__ dk, T* __restrict__ dv, Dims dm) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + BN * LD;
  float* Qs = Vs + BN * LD;
  float* dOs = Qs + BM * LD;
  float* Pt = dOs + BM * LD;
  float* dSt = Pt + BN * LP;
  float* rowstat = dSt + BN * LP;                  // lse2[64], delta[64]
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int mblk = (int)(blockIdx.x % dm.nblk);   // key block: heavy (early) ones first
  const int bkh_i = blockIdx.x / dm.nblk;
  const int kh = bkh_i % dm.Hkv, b = bkh_i / dm.Hkv;
  const int64_t key0 = (int64_t)bkh_i * dm.S + (int64_t)mblk * BN;
  const float c2 = dm.scale * kLog2e;

  load_tile<T>(Ks, [&](int r) { return k_seg + (key0 + r) * kD; }, 1.f);
  load_tile<T>(Vs, [&](int r) { return v_seg + (key0 + r) * kD; }, 1.f);
  float dK[4][8], dV[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) { dK[i][c] = 0.f; dV[i][c] = 0.f; }

  for (int hh = 0; hh < dm.G; ++hh) {
    const int h = kh * dm.G + hh;
    const int64_t bh = (int64_t)b * dm.Hq + h;
    for (int n = mblk; n < dm.nblk; ++n) {
      const int64_t row0 = bh * dm.S + (int64_t)n * BM;
      __syncthreads();
      load_tile<T>(Qs, [&](int r) { return q + (row0 + r) * kD; }, 1.f);
      load_tile<T>(dOs, [&](int r) { return d_o + (row0 + r) * kD; }, 1.f);
      if (threadIdx.x < BM) {
        rowstat[threadIdx.x] = lse[row0 + threadIdx.x] * kLog2e;
        rowstat[BM + threadIdx.x] = delta[row0 + threadIdx.x];
      }
      __syncthreads();
      float s[4][4] = {}, dp[4][4] = {};
      mm_rows_cols(Ks, Qs, s);      // [key][query]
      mm_rows_cols(Vs, dOs, dp);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t u = (int64_t)mblk * BN + 4 * ty + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qc = tx + 16 * j;
          const int64_t t = (int64_t)n * BM + qc;
          const float p = (u <= t) ? exp2f(s[i][j] * c2 - rowstat[qc]) : 0.f;
          Pt[(4 * ty + i) * LP + qc] = p;
          dSt[(4 * ty + i) * LP + qc] = p * (dp[i][j] - rowstat[BM + qc]);
        }
      }
      __syncthreads();
      mm_p_v(Pt, dOs, dV);
      mm_p_v(dSt, Qs, dK);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = key0 + 4 * ty + i;
    const float sc = dm.scale;
    store4(dk + row * kD + 4 * tx, make_float4(dK[i][0] * sc, dK[i][1] * sc, dK[i][2] * sc, dK[i][3] * sc));
    store4(dk + row * kD + 64 + 4 * tx, make_float4(dK[i][4] * sc, dK[i][5] * sc, dK[i][6] * sc, dK[i][7] * sc));
    store4(dv + row * kD + 4 * tx, make_float4(dV[i][0], dV[i][1], dV[i][2], dV[i][3]));
    store4(dv + row * kD + 64 + 4 * tx, make_float4(dV[i][4], dV[i][5], dV[i][6], dV[i][7]));
  }
}

constexpr size_t kFwdSmem = (size_t)(BM * LD + 2 * BN * LD + BM * LP) * 4;
constexpr size_t kDqSmem = (size_t)(2 * BM * LD + 2 * BN * LD + BM * LP) * 4;
constexpr size_t kDkdvSmem = (size_t)(2 * BN * LD + 2 * BM * LD + 2 * BN * LP + 2 * BM) * 4;

template <typename T>
cudaError_t fwd(const void* q, const void* kh, const void* vh, const void* ks, const void* vs, const int32_t* gi,
                void* o, float* lse, int B, Dims dm, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFwdSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (int64_t)B * dm.Hq * dm.nblk;
  fwd_kernel<T><<<(unsigned)grid, kThreads, kFwdSmem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(kh), static_cast<const T*>(vh), static_cast<const T*>(ks),
      static_cast<const T*>(vs), gi, static_cast<T*>(o), lse, dm);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_delta(const void* o, const void* d_o, float* delta, int B, Dims dm, cudaStream_t st) {
  const int64_t rows = (int64_t)B * dm.Hq * dm.S;
  bwd_delta_kernel<T><<<(unsigned)((rows + 63) / 64), kThreads, 0, st>>>(static_cast<const T*>(o),
                                                                       static_cast<const T*>(d_o), delta, rows);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_dkdv(const void* q, const void* ks, const void* vs, const float* lse, const void* d_o,
                     const float* delta, void* dk, void* dv, int B, Dims dm, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDkdvSmem);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<T><<<(unsigned)((int64_t)B * dm.Hkv * dm.nblk), kThreads, kDkdvSmem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(ks), static_cast<const T*>(vs), static_cast<const T*>(d_o),
      lse, delta, static_cast<T*>(dk), static_cast<T*>(dv), dm);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_dq(const void* q, const void* kh, const void* vh, const void* ks, const void* vs, const int32_t* gi,
                   const float* lse, const void* d_o, const float* delta, void* dq, int B, Dims dm,
                   cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDqSmem);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<T><<<(unsigned)((int64_t)B * dm.Hq * dm.nblk), kThreads, kDqSmem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(kh), static_cast<const T*>(vh), static_cast<const T*>(ks),
      static_cast<const T*>(vs), gi, static_cast<const T*>(d_o), lse, delta, static_cast<T*>(dq), dm);
  return cudaGetLastError();
}

}  // namespace simt

cudaError_t launch_attn_fwd_simt(bool bf16, const void* q, const void* kh, const void* vh, const void* ks,
                                 const void* vs, const int32_t* gi, void* o, float* lse, int B, int Hq, int Hkv,
                                 int64_t H, int64_t S, int64_t Hs, int kg, int nsg, float scale, int* status,
                                 cudaStream_t st) {
  simt::Dims dm{Hq, Hkv, Hq / Hkv, kg, (int)(S / kQBlock), nsg, H, S, Hs, scale, status};
  return bf16 ? simt::fwd<__nv_bfloat16>(q, kh, vh, ks, vs, gi, o, lse, B, dm, st)
              : simt::fwd<float>(q, kh, vh, ks, vs, gi, o, lse, B, dm, st);
}

cudaError_t launch_bwd_delta_simt(bool bf16, const void* o, const void* d_o, float* delta, int B, int Hq,
                                  int64_t S, cudaStream_t st) {
  simt::Dims dm{Hq, 1, Hq, 0, (int)(S / kQBlock), 0, 0, S, 0, 0.f, nullptr};
  return bf16 ? simt::bwd_delta<__nv_bfloat16>(o, d_o, delta, B, dm, st)
              : simt::bwd_delta<float>(o, d_o, delta, B, dm, st);
}

cudaError_t launch_bwd_dkdv_simt(bool bf16, const void* q, const void* ks, const void* vs, const float* lse,
                                 const void* d_o, const float* delta, void* dk, void* dv, int B, int Hq, int Hkv,
                                 int64_t H, int64_t S, int kg, float scale, cudaStream_t st) {
  simt::Dims dm{Hq, Hkv, Hq / Hkv, kg, (int)(S / kQBlock), 0, H, S, H, scale, nullptr};
  return bf16 ? simt::bwd_dkdv<__nv_bfloat16>(q, ks, vs, lse, d_o, delta, dk, dv, B, dm, st)
              : simt::bwd_dkdv<float>(q, ks, vs, lse, d_o, delta, dk, dv, B, dm, st);
}

cudaError_t launch_bwd_dq_simt(bool bf16, const void* q, const void* kh, const void* vh, const void* ks,
                               const void* vs, const int32_t* gi, const float* lse, const void* d_o,
                               const float* delta, void* dq, int B, int Hq, int Hkv, int64_t H, int64_t S,
                               int64_t Hs, int kg, int nsg, float scale, int* status, cudaStream_t st) {
  simt::Dims dm{Hq, Hkv, Hq / Hkv, kg, (int)(S / kQBlock), nsg, H, S, Hs, scale, status};
  return bf16 ? simt::bwd_dq<__nv_bfloat16>(q, kh, vh, ks, vs, gi, lse, d_o, delta, dq, B, dm, st)
              : simt::bwd_dq<float>(q, kh, vh, ks, vs, gi, lse, d_o, delta, dq, B, dm, st);
}

}  // namespace hga
