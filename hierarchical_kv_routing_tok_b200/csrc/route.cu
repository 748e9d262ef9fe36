// Two-level HGA routing ("Long-Context Fine-Tuning with Limited VRAM",
// gist.science Technical Summary 2.1 "Chunk Selection" / "Group Selection";
// pith.science review Figure 1): the query block scores every history chunk
// summary, keeps the best top_chunks, then scores the 8 group summaries of
// each kept chunk and keeps the best top_groups.
//
// One CTA per (batch, KV head, 64-query block).  The block query (mean over
// the block's positions and the KV head's query heads) stays in shared memory,
// scores are warp dot products against float32 summaries (L2-resident), and
// the top-k is exact: a one-pass rank selection, a CTA-wide radix select on
// order-preserving 32-bit keys, or a threshold filter followed by the rank
// selection of the keys that pass it, whichever is cheapest for the level's size; all
// finish with an index-ordered compaction, so ties go to the lower index and the
// output comes out sorted ascending.  This is not a dense contraction
// (M = 1 per CTA), so it runs on the CUDA cores.
//
// The same kernel also runs the two levels separately, for routing with a device cache of group
// summaries (the group summaries of a long history in host memory, "Technical Summary" 2.1 Group
// Selection): mode 1 stops after level 1 and writes the chunk indices and the block query; mode 2
// starts from those and scores the group summaries of the chosen chunks from their cache slots.
//
// Long histories route in three launches instead of one, so that each chunk summary is read once
// per (batch, KV head) rather than once per query block: mode 3 forms the block queries;
// chunk_score_kernel scores every chunk of a (batch, KV head) against all of its block queries (a
// warp per chunk row, the row in registers, the block queries in shared memory); mode 4 selects
// each block's chunks from its row of scores and runs level 2 as mode 0 does.
#include "common.cuh"

namespace hga {

constexpr int kRouteThreads = 512;
// Choice of exact top-k for n candidates (cycles of one CTA of 512 threads, two CTAs per SM, B200):
// rank counting grows as n^2 (n = 128: 2.9K, 224: 6.5K, 256: 7.3K, 512: 24.5K), the radix select is
// flat (6.8K-7.3K up to n = 512, 9.7K at 2016), the threshold filter pays when few keys pass it
// (k <= n / 8: n = 224, k = 16: 4.7K; n = 2016, k = 32: 8.4K) and not otherwise (n = 256, k = 128:
// 18.8K).
constexpr int kRankSelectMax = 256;
__device__ __forceinline__ void block_select_topk_any(const uint32_t* keys, int n, int k, int* out, int* hist,
                                                      int* scratch, uint32_t* ckeys, int* cpos);
constexpr int kScratchInts = 32;   // warp totals (16) + broadcast slots

// Larger score -> larger key; +0 and -0 map to the same key.
__device__ __forceinline__ uint32_t order_key(float s) {
  if (s == 0.f) s = 0.f;
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive scan of one int per thread over the CTA; returns the block total in *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kRouteThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kRouteThreads / 32) warp_tot[lane] = t;   // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp == 0 ? 0 : warp_tot[warp - 1]);
  *total = warp_tot[kRouteThreads / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// Select the k largest keys[0..n) (ties: lower position first); write the selected
// positions, ascending, to out[0..k).  All threads of the CTA must call it.
__device__ void block_select_topk(const uint32_t* keys, int n, int k, int* out, int* hist,
                                  int* scratch /* kScratchInts ints */) {
  int* warp_tot = scratch;
  int* bcast = scratch + kRouteThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kRouteThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kRouteThreads) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      int c[8], s = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { c[e] = hist[255 - 8 * lane - e]; s += c[e]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, incl >= remaining);
      const int L = __ffs(ball) - 1;               // always exists: total >= remaining
      if (lane == L) {
        int cum = incl - s, digit = 0, rem = remaining;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + c[e] >= remaining) { digit = 255 - 8 * lane - e; rem = remaining - cum; break; }
          cum += c[e];
        }
        bcast[0] = digit;
        bcast[1] = rem;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)bcast[0] << shift;
    pmask |= 0xFFu << shift;
    remaining = bcast[1];
    __syncthreads();
  }
  // keys > prefix are all taken; of the keys == prefix, the first `remaining` in index order.
  const int per = (n + kRouteThreads - 1) / kRouteThreads;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int eq = 0;
  for (int i = lo; i < hi; ++i) eq += (keys[i] == prefix);
  int tot;
  int eq_before = block_exclusive_scan(eq, warp_tot, &tot);
  int cnt = 0;
  {
    int e = eq_before;
    for (int i = lo; i < hi; ++i) {
      const uint32_t key = keys[i];
      if (key > prefix) ++cnt;
      else if (key == prefix) { if (e < remaining) ++cnt; ++e; }
    }
  }
  int pos = block_exclusive_scan(cnt, warp_tot, &tot);
  {
    int e = eq_before;
    for (int i = lo; i < hi; ++i) {
      const uint32_t key = keys[i];
      bool take = false;
      if (key > prefix) take = true;
      else if (key == prefix) { take = e < remaining; ++e; }
      if (take) out[pos++] = i;
    }
  }
  __syncthreads();
}

// Select the k largest keys[0..n) for n <= kRouteThreads: thread i computes the rank of key i
// (number of keys that precede it in the order "larger first, lower position first") by comparing
// against broadcast 16-byte shared-memory reads of four keys at a time (keys[n..n4) hold 0, which
// precedes nothing and is preceded by every score), keeps it if rank < k, and an index-ordered
// scan of the kept flags writes the positions ascending.  One pass, two barriers.  A key at a lower
// position precedes key i when it is >= key i, one at a higher position when it is > key i: every
// score's key is at least 1, so the four-key groups before i's own compare against ki - 1 and the
// others against ki, and i's own group adds its earlier equal keys.
__device__ void block_select_topk_small(const uint32_t* keys, int n, int k, int* out, int* scratch,
                                        const int* pos_of = nullptr) {
  const int i = threadIdx.x;
  bool take = false;
  if (i < n) {
    const uint32_t ki = keys[i];
    const uint4* k4 = reinterpret_cast<const uint4*>(keys);
    const int n4 = (n + 3) >> 2, i4 = i >> 2;
    int rank = 0;
#pragma unroll 4
    for (int j4 = 0; j4 < n4; ++j4) {
      const uint4 v = k4[j4];
      const uint32_t thr = ki - (j4 < i4 ? 1u : 0u);
      rank += (int)(v.x > thr) + (int)(v.y > thr) + (int)(v.z > thr) + (int)(v.w > thr);
    }
    const uint4 v = k4[i4];
    const int e = i & 3;
    rank += (int)(e > 0 && v.x == ki) + (int)(e > 1 && v.y == ki) + (int)(e > 2 && v.z == ki);
    take = rank < k;
  }
  int tot;
  const int pos = block_exclusive_scan(take ? 1 : 0, scratch, &tot);
  if (take) out[pos] = pos_of ? pos_of[i] : i;
  __syncthreads();
}

// Select the k largest of keys[0..n) for k <= n, n > kRankSelectMax.  Every key >= T, T the least
// of the maxima of k disjoint position ranges, is a candidate: each range holds a key >= T, so at
// least k keys are >= T and the k largest (ties included) all are.  The candidates, compacted in
// position order into ckeys / cpos, are ranked as in block_select_topk_small when there are at most
// kRouteThreads of them (the order among them is the order among all keys); otherwise the radix
// select runs on all n keys.  Writes the selected positions ascending to out[0..k).
__device__ void block_select_topk_filtered(const uint32_t* keys, int n, int k, int* out, int* hist, int* scratch,
                                           uint32_t* ckeys, int* cpos) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned* thr = reinterpret_cast<unsigned*>(hist);
  if (tid == 0) *thr = 0xffffffffu;
  __syncthreads();
  for (int g = warp; g < k; g += kRouteThreads / 32) {
    const int lo = (int)((int64_t)g * n / k), hi = (int)((int64_t)(g + 1) * n / k);
    unsigned m = 0u;
    for (int i = lo + lane; i < hi; i += 32) m = max(m, keys[i]);
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) atomicMin(thr, m);
  }
  __syncthreads();
  const unsigned T = *thr;
  const int per = (n + kRouteThreads - 1) / kRouteThreads;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int cnt = 0;
  for (int i = lo; i < hi; ++i) cnt += keys[i] >= T;
  int tot;
  int pos = block_exclusive_scan(cnt, scratch, &tot);
  if (tot > kRouteThreads) {                  // block-uniform
    block_select_topk(keys, n, k, out, hist, scratch);
    return;
  }
  for (int i = lo; i < hi; ++i)
    if (keys[i] >= T) {
      ckeys[pos] = keys[i];
      cpos[pos] = i;
      ++pos;
    }
  if (tid < 4 && tot + tid < ((tot + 3) & ~3)) ckeys[tot + tid] = 0u;
  __syncthreads();
  block_select_topk_small(ckeys, tot, k, out, scratch, cpos);
}

__device__ __forceinline__ void block_select_topk_any(const uint32_t* keys, int n, int k, int* out, int* hist,
                                                      int* scratch, uint32_t* ckeys, int* cpos) {
  if (n <= 128)
    block_select_topk_small(keys, n, k, out, scratch);
  else if (8 * k <= n)
    block_select_topk_filtered(keys, n, k, out, hist, scratch, ckeys, cpos);
  else if (n <= kRankSelectMax)
    block_select_topk_small(keys, n, k, out, scratch);
  else
    block_select_topk(keys, n, k, out, hist, scratch);
}

// Dot products of qb (smem, 128 floats) with `count` rows of a float32 [*, 128] table,
// row ids given by row_of(i); one warp per row, 8 rows in flight per warp.
template <typename RowOf>
__device__ __forceinline__ void score_rows(const float* qb, const float* __restrict__ table, int count,
                                           RowOf row_of, uint32_t* keys_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float4 qv = *reinterpret_cast<const float4*>(qb + 4 * lane);
  constexpr int W = kRouteThreads / 32;
  constexpr int U = 8;
  for (int i0 = warp; i0 < count; i0 += U * W) {
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * W;
      s[u] = 0.f;
      if (i < count) {
        const float4 c = __ldg(reinterpret_cast<const float4*>(table + (int64_t)row_of(i) * kD) + lane);
        s[u] = qv.x * c.x + qv.y * c.y + qv.z * c.z + qv.w * c.w;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s[u] += __shfl_xor_sync(0xffffffffu, s[u], o);
      const int i = i0 + u * W;
      if (lane == 0 && i < count) keys_out[i] = order_key(s[u]);
    }
  }
}

// Routing modes and the inputs / outputs of the cached group level.
enum RouteMode { kRouteFull = 0, kRouteChunks = 1, kRouteGroupsCached = 2, kRouteQuery = 3, kRouteFromScores = 4 };
struct RouteCache {
  float* qb;                // [units][128] block queries: written in modes 1 and 3, read in modes 2 and 4
  const int32_t* slot_of;   // mode 2: [B*Hkv][nch_stride] cache slot of each chunk (-1: not cached)
  const float* gcache;      // mode 2: [B*Hkv][cap][8][128] group summaries of the cached chunks
  int cap;                  // mode 2: cache slots per (batch, KV head)
  int* status;              // mode 2: a chosen chunk missing from the cache records HGA_ERR_ARG here
  const uint32_t* scores;   // mode 4: [units][nc_pad] order keys of the chunk scores (chunk_score_kernel)
  int nc_pad;               // mode 4: row stride of `scores`
};

template <typename T, int MODE>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(
    const T* __restrict__ q, const T* __restrict__ q_prev, int causal, const float* __restrict__ group_sum,
    const float* __restrict__ chunk_sum, int32_t* __restrict__ chunk_idx, int32_t* __restrict__ group_idx, int Hq,
    int Hkv, int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, const RouteCache rc) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  if (threadIdx.x == 0) pdl_trigger();
  constexpr int N = Vec16<T>::N;
  constexpr int LPR = kD / N;
  constexpr int RP = kRouteThreads / LPR;       // rows reduced in parallel
  const int nblk = (int)(S / kQBlock);
  const int unit = blockIdx.x;                  // (b*Hkv + kh)*nblk + n
  const int n = unit % nblk;
  const int bkh = unit / nblk;
  const int kh = bkh % Hkv, b = bkh / Hkv;
  const int G = Hq / Hkv;

  float* red = reinterpret_cast<float*>(smem_raw);              // [RP][128]
  float* qb = red + RP * kD;                                      // [128]
  int* hist = reinterpret_cast<int*>(qb + kD);                    // [256]
  int* scratch = hist + 256;                                      // [kScratchInts]
  int* csel = scratch + kScratchInts;                             // [kc]
  int* gpos = csel + ((kc + 3) & ~3);                             // [kg]
  uint32_t* keys = reinterpret_cast<uint32_t*>(gpos + ((kg + 3) & ~3));   // [max(nch, 8kc) rounded to 4]
  const int nkeys4 = (((nch > 8 * kc) ? nch : 8 * kc) + 3) & ~3;
  uint32_t* ckeys = keys + nkeys4;                                        // [kRouteThreads] candidates
  int* cpos = reinterpret_cast<int*>(ckeys + kRouteThreads);              // [kRouteThreads]

  // ---- block query: mean over G heads x 64 positions of the routing block -- block n itself, or
  // for strictly causal routing block n-1 (block 0: the previous segment's last block q_prev
  // [B, Hq, 64, D], or a zero query when there is none)
  const T* qsrc = q;
  int64_t s_src = S, t_src = (int64_t)n * kQBlock;
  bool zero_query = false;
  if (causal) {
    if (n > 0) {
      t_src -= kQBlock;
    } else if (q_prev) {
      qsrc = q_prev;
      s_src = kQBlock;
      t_src = 0;
    } else {
      zero_query = true;
    }
  }
  if (MODE == kRouteGroupsCached) {
    // the block query and the chosen chunks come from the level-1 call (a kernel before)
    pdl_wait();
    if (threadIdx.x < kD) qb[threadIdx.x] = rc.qb[(int64_t)unit * kD + threadIdx.x];
    for (int i = threadIdx.x; i < kc; i += kRouteThreads) csel[i] = chunk_idx[(int64_t)unit * kc + i];
    __syncthreads();
  } else if (MODE == kRouteFromScores) {
    // the block query (mode 3) and this block's row of chunk scores (chunk_score_kernel)
    pdl_wait();
    if (threadIdx.x < kD) qb[threadIdx.x] = rc.qb[(int64_t)unit * kD + threadIdx.x];
    const uint4* src = reinterpret_cast<const uint4*>(rc.scores + (int64_t)unit * rc.nc_pad);
    for (int i = threadIdx.x; i < rc.nc_pad / 4; i += kRouteThreads) reinterpret_cast<uint4*>(keys)[i] = src[i];
    __syncthreads();
  } else {
    const int tid = threadIdx.x;
    const int col = (tid % LPR) * N, r0 = tid / LPR;
    float acc[N];
#pragma unroll
    for (int e = 0; e < N; ++e) acc[e] = 0.f;
    const int R = G * kQBlock;
    constexpr int UQ = 8;                        // 16-byte loads in flight per thread
    for (int r1 = r0; r1 < R; r1 += UQ * RP) {
      uint4 raw[UQ];                             // kept packed until accumulation (register budget)
#pragma unroll
      for (int u = 0; u < UQ; ++u) {
        const int r = r1 + u * RP;
        if (r < R && !zero_query) {
          const int h = kh * G + r / kQBlock;
          const int64_t t = t_src + r % kQBlock;
          raw[u] = *reinterpret_cast<const uint4*>(qsrc + (((int64_t)b * Hq + h) * s_src + t) * kD + col);
        } else {
          raw[u] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < UQ; ++u) {
        float v[N];
        Vec16<T>::load(reinterpret_cast<const T*>(&raw[u]), v);
#pragma unroll
        for (int e = 0; e < N; ++e) acc[e] += v[e];
      }
    }
#pragma unroll
    for (int e = 0; e < N; ++e) red[r0 * kD + col + e] = acc[e];
    __syncthreads();
    if (tid < kD) {
      float s = 0.f;
      for (int r = 0; r < RP; ++r) s += red[r * kD + tid];
      qb[tid] = s / (float)R;
    }
    __syncthreads();
    if (MODE == kRouteQuery) {
      if (tid < kD) rc.qb[(int64_t)unit * kD + tid] = qb[tid];
      pdl_wait();   // completes only after the kernel before: the launch chain keeps its order
      return;
    }
  }

  if (MODE != kRouteGroupsCached) {
    const int nc1 = nch - nsc;
    if (MODE != kRouteFromScores) {
      // the block query needs only q: the summaries are read once the kernel before has completed
      pdl_wait();

      // ---- level 1: the chunks outside the sink window (the first nsc chunks are always attended
      // and never routed); candidate i is chunk nsc + i, so lower position = lower chunk index
      const float* cs = chunk_sum + (int64_t)bkh * nch_stride * kD;   // summary buffers hold nch_stride chunks
      score_rows(qb, cs, nc1, [nsc](int i) { return nsc + i; }, keys);
      if (threadIdx.x < 4 && nc1 + (int)threadIdx.x < ((nc1 + 3) & ~3)) keys[nc1 + threadIdx.x] = 0u;
      __syncthreads();
    }
    block_select_topk_any(keys, nc1, kc, csel, hist, scratch, ckeys, cpos);
    if (nsc) {
      for (int i = threadIdx.x; i < kc; i += kRouteThreads) csel[i] += nsc;
      __syncthreads();
    }
    if (MODE == kRouteChunks) {
      for (int i = threadIdx.x; i < kc; i += kRouteThreads) chunk_idx[(int64_t)unit * kc + i] = csel[i];
      if (threadIdx.x < kD) rc.qb[(int64_t)unit * kD + threadIdx.x] = qb[threadIdx.x];
      return;
    }
  }

  // ---- level 2: the 8 groups of every selected chunk, from the summary table or from the chunk's
  // cache slot (a chunk that has none records HGA_ERR_ARG and reads slot 0)
  const int ncand = kc * (kChunk / kGroup);
  if (MODE == kRouteGroupsCached) {
    const float* gc = rc.gcache + (int64_t)bkh * rc.cap * (kChunk / kGroup) * kD;
    const int32_t* so = rc.slot_of + (int64_t)bkh * nch_stride;
    const int cap = rc.cap;
    int* st = rc.status;
    score_rows(qb, gc, ncand,
               [csel, so, cap, st](int c) {
                 int slot = __ldg(so + csel[c >> 3]);
                 if (slot < 0 || slot >= cap) {
                   set_status(st, -1);
                   slot = 0;
                 }
                 return slot * 8 + (c & 7);
               },
               keys);
  } else {
    const float* gs = group_sum + (int64_t)bkh * nch_stride * (kChunk / kGroup) * kD;
    score_rows(qb, gs, ncand, [csel](int c) { return csel[c >> 3] * 8 + (c & 7); }, keys);
  }
  if (threadIdx.x < 4 && ncand + (int)threadIdx.x < ((ncand + 3) & ~3)) keys[ncand + threadIdx.x] = 0u;
  __syncthreads();
  block_select_topk_any(keys, ncand, kg, gpos, hist, scratch, ckeys, cpos);

  for (int i = threadIdx.x; i < kc; i += kRouteThreads) chunk_idx[(int64_t)unit * kc + i] = csel[i];
  for (int i = threadIdx.x; i < kg; i += kRouteThreads)
    group_idx[(int64_t)unit * kg + i] = csel[gpos[i] >> 3] * 8 + (gpos[i] & 7);
}

size_t route_smem_bytes(bool bf16, int nch, int kc, int kg) {
  const int RP = kRouteThreads / (kD / (bf16 ? 8 : 4));
  size_t words = (size_t)RP * kD + kD + 256 + kScratchInts + ((kc + 3) & ~3) + ((kg + 3) & ~3) +
                 (size_t)(((nch > 8 * kc ? nch : 8 * kc) + 3) & ~3) + 2 * kRouteThreads;
  return words * 4;
}

template <typename T, int MODE>
static cudaError_t launch_route_t(const void* q, const void* q_prev, bool causal, const float* group_sum,
                                  const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, int B, int Hq,
                                  int Hkv, int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, size_t smem,
                                  const RouteCache& rc, cudaStream_t stream) {
  const int64_t units = (int64_t)B * Hkv * (S / kQBlock);
  if (units == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(route_kernel<T, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(route_kernel<T, MODE>, dim3((unsigned)units), dim3(kRouteThreads), smem, stream, 1,
                       static_cast<const T*>(q), static_cast<const T*>(q_prev), causal ? 1 : 0, group_sum, chunk_sum,
                       chunk_idx, group_idx, Hq, Hkv, S, nch, nch_stride, nsc, kc, kg, rc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_route(bool bf16, const void* q, const void* q_prev, bool causal, const float* group_sum,
                         const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, int B, int Hq, int Hkv,
                         int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, cudaStream_t stream) {
  const size_t smem = route_smem_bytes(bf16, nch, kc, kg);
  const RouteCache rc{nullptr, nullptr, nullptr, 0, nullptr, nullptr, 0};
  return bf16 ? launch_route_t<__nv_bfloat16, kRouteFull>(q, q_prev, causal, group_sum, chunk_sum, chunk_idx, group_idx, B, Hq, Hkv,
                                              S, nch, nch_stride, nsc, kc, kg, smem, rc, stream)
              : launch_route_t<float, kRouteFull>(q, q_prev, causal, group_sum, chunk_sum, chunk_idx, group_idx, B, Hq,
                                                  Hkv, S, nch, nch_stride, nsc, kc, kg, smem, rc, stream);
}

// Level 1 only: chunk_idx and the block queries qb [B, Hkv, S/64, 128] float32.
cudaError_t launch_route_chunks(bool bf16, const void* q, const void* q_prev, bool causal, const float* chunk_sum,
                                int32_t* chunk_idx, float* qb, int B, int Hq, int Hkv, int64_t S, int nch,
                                int nch_stride, int nsc, int kc, cudaStream_t stream) {
  const size_t smem = route_smem_bytes(bf16, nch, kc, 1);
  const RouteCache rc{qb, nullptr, nullptr, 0, nullptr, nullptr, 0};
  return bf16 ? launch_route_t<__nv_bfloat16, kRouteChunks>(q, q_prev, causal, nullptr, chunk_sum, chunk_idx, nullptr, B, Hq, Hkv, S,
                                              nch, nch_stride, nsc, kc, 1, smem, rc, stream)
              : launch_route_t<float, kRouteChunks>(q, q_prev, causal, nullptr, chunk_sum, chunk_idx, nullptr, B, Hq,
                                                    Hkv, S, nch, nch_stride, nsc, kc, 1, smem, rc, stream);
}

// Level 2 from the group-summary cache: group_idx from the block queries and chunk_idx of level 1.
cudaError_t launch_route_groups_cached(const float* qb, const int32_t* chunk_idx, const int32_t* slot_of,
                                       const float* gcache, int cap, int32_t* group_idx, int B, int Hkv, int64_t S,
                                       int nch_stride, int kc, int kg, int* status, cudaStream_t stream) {
  // the kernel's shared memory holds keys for 8 kc candidates; no chunk level runs
  const size_t smem = route_smem_bytes(false, 1, kc, kg);
  const RouteCache rc{const_cast<float*>(qb), slot_of, gcache, cap, status, nullptr, 0};
  // q is not read in this mode: any valid element type; Hq = Hkv (G = 1) keeps the unused block-query
  // arithmetic trivially in range
  return launch_route_t<float, kRouteGroupsCached>(qb, nullptr, false, nullptr, nullptr, const_cast<int32_t*>(chunk_idx), group_idx, B, Hkv,
                               Hkv, S, 1, nch_stride, 0, kc, kg, smem, rc, stream);
}

// ---- chunk scores of all block queries of a (batch, KV head), for the three-launch routing
constexpr int kScoreWarps = 16;
constexpr int kScoreRowsPerWarp = 2;   // rows a warp scores per round
constexpr int kScoreRowsPerRound = kScoreWarps * kScoreRowsPerWarp;

// Grid (B*Hkv, row slices of `rounds` x 32 rows: one wave on the GPU).  In round t, warp w of CTA
// (bkh, y) scores chunk rows nsc + i, i = y * 32 * rounds + 32 t + 2 w (+ 1), against the block queries
// qb[bkh*nblk .. + nblk) (shared memory), the next round's rows already loading: lane l holds dims
// 4l .. 4l+3 of a row and multiplies them with the same dims of 32 block queries at a time, and a
// recursive-halving exchange over the lanes leaves lane b with the full dot product of block b.
// Writes the order keys to scores[(bkh*nblk + blk) * nc_pad + i]; the pad entries [nc1, nc_pad) get
// 0, which every score precedes.
__global__ void __launch_bounds__(kScoreWarps * 32, 1) chunk_score_kernel(const float* __restrict__ qb_all,
                                                                         const float* __restrict__ chunk_sum,
                                                                         uint32_t* __restrict__ scores, int nblk,
                                                                         int nch_stride, int nsc, int nc1, int nc_pad,
                                                                         int rounds) {
  extern __shared__ __align__(16) float qs[];   // [nblk rounded up to 32][128]
  if (threadIdx.x == 0) pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t bkh = blockIdx.x;
  const int nb32 = (nblk + 31) & ~31;
  const int base = (int)blockIdx.y * kScoreRowsPerRound * rounds + kScoreRowsPerWarp * warp;
  const float* cs = chunk_sum + (bkh * nch_stride + nsc) * kD;
  auto load_rows = [&](int t, float4(&rw)[kScoreRowsPerWarp]) {
#pragma unroll
    for (int r = 0; r < kScoreRowsPerWarp; ++r) {
      const int i = base + kScoreRowsPerRound * t + r;
      rw[r] = i < nc1 ? __ldg(reinterpret_cast<const float4*>(cs + (int64_t)i * kD) + lane)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  pdl_wait();   // the block queries come from the kernel before, the summaries from the one before it
  float4 cur[kScoreRowsPerWarp], nxt[kScoreRowsPerWarp];
  load_rows(0, cur);
  {
    const float4* src = reinterpret_cast<const float4*>(qb_all + bkh * nblk * kD);
    float4* dst = reinterpret_cast<float4*>(qs);
    for (int i = threadIdx.x; i < nb32 * (kD / 4); i += blockDim.x)
      dst[i] = i < nblk * (kD / 4) ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  uint32_t* out = scores + bkh * nblk * (int64_t)nc_pad;
  for (int t = 0; t < rounds; ++t) {
    if (t + 1 < rounds) load_rows(t + 1, nxt);
    for (int g = 0; g < nb32; g += 32) {
      // each block query's 16 bytes are read once for the warp's rows
      float p[kScoreRowsPerWarp][32];
#pragma unroll
      for (int b = 0; b < 32; ++b) {
        const float4 q4 = reinterpret_cast<const float4*>(qs + (g + b) * kD)[lane];
#pragma unroll
        for (int r = 0; r < kScoreRowsPerWarp; ++r)
          p[r][b] = q4.x * cur[r].x + q4.y * cur[r].y + q4.z * cur[r].z + q4.w * cur[r].w;
      }
#pragma unroll
      for (int r = 0; r < kScoreRowsPerWarp; ++r) {
        // recursive halving: after the step with offset o, lane l keeps the o blocks whose index has
        // bit log2(o) equal to that bit of l, summed over lane pairs l, l ^ o; at the end lane b holds
        // block b's sum over all 32 lanes
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const bool upper = (lane & o) != 0;
#pragma unroll
          for (int k = 0; k < o; ++k) {
            const float send = upper ? p[r][k] : p[r][k + o];
            const float keep = upper ? p[r][k + o] : p[r][k];
            p[r][k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        const int i = base + kScoreRowsPerRound * t + r, blk = g + lane;
        if (blk < nblk) {
          if (i < nc1) out[(int64_t)blk * nc_pad + i] = order_key(p[r][0]);
          else if (i < nc_pad) out[(int64_t)blk * nc_pad + i] = 0u;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kScoreRowsPerWarp; ++r) cur[r] = nxt[r];
  }
}

// Chunks (outside the sink window) from which routing runs in three launches when the caller passes
// a workspace.  Measured on B200 (B = 1, 8 KV heads, 32 blocks, 16 / 64 routed chunks / groups, 32 /
// 128 at 2016 chunks; summaries not in L2), one launch against three: 224 chunks 22.6 against
// 25.6 us, 512 26.7 against 25.6, 1024 34.8 against 29.8, 2016 55.3 against 44.0.
constexpr int kSplitMinChunks = 512;

// chunk_score_kernel keeps all block queries of a (batch, KV head) in shared memory
constexpr size_t kScoreSmemMax = 200 * 1024;

int route_split_nc_pad(int nch, int nsc) { return ((nch - nsc) + 3) & ~3; }
bool route_uses_split(int64_t nblk, int nch, int nsc) {
  return nch - nsc >= kSplitMinChunks && (size_t)((nblk + 31) & ~31) * kD * sizeof(float) <= kScoreSmemMax;
}
// units = B * Hkv * nblk
size_t route_split_bytes(int64_t units, int64_t nblk, int nch, int nsc) {
  if (!route_uses_split(nblk, nch, nsc)) return 0;
  return (size_t)units * kD * sizeof(float) + (size_t)units * route_split_nc_pad(nch, nsc) * sizeof(uint32_t);
}

// Three-launch routing with scratch = route_split_bytes(...) bytes (16-byte aligned): block queries,
// chunk scores, selection + level 2.  Same outputs as launch_route.
cudaError_t launch_route_split(bool bf16, const void* q, const void* q_prev, bool causal, const float* group_sum,
                               const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, int B, int Hq,
                               int Hkv, int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, void* scratch,
                               cudaStream_t stream) {
  const int64_t nblk = S / kQBlock;
  const int64_t units = (int64_t)B * Hkv * nblk;
  if (units == 0) return cudaSuccess;
  const int nc1 = nch - nsc, nc_pad = route_split_nc_pad(nch, nsc);
  float* qb = static_cast<float*>(scratch);
  uint32_t* scores = reinterpret_cast<uint32_t*>(qb + units * kD);
  // 1. block queries
  RouteCache rc{qb, nullptr, nullptr, 0, nullptr, nullptr, 0};
  cudaError_t e = bf16 ? launch_route_t<__nv_bfloat16, kRouteQuery>(q, q_prev, causal, nullptr, nullptr, nullptr, nullptr, B, Hq,
                                                            Hkv, S, nch, nch_stride, nsc, kc, kg,
                                                            route_smem_bytes(true, nch, kc, kg), rc, stream)
                       : launch_route_t<float, kRouteQuery>(q, q_prev, causal, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv,
                                                            S, nch, nch_stride, nsc, kc, kg,
                                                            route_smem_bytes(false, nch, kc, kg), rc, stream);
  if (e != cudaSuccess) return e;
  // 2. chunk scores: enough rounds per CTA that the grid is one wave
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int64_t total_rounds = (int64_t)B * Hkv * ((nc_pad + kScoreRowsPerRound - 1) / kScoreRowsPerRound);
  const int rounds = (int)((total_rounds + sms - 1) / sms);
  const int rows_per_cta = kScoreRowsPerRound * rounds;
  const dim3 grid((unsigned)(B * Hkv), (unsigned)((nc_pad + rows_per_cta - 1) / rows_per_cta));
  const size_t smem2 = (size_t)((nblk + 31) & ~31) * kD * sizeof(float);
  e = cudaFuncSetAttribute(chunk_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (e != cudaSuccess) return e;
  e = launch_dependent(chunk_score_kernel, grid, dim3(kScoreWarps * 32), smem2, stream, 1,
                       static_cast<const float*>(qb), chunk_sum, scores, (int)nblk, nch_stride, nsc, nc1, nc_pad,
                       rounds);
  if (e != cudaSuccess) return e;
  // 3. selection from the scores, then level 2
  rc.scores = scores;
  rc.nc_pad = nc_pad;
  // the kernel lays its shared memory out from nch (>= nc_pad: nch = nsc + nc1, nc_pad = nc1 rounded up to 4)
  const size_t smem3 = route_smem_bytes(bf16, nch, kc, kg);
  return bf16 ? launch_route_t<__nv_bfloat16, kRouteFromScores>(q, q_prev, causal, group_sum, chunk_sum, chunk_idx, group_idx, B,
                                                        Hq, Hkv, S, nch, nch_stride, nsc, kc, kg, smem3, rc, stream)
              : launch_route_t<float, kRouteFromScores>(q, q_prev, causal, group_sum, chunk_sum, chunk_idx, group_idx, B, Hq,
                                                        Hkv, S, nch, nch_stride, nsc, kc, kg, smem3, rc, stream);
}

}  // namespace hga
