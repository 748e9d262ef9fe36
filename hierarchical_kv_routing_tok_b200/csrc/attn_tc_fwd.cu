// Routed + causal-local attention forward on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Method: "Long-Context Fine-Tuning with Limited VRAM", gist.science Technical Summary 2.1
// ("Exact-Token Attention": only the exact K/V of the selected groups are loaded) with the
// causal local window of the active segment (pith.science review, Figure 2 caption), one softmax
// over both key sets, online-softmax accumulation in the FlashAttention form the pages cite.
//
// One CTA per (batch, KV head, 64-query block, pair of query-head pairs): its query tile is
// hpc = 2 * NT query heads x 64 positions = NT M-tiles of 128 rows that share one routed key set,
// so every gathered K/V byte feeds NT MMAs.  Key tiles hold 128 keys, the causal-local tiles first
// (they need only the step's inputs, so they run while the router, the kernel before, finishes
// and while the routed groups' indices are read and their K/V gathered), then the routed ones:
//   local tiles:  128 consecutive segment rows, two 128x64 boxes ("tile layout");
//   routed tiles: 16 groups of 8 history rows, each group fetched by TMA as one 3-D box whose two
//                 64-dim halves land in its own two 1 KB swizzle atoms ("group layout").
// Warp roles: warp 0 = TMA producer, warp 1 = TMEM owner + single-thread MMA issuer,
// warps 4.. = one softmax warpgroup per M-tile (thread = TMEM lane = query row).
// TMEM: S_i (128 fp32 columns, P_i packed bf16 aliased into its first 64) and O_i (128 columns).
// Issue order S_0 S_1 | PV_0 S_0' PV_1 S_1' | ... lets softmax i work on S_i while the tensor
// core runs the other tile's MMAs; completion of S_i(j+1) implies completion of PV_i(j), so the
// softmax may rescale O_i (lazily, only when its row max grows by more than 2^8) right after it.
// Every mbarrier wait is bounded; on timeout the CTA records HGA_ERR_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace hga {
namespace tcfwd {

using namespace tc;

constexpr int BN = 128;                    // keys per tile
constexpr uint32_t kHalfBytes = BN * 128;  // one 64-dim half of a tile
constexpr uint32_t kTileBytes = 2 * kHalfBytes;
constexpr float kRescaleThreshold = 8.f;   // log2 units

struct Params {
  int B, Hq, Hkv, G, hpc, kg, nblk;
  int nsg;        // sink groups at the start of every block's history key list
  int64_t H, S;
  int64_t Hs;     // history rows per (batch, KV head) in k_hist / v_hist (>= H)
  float scale_log2;
  const int32_t* group_idx;
  __nv_bfloat16* o;
  float* lse;
  int* status;
  uint64_t wait_ns;     // limit of every bounded mbarrier wait (drains excepted)
};

constexpr int kIdxRegs = 8;                // history slots per producer lane read up front (256)
constexpr int KS = 3;                      // K stages (K runs ahead of V)
constexpr int VS = 2;                      // V stages

template <int NT>
struct Smem {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + NT * kTileBytes;
  static constexpr uint32_t kV = kK + KS * kTileBytes;
  static constexpr uint32_t kBar = kV + VS * kTileBytes;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[NT], p_full[NT], o_final,
  // mma_done
  static constexpr int kNumBars = 1 + 2 * KS + 2 * VS + 2 * NT + 2;
  static constexpr uint32_t kMisc = kBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = kMisc + 16;
};


template <int NT>
__global__ void __launch_bounds__(128 + 128 * NT, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                  const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_ks,
                  const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_o,
                  const Params p) {
  using L = Smem<NT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBar;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const uint32_t q_full = BAR(0);
  auto k_full = [&](int s) { return BAR(1 + s); };
  auto k_empty = [&](int s) { return BAR(1 + KS + s); };
  auto v_full = [&](int s) { return BAR(1 + 2 * KS + s); };
  auto v_empty = [&](int s) { return BAR(1 + 2 * KS + VS + s); };
  auto s_full = [&](int i) { return BAR(1 + 2 * KS + 2 * VS + i); };
  auto p_full = [&](int i) { return BAR(1 + 2 * KS + 2 * VS + NT + i); };
  const uint32_t o_final = BAR(1 + 2 * KS + 2 * VS + 2 * NT);
  const uint32_t mma_done = BAR(2 + 2 * KS + 2 * VS + 2 * NT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- unit decode: heavy (late) query blocks first
  const int hg = p.G / p.hpc;
  int c = blockIdx.x;
  const int hgi = c % hg;
  c /= hg;
  const int bkh = c % (p.B * p.Hkv);
  const int n = p.nblk - 1 - c / (p.B * p.Hkv);
  const int b = bkh / p.Hkv, kh = bkh % p.Hkv;
  const int h0 = kh * p.G + hgi * p.hpc;
  const int n_hist = 8 * (p.nsg + p.kg);                 // sink + routed history keys
  const int n_rt = (n_hist + BN - 1) / BN;
  const int n_lt = n / 2 + 1;
  const int T = n_rt + n_lt;
  const int32_t* gi = p.group_idx + ((int64_t)bkh * p.nblk + n) * p.kg;
  const int64_t ngr = p.H / kGroup;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int i = 0; i < NT; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), 128);
    }
    mbar_init(o_final, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), NT * 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();

  if (warp == 0 || warp == 2) {
    // ======================= TMA producers: warp 0 loads Q and the K tiles, warp 2 the V tiles,
    // each through its own ring of stages, so K can run ahead of V.
    const int kv = warp == 2;
    const int NS = kv ? VS : KS;
    if (!kv && lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kh);
      tma_prefetch_desc(&tm_ks);
      mbar_arrive_expect_tx(q_full, NT * kTileBytes);
      for (int t = 0; t < NT; ++t)
        for (int j = 0; j < 2; ++j) {
          const int64_t row = ((int64_t)b * p.Hq + h0 + 2 * t + j) * p.S + (int64_t)n * kQBlock;
          for (int h = 0; h < 2; ++h)
            tma_load_2d(sbase + L::kQ + t * kTileBytes + h * kHalfBytes + j * (kHalfBytes / 2), &tm_q, 64 * h,
                        (int32_t)row, q_full);
        }
    }
    if (kv && lane == 0) {
      tma_prefetch_desc(&tm_vh);
      tma_prefetch_desc(&tm_vs);
    }
    int32_t gidx[kIdxRegs];
    int issued[KS] = {0, 0, 0};
    for (int j = 0; j < T; ++j) {
      const int jr = j - n_lt;                            // routed tile index (>= 0: routed)
      if (jr == 0) {
        // the block's history group indices, written by the router (the kernel before): waited
        // for only here, after the local tiles, and all read in one round trip (lane l holds
        // slots l, l + 32, ...; longer lists read the rest per tile)
        pdl_wait();
#pragma unroll
        for (int i = 0; i < kIdxRegs; ++i) {
          const int slot = 32 * i + lane;
          gidx[i] = slot < 16 * n_rt ? routed_group(gi, slot, p.nsg, p.kg, ngr, p.status) : 0;
        }
      }
      const int s = j % NS;
      const uint32_t full = kv ? v_full(s) : k_full(s);
      const uint32_t empty = kv ? v_empty(s) : k_empty(s);
      const uint32_t dst = sbase + (kv ? L::kV : L::kK) + s * kTileBytes;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(empty, ((j / NS) & 1) ^ 1, abort_flag, p.status, p.wait_ns);
        if (ok) mbar_arrive_expect_tx(full, kTileBytes);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (jr >= 0) {
        // 16 routed groups, one per lane, each group's 8 rows one 3-D box (its two 64-column halves
        // land 1 KB apart)
        int32_t g;
        if (jr < 2 * kIdxRegs) {
          int32_t sel = 0;
#pragma unroll
          for (int i = 0; i < kIdxRegs; ++i)
            if (i == (jr >> 1)) sel = gidx[i];
          g = __shfl_sync(0xffffffffu, sel, (16 * jr + lane) & 31);
        } else {
          g = lane < 16 ? routed_group(gi, jr * 16 + lane, p.nsg, p.kg, ngr, p.status) : 0;
        }
        if (g < 0) g = 0;
        if (lane < 16)
          tma_load_3d(dst + lane * 2048, kv ? &tm_vh : &tm_kh, 0, (int32_t)((int64_t)bkh * p.Hs + (int64_t)g * kGroup),
                      0, full);
      } else if (lane == 0) {
        const int jl = j;
        const int32_t row = (int32_t)((int64_t)bkh * p.S + (int64_t)jl * BN);
        const CUtensorMap* m = kv ? &tm_vs : &tm_ks;
        tma_load_2d(dst, m, 0, row, full);
        tma_load_2d(dst + kHalfBytes, m, 64, row, full);
      }
      __syncwarp();
      ++issued[s];
    }
    // every load this warp issued has landed before the CTA may exit (the Q tile included: a CTA
    // that gave up early may not have waited for it)
    if (lane == 0) {
      for (int s = 0; s < NS; ++s)
        if (issued[s]) drain_wait(kv ? v_full(s) : k_full(s), (issued[s] - 1) & 1, p.status);
      if (!kv) drain_wait(q_full, 0, p.status);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer: the whole warp runs the loop (warp-uniform descriptors
    // and waits) and one elected lane issues each tcgen05 instruction.  All shared-memory
    // descriptors are built before each unrolled MMA sequence, so the sequence issues back to back.
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kD, true);
      uint64_t qd[NT][8], kd[8], vd[8];
#pragma unroll
      for (int i = 0; i < NT; ++i) kmajor_descs(qd[i], sbase + L::kQ + i * kTileBytes, kHalfBytes, 1024);
      auto build_k = [&](int j) {
        const bool routed = j >= n_lt;
        kmajor_descs(kd, sbase + L::kK + (j % KS) * kTileBytes, routed ? 1024u : kHalfBytes, routed ? 2048u : 1024u);
      };
      auto build_v = [&](int j) {
        const bool routed = j >= n_lt;
        mnmajor_descs<8>(vd, sbase + L::kV + (j % VS) * kTileBytes, routed ? 1024u : kHalfBytes,
                         routed ? 2048u : 1024u);
      };
      bool ok = mbar_wait_w(q_full, 0, abort_flag, p.status, p.wait_ns) && mbar_wait_w(k_full(0), 0, abort_flag, p.status, p.wait_ns);
      if (ok) {
        tc_fence_after();
        build_k(0);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + i * 128, qd[i][ks], kd[ks], idesc_qk, ks > 0);
          mma_commit_w(s_full(i));
        }
        mma_commit_w(k_empty(0));
      }
      for (int j = 0; ok && j < T; ++j) {
        ok = mbar_wait_w(v_full(j % VS), (j / VS) & 1, abort_flag, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        build_v(j);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          ok = mbar_wait_w(p_full(i), j & 1, abort_flag, p.status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts_w(tmem + NT * 128 + i * 128, tmem + i * 128 + ks * 8, vd[ks], idesc_pv, (j > 0 || ks > 0));
          if (j + 1 < T) {
            // the next K tile is only needed now, after this tile's first PV is queued
            if (i == 0) {
              ok = mbar_wait_w(k_full((j + 1) % KS), ((j + 1) / KS) & 1, abort_flag, p.status, p.wait_ns);
              if (!ok) break;
              tc_fence_after();
              build_k(j + 1);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + i * 128, qd[i][ks], kd[ks], idesc_qk, ks > 0);
            mma_commit_w(s_full(i));
          }
        }
        if (!ok) break;
        mma_commit_w(v_empty(j % VS));
        if (j + 1 < T) mma_commit_w(k_empty((j + 1) % KS));
      }
      if (ok) mma_commit_w(o_final);
      mma_commit_w(mma_done);
      drain_wait(mma_done, 0, p.status);
    }
  } else if (warp >= 4) {
    // ======================= softmax / epilogue, one warpgroup per M-tile
    const int i = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // row of the M-tile = TMEM lane
    const int head = h0 + 2 * i + (r >> 6);
    const int64_t t_pos = (int64_t)n * kQBlock + (r & 63);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + i * 128;
    const uint32_t tO = tmem + lane_off + NT * 128 + i * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      ok = mbar_wait(s_full(i), j & 1, abort_flag, p.status, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool routed = j >= n_lt;
      int nvalid;
      if (routed) {
        nvalid = min(BN, n_hist - (j - n_lt) * BN);
      } else {
        const int64_t u0 = (int64_t)j * BN;
        nvalid = (int)max((int64_t)0, min((int64_t)BN, t_pos - u0 + 1));
      }
      // The whole 128-column row is loaded with one TMEM round trip and kept in registers.
      uint32_t v[128];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
      tmem_wait_ld();
      if (nvalid < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e >= nvalid) v[e] = __float_as_uint(-INFINITY);
      }
      // row max of the raw logits (the scale is positive)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; e += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(v[e]));
        mx1 = fmaxf(mx1, __uint_as_float(v[e + 1]));
      }
      const float mx = fmaxf(mx0, mx1) * p.scale_log2;
      // lazy rescale: move the reference max only when it grows by more than 2^8
      const bool need = mx > m + kRescaleThreshold || (m == -INFINITY && mx > -INFINITY);
      const float mnew = need ? mx : m;
      const float alpha = need ? ex2(m - mnew) : 1.f;   // m = -inf -> 0
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
      }
      l *= alpha;
      m = mnew;
      const float mref = (m == -INFINITY) ? 0.f : m;
      // probabilities (masked logits are -inf -> 0), row sum, bf16 P into the first 64 columns of S
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(v[cc * 32 + e]), p.scale_log2, -mref));
          const float p1 = ex2(fmaf(__uint_as_float(v[cc * 32 + e + 1]), p.scale_log2, -mref));
          rs0 += p0;
          rs1 += p1;
          pk[e >> 1] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + cc * 16, pk);
      }
      const float rs = rs0 + rs1;
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(i));
    }
    if (ok) {
      ok = mbar_wait(o_final, 0, abort_flag, p.status, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // O / l as bf16 into this M-tile's (now unused) Q area, in the layout its Q tile was loaded
      // in (two 64-dim halves, 128-byte swizzle), then each warp stores its 32 rows with TMA (one
      // 32-row box per half): full 128-byte lines instead of one 16-byte piece per row per store
      // instruction.  After o_final every MMA has completed, so nothing reads Q any more.
      tc_fence_after();
      const float inv = 1.f / l;
      const uint32_t qt = sbase + L::kQ + i * kTileBytes + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tO + cc * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pk[e >> 1] = pack_bf16(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv);
        // columns 32 cc .. 32 cc + 31: half cc / 2, 16-byte chunks 4 (cc % 2) .. + 3 of the row
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t chunk = (uint32_t)(4 * (cc & 1) + q4);
          const uint32_t a = qt + (uint32_t)(cc >> 1) * kHalfBytes + ((chunk ^ (uint32_t)(r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * q4]), "r"(pk[4 * q4 + 1]),
                       "r"(pk[4 * q4 + 2]), "r"(pk[4 * q4 + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // rows 32 quarter .. + 31 of the M-tile: head 2 i + quarter / 2, positions 32 (quarter % 2) ..
        const int64_t orow =
            ((int64_t)b * p.Hq + h0 + 2 * i + (quarter >> 1)) * p.S + (int64_t)n * kQBlock + 32 * (quarter & 1);
        for (int h = 0; h < 2; ++h)
          tma_store_2d(&tm_o, 64 * h, (int32_t)orow, sbase + L::kQ + i * kTileBytes + h * kHalfBytes + quarter * 4096);
        bulk_commit_group();
        bulk_wait_read_all();   // the shared-memory source must be read before the CTA exits
      }
      __syncwarp();
      p.lse[((int64_t)b * p.Hq + head) * p.S + t_pos] = (m + __log2f(l)) * 0.6931471805599453f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NT * 256);
  }
  // a CTA that gave up before reading the router's output still completes only after the kernel
  // before it, so the launch chain keeps its order
  pdl_wait();
}

}  // namespace tcfwd

// ------------------------------------------------------------------ host side
bool make_map_bf16_groups(CUtensorMap* m, const void* base, uint64_t rows);
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;   // resolved once; the driver symbol never changes
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D bf16 map over a [rows, 128] row-major tensor, boxes of {64 dims, box_rows rows}, 128B swizzle.
bool make_map_bf16_rows(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map over a [rows, 128] row-major tensor seen as {64 dims, rows, 2 halves} (the halves 128
// bytes apart in global memory): a box {64, 8, 2} is one 8-row group, landing in shared memory as
// two 1 KB 128B-swizzled atoms, first the dims 0-63 of its 8 rows, then the dims 64-127.
bool make_map_bf16_groups(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, 2};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)kGroup, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attn_fwd_tc_supported(int Hq, int Hkv) {
  const int G = Hq / Hkv;
  return G % 2 == 0;
}

cudaError_t launch_attn_fwd_tc(const void* q, const void* kh, const void* vh, const void* ks, const void* vs,
                               const int32_t* gi, void* o, float* lse, int B, int Hq, int Hkv, int64_t H, int64_t S,
                               int64_t Hs, int kg, int nsg, float scale, int* status, uint64_t wait_ns,
                               cudaStream_t st) {
  CUtensorMap mq, mkh, mvh, mks, mvs;
  // with no history the history maps are never used: map the segment instead (maps need rows > 0)
  const void* kh_m = Hs ? kh : ks;
  const void* vh_m = Hs ? vh : vs;
  const uint64_t hrows = (uint64_t)B * Hkv * (Hs ? Hs : S);
  CUtensorMap mo;   // O stores: one 32-row box per warp and 64-dim half
  if (!make_map_bf16_rows(&mq, q, (uint64_t)B * Hq * S, 64) || !make_map_bf16_rows(&mo, o, (uint64_t)B * Hq * S, 32) ||
      !make_map_bf16_groups(&mkh, kh_m, hrows) ||
      !make_map_bf16_groups(&mvh, vh_m, hrows) ||
      !make_map_bf16_rows(&mks, ks, (uint64_t)B * Hkv * S, tcfwd::BN) ||
      !make_map_bf16_rows(&mvs, vs, (uint64_t)B * Hkv * S, tcfwd::BN))
    return cudaErrorInvalidValue;
  const int G = Hq / Hkv;
  tcfwd::Params p{B, Hq, Hkv, G, (G % 4 == 0) ? 4 : 2, kg, (int)(S / kQBlock), nsg, H, S, Hs,
                  scale * 1.4426950408889634f, gi, static_cast<__nv_bfloat16*>(o), lse, status, wait_ns};
  const int64_t grid = (int64_t)B * Hkv * p.nblk * (G / p.hpc);
  cudaError_t e;
  if (p.hpc == 4) {
    const size_t smem = tcfwd::Smem<2>::kBytes + 1024;
    e = cudaFuncSetAttribute(tcfwd::fwd_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_dependent(tcfwd::fwd_tc_kernel<2>, dim3((unsigned)grid), dim3(384), smem, st, 1, mq, mkh, mvh, mks, mvs,
                         mo, p);
    if (e != cudaSuccess) return e;
  } else {
    const size_t smem = tcfwd::Smem<1>::kBytes + 1024;
    e = cudaFuncSetAttribute(tcfwd::fwd_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_dependent(tcfwd::fwd_tc_kernel<1>, dim3((unsigned)grid), dim3(256), smem, st, 1, mq, mkh, mvh, mks, mvs,
                         mo, p);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace hga
