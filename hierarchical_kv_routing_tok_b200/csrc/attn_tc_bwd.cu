// Routed + causal-local attention backward on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Method: "Long-Context Fine-Tuning with Limited VRAM", gist.science Technical Summary 2.1
// (routing carries no gradient; the gather and the exact-token attention are differentiable) and
// 2.2 (history K/V detached at the segment boundary, so only q and the active segment's K/V
// receive gradients), with the softmax backward in the FlashAttention form the pages cite:
// P = exp(S - lse), dP = dO V^T, dS = P o (dP - delta), dQ = scale dS K, dK = scale dS^T Q,
// dV = P^T dO.
//
// dq_tc_kernel: one CTA per (batch, KV head, query block, pair of query heads) = one M=128 query
//   tile.  Key tiles of 128 keys (routed: 16 groups of 8 history rows; local: 128 segment rows), so
//   that every MMA has N = 128.  TMEM: S double-buffered, dP, dQ (4 x 128 columns).  The
//   element-wise warps load S(j) and dP(j) once, release dP for dP(j+1), and pack bf16 dS(j) into
//   S(j)'s columns, from which dQ += dS K reads it.
// dkdv_tc_kernel: one CTA (or a cluster of two) per (batch, KV head, 128-key tile); keys are the
//   M dimension: S^T = K Q^T and dP^T = V dO^T (64 queries per step, double-buffered in TMEM),
//   then dV += P^T dO and dK += dS^T Q with P^T / dS^T read from TMEM.  The G query heads of the
//   KV head accumulate into the same TMEM dK / dV, one head after another; in a cluster of two each
//   CTA takes G/2 heads and each hands the float32 sums of the rows the other writes over through
//   an L2-resident exchange area of the workspace, so the result is reproducible.
// Warp roles as in the forward: warp 0 TMA, warp 1 TMEM owner + single-thread MMA issuer,
// warps 4..19 four element-wise warpgroups (thread = TMEM lane = row; the warpgroups split a
// tile's columns so that each thread handles 32 elements per step).  All mbarrier waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace hga {

bool make_map_bf16_rows(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows);
bool make_map_bf16_groups(CUtensorMap* m, const void* base, uint64_t rows);

namespace tcbwd {

using namespace tc;

constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kQTile = 128 * 256;      // 128 rows x 128 dims bf16
constexpr uint32_t kQHalf = 128 * 128;

// ======================================================================================== dQ
namespace dq {

constexpr int BN = 128;                     // keys per tile (the N of S = Q K^T and dP = dO V^T)
constexpr uint32_t kKVTile = BN * 256;      // 32 KB
constexpr uint32_t kKVHalf = BN * 128;      // 16 KB (local layout)
constexpr int KS = 3;                       // K stages (a K tile lives until its dQ MMAs are done)
constexpr int VS = 2;                       // V stages (a V tile lives until its dP MMAs are done)
constexpr int kEWWarps = 16;                // four element-wise warpgroups
constexpr int kIdxRegs = 8;                 // history slots per producer lane read ahead (256 a unit)

struct Params {
  int B, Hq, Hkv, G, kg, nblk;
  int nsg;        // sink groups at the start of every block's history key list
  int64_t H, S;
  int64_t Hs;     // history rows per (batch, KV head) in k_hist / v_hist (>= H)
  float c2;       // scale * log2(e)
  float scale;
  const int32_t* group_idx;
  const float* lse;
  const __nv_bfloat16* o;   // forward output: delta = rowsum(dO o O) is formed here
  float* delta;             // delta of this kernel's rows, written for the dK/dV kernel
  __nv_bfloat16* dq;
  int* status;
  uint64_t wait_ns;     // limit of every bounded mbarrier wait (drains excepted)
};

struct Smem {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kQ + kQTile;
  static constexpr uint32_t kK = kDO + kQTile;
  static constexpr uint32_t kV = kK + KS * kKVTile;
  static constexpr uint32_t kBar = kV + VS * kKVTile;
  // qdo_full, kv_full[KS], k_empty[KS], v_empty[VS], s_full[2], dp_full, dp_free, ds_full[2],
  // dq_ready, mma_done, qdo_empty, delta_bar, qdo_issued
  static constexpr int kNumBars = 1 + 2 * KS + VS + 12;
  static constexpr uint32_t kMisc = kBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = kMisc + 16;
};
static_assert(Smem::kBytes + 1024 <= 227 * 1024, "dq shared memory exceeds the per-CTA limit");

// Work unit u (heavy first): (batch, KV head, query block, pair of query heads), unit 0 being the
// last query block.  A persistent CTA c of G takes the units c, 2G-1-c, 2G+c, 4G-1-c, ... (a snake
// over the list, which spreads the long units evenly).
struct Unit {
  int b, bkh, n, h0, T;
};
__device__ __forceinline__ int unit_of_cta(int k, int c, int G) {
  const int round = k >> 1;
  return (k & 1) ? (2 * round + 2) * G - 1 - c : 2 * round * G + c;
}
__device__ __forceinline__ Unit decode_unit(int u, const Params& p, int n_rt) {
  const int hp = p.G / 2;
  Unit x;
  const int hpi = u % hp;
  u /= hp;
  x.bkh = u % (p.B * p.Hkv);
  x.n = p.nblk - 1 - u / (p.B * p.Hkv);
  x.b = x.bkh / p.Hkv;
  x.h0 = (x.bkh % p.Hkv) * p.G + 2 * hpi;
  x.T = n_rt + ((x.n + 1) * kQBlock + BN - 1) / BN;              // history tiles + causal-prefix tiles
  return x;
}

// Persistent: one CTA per SM walks its units; per unit a single M=128 tile whose rows 0-63 are the
// block's queries of head h0 and rows 64-127 those of head h0+1, over key tiles of 128 (the sink
// and routed groups of the block, 16 groups per tile, then the causal segment prefix).
// TMEM: S in two buffers (columns 0 and 128), dP (256), dQ (384).  Per tile j the MMA warp issues
// dP(j+1) and S(j+1) as soon as the element-wise warps have loaded S(j), dP(j) into registers, and
// dQ(j) += dS(j) K(j) when they have written dS(j) (bf16, packed into S(j)'s columns).  A running
// tile count J carries the K/V ring and the per-tile barrier phases across units; the next unit's
// Q/dO are loaded (warp 2) as soon as the last S, dP MMAs of the current unit have read them.
__global__ void __launch_bounds__(128 + 32 * kEWWarps, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_vh,
                 const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                 const Params p) {
  using L = Smem;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBar;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const uint32_t qdo_full = BAR(0);
  auto kv_full = [&](int s) { return BAR(1 + s); };          // K(J) and V(J) of tile J, slot J mod KS
  auto k_empty = [&](int s) { return BAR(1 + KS + s); };
  auto v_empty = [&](int s) { return BAR(1 + 2 * KS + s); };
  // S, dS of tile J live in S buffer J mod 2: their barriers are per buffer (phase J / 2), so that
  // S(J+1), issued before the element-wise warps are done with tile J, never runs a phase ahead
  auto s_full = [&](int b) { return BAR(1 + 2 * KS + VS + b); };
  const uint32_t dp_full = BAR(3 + 2 * KS + VS);
  const uint32_t dp_free = BAR(4 + 2 * KS + VS);
  auto ds_full = [&](int b) { return BAR(5 + 2 * KS + VS + b); };
  const uint32_t dq_ready = BAR(7 + 2 * KS + VS);
  const uint32_t mma_done = BAR(8 + 2 * KS + VS);
  const uint32_t qdo_empty = BAR(9 + 2 * KS + VS);          // the unit's Q/dO fully read
  const uint32_t delta_bar = BAR(10 + 2 * KS + VS);         // delta partial sums in TMEM
  const uint32_t qdo_issued = BAR(11 + 2 * KS + VS);        // a unit's Q/dO loads are issued
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_hist = 8 * (p.nsg + p.kg);                         // sink + routed history keys
  const int n_rt = (n_hist + BN - 1) / BN;                        // history tiles
  const int n_units = p.B * p.Hkv * p.nblk * (p.G / 2);
  const int G = gridDim.x, cta = blockIdx.x;
  const int64_t ngr = p.H / kGroup;

  if (threadIdx.x == 0) {
    mbar_init(qdo_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(kv_full(s), 2);             // the K and the V producer
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < VS; ++s) mbar_init(v_empty(s), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(ds_full(b), kEWWarps);
    }
    mbar_init(dp_full, 1);
    mbar_init(dp_free, kEWWarps);
    mbar_init(dq_ready, 1);
    mbar_init(mma_done, 1);
    mbar_init(qdo_empty, 1 + kEWWarps);     // the MMA warp's commit + every element-wise warp
    mbar_init(delta_bar, kEWWarps);
    mbar_init(qdo_issued, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();

  if (warp == 0 || warp == 3) {
    // ======================= TMA producers of K(J) (warp 0) and V(J) (warp 3), each into its own
    // ring, across all units; both arrive on kv_full of the tile.  A routed history group (8 rows)
    // is one 3-D box: its two 64-column halves land 1 KB apart in the group layout.  A unit's
    // group indices are read one unit ahead, all in one round trip (lane l holds slots l, l + 32,
    // ...), so the index reads never stand between a free slot and its loads.  A unit's first
    // tiles are issued only after its Q/dO loads: those are needed first, and otherwise wait in the
    // TMA queue behind the dozens of group boxes the rings run ahead.
    const bool is_v = warp == 3;
    const CUtensorMap* hist_map = is_v ? &tm_vh : &tm_kh;
    const CUtensorMap* seg_map = is_v ? &tm_vs : &tm_ks;
    int issued[KS] = {0, 0, 0};
    int J = 0;
    bool ok = true;
    int32_t cur[kIdxRegs], nxt[kIdxRegs];
    auto read_idx = [&](int k, int32_t(&r)[kIdxRegs]) {
      const int u = unit_of_cta(k, cta, G);
      if (u >= n_units) return;
      const Unit x = decode_unit(u, p, n_rt);
      const int32_t* gi = p.group_idx + ((int64_t)x.bkh * p.nblk + x.n) * p.kg;
#pragma unroll
      for (int i = 0; i < kIdxRegs; ++i) {
        const int slot = 32 * i + lane;
        r[i] = slot < 16 * n_rt ? routed_group(gi, slot, p.nsg, p.kg, ngr, p.status) : 0;
      }
    };
    pdl_wait();                 // the group indices come from the router (completed before the kernel before)
    read_idx(0, nxt);
    for (int k = 0; ok; ++k) {
      const int u = unit_of_cta(k, cta, G);
      if (u >= n_units) break;
      const Unit x = decode_unit(u, p, n_rt);
      const int32_t* gi = p.group_idx + ((int64_t)x.bkh * p.nblk + x.n) * p.kg;
#pragma unroll
      for (int i = 0; i < kIdxRegs; ++i) cur[i] = nxt[i];
      read_idx(k + 1, nxt);
      if (k > 0) {
        int okq = 1;
        if (lane == 0) okq = mbar_wait(qdo_issued, k & 1, abort_flag, p.status, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, okq, 0) != 0;
        if (!ok) break;
      }
      for (int j = 0; j < x.T; ++j, ++J) {
        const int ks = J % KS, vs = J % VS;
        int okk = 1;
        if (lane == 0) {
          okk = is_v ? mbar_wait(v_empty(vs), ((J / VS) & 1) ^ 1, abort_flag, p.status, p.wait_ns)
                     : mbar_wait(k_empty(ks), ((J / KS) & 1) ^ 1, abort_flag, p.status, p.wait_ns);
          if (okk) mbar_arrive_expect_tx(kv_full(ks), kKVTile);
        }
        ok = __shfl_sync(0xffffffffu, okk, 0) != 0;
        if (!ok) break;
        const uint32_t dst = is_v ? sbase + L::kV + vs * kKVTile : sbase + L::kK + ks * kKVTile;
        if (j < n_rt) {
          // 16 routed groups, one per lane
          int32_t g;
          if (j < 2 * kIdxRegs) {
            int32_t sel = 0;
#pragma unroll
            for (int i = 0; i < kIdxRegs; ++i)
              if (i == (j >> 1)) sel = cur[i];
            g = __shfl_sync(0xffffffffu, sel, (16 * j + lane) & 31);
          } else {
            g = lane < 16 ? routed_group(gi, j * 16 + lane, p.nsg, p.kg, ngr, p.status) : 0;
          }
          if (g < 0) g = 0;
          if (lane < 16)
            tma_load_3d(dst + lane * 2048, hist_map, 0, (int32_t)((int64_t)x.bkh * p.Hs + (int64_t)g * kGroup), 0,
                        kv_full(ks));
        } else if (lane == 0) {
          const int32_t row = (int32_t)((int64_t)x.bkh * p.S + (int64_t)(j - n_rt) * BN);
          tma_load_2d(dst, seg_map, 0, row, kv_full(ks));
          tma_load_2d(dst + kKVHalf, seg_map, 64, row, kv_full(ks));
        }
        __syncwarp();
        ++issued[ks];
      }
    }
    // every load this warp issued has landed (its tile's barrier completed) before the CTA exits
    if (lane == 0)
      for (int s = 0; s < KS; ++s)
        if (issued[s]) drain_wait(kv_full(s), (issued[s] - 1) & 1, p.status);
    __syncwarp();
  } else if (warp == 2) {
    // ======================= TMA producer of each unit's Q and dO (once the previous unit's
    // last S, dP MMAs and delta reads are done with them)
    int loads = 0;
    if (lane == 0) {
      for (int k = 0;; ++k) {
        const int u = unit_of_cta(k, cta, G);
        if (u >= n_units) break;
        if (k > 0 && !mbar_wait(qdo_empty, (k - 1) & 1, abort_flag, p.status, p.wait_ns)) break;
        const Unit x = decode_unit(u, p, n_rt);
        mbar_arrive_expect_tx(qdo_full, 2 * kQTile);
        for (int jh = 0; jh < 2; ++jh) {
          const int64_t row = ((int64_t)x.b * p.Hq + x.h0 + jh) * p.S + (int64_t)x.n * kQBlock;
          for (int h = 0; h < 2; ++h) {
            const uint32_t off = h * kQHalf + jh * (kQHalf / 2);
            tma_load_2d(sbase + L::kQ + off, &tm_q, 64 * h, (int32_t)row, qdo_full);
            tma_load_2d(sbase + L::kDO + off, &tm_do, 64 * h, (int32_t)row, qdo_full);
          }
        }
        mbar_arrive(qdo_issued);
        ++loads;
      }
      if (loads) drain_wait(qdo_full, (loads - 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer: the whole warp runs the loop (warp-uniform descriptors
    // and waits) and one elected lane issues each tcgen05 instruction.  Q and dO sit at fixed
    // addresses, so their descriptor arrays are built once; K / V stage descriptors come from
    // prebuilt bases.  Global tile J: K stage J mod KS, V stage J mod VS, S buffer J mod 2.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, BN, false);
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, kD, true);
    uint64_t qa[8], da[8];
    kmajor_descs(qa, sbase + L::kQ, kQHalf, 1024);
    kmajor_descs(da, sbase + L::kDO, kQHalf, 1024);
    // routed tiles: group g at g * 2048 bytes, 64-column halves 1024 apart; local tiles: halves
    // kKVHalf apart, 8-row groups 1024 apart.  Stage st is st * kKVTile bytes after stage 0.
    const uint64_t k_rt = smem_desc_sw128(sbase + L::kK, 16, 2048), k_lc = smem_desc_sw128(sbase + L::kK, 16, 1024);
    const uint64_t v_rt = smem_desc_sw128(sbase + L::kV, 16, 2048), v_lc = smem_desc_sw128(sbase + L::kV, 16, 1024);
    const uint64_t kmn_rt = smem_desc_sw128(sbase + L::kK, 1024, 2048);
    const uint64_t kmn_lc = smem_desc_sw128(sbase + L::kK, kKVHalf, 1024);
    // S(J) = Q K(J)^T into S buffer J mod 2; dP(J) = dO V(J)^T; `rt`: a routed-history tile
    auto issue_s = [&](int J, bool rt) {
      tc_fence_after();
      const uint64_t soff = (uint64_t)((J % KS) * (kKVTile >> 4));
      uint64_t bb[8];
      kmajor_from_base(bb, (rt ? k_rt : k_lc) + soff, rt ? (1024u >> 4) : (kKVHalf >> 4));
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + (J & 1) * 128, qa[ks], bb[ks], idesc_s, ks > 0);
      mma_commit_w(s_full(J & 1));
    };
    auto issue_dp = [&](int J, bool rt) {
      tc_fence_after();
      const uint64_t soff = (uint64_t)((J % VS) * (kKVTile >> 4));
      uint64_t bb[8];
      kmajor_from_base(bb, (rt ? v_rt : v_lc) + soff, rt ? (1024u >> 4) : (kKVHalf >> 4));
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + 256, da[ks], bb[ks], idesc_s, ks > 0);
      mma_commit_w(dp_full);
      mma_commit_w(v_empty(J % VS));
    };
    // dQ (+)= dS(J) K(J); dS of keys 32w..32w+31 sits in columns 32w..32w+15 of S buffer J mod 2
    auto issue_dq = [&](int J, bool rt, bool first) {
      const uint64_t soff = (uint64_t)((J % KS) * (kKVTile >> 4));
      uint64_t bb[8];
      mnmajor_from_base<8>(bb, (rt ? kmn_rt : kmn_lc) + soff, rt ? (2 * 2048u) >> 4 : (2 * 1024u) >> 4);
      const uint32_t sb = tmem + (J & 1) * 128;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ts_w(tmem + 384, sb + (ks >> 1) * 32 + (ks & 1) * 8, bb[ks], idesc_dq, !(first && ks == 0));
    };
    // Per tile J: S(J+1) as soon as its K tile has landed (the other S buffer, whose dS(J-1) the
    // last dQ MMA has read); dP(J+1) once the element-wise warps hold dP(J); dQ += dS(J) K(J) once
    // they have written dS(J).  The next tile may be the next unit's first, once its Q/dO have
    // landed: at a unit's last tile dQ += dS K is issued first and dQ released, so that the
    // element-wise warps' dQ epilogue and the next unit's delta do not wait for the next unit's
    // loads.  The unit's Q/dO are released after its last dP MMAs (issued after its last S MMAs).
    bool ok = true;
    int J = 0;
    Unit x{};
    int u = unit_of_cta(0, cta, G);
    if (u < n_units) {
      x = decode_unit(u, p, n_rt);
      ok = mbar_wait_w(qdo_full, 0, abort_flag, p.status, p.wait_ns) && mbar_wait_w(kv_full(0), 0, abort_flag, p.status, p.wait_ns);
      if (ok) {
        issue_s(0, 0 < n_rt);
        issue_dp(0, 0 < n_rt);
        if (x.T == 1) mma_commit_w(qdo_empty);
      }
    }
    for (int k = 0; ok && u < n_units; ++k) {
      const int un = unit_of_cta(k + 1, cta, G);
      const bool has_next = un < n_units;
      const Unit xn = has_next ? decode_unit(un, p, n_rt) : x;
      for (int j = 0; j < x.T; ++j, ++J) {
        const bool last = j + 1 == x.T;
        const bool next = !last || has_next;
        const int jn = last ? 0 : j + 1;          // the next tile's index in its unit
        const int Tn = last ? xn.T : x.T;
        auto finish_tile = [&]() {                // dQ (+)= dS(J) K(J), then K(J) is free
          ok = mbar_wait_w(ds_full(J & 1), (J >> 1) & 1, abort_flag, p.status, p.wait_ns);
          if (!ok) return;
          tc_fence_after();
          issue_dq(J, j < n_rt, j == 0);
          mma_commit_w(k_empty(J % KS));
        };
        if (last) {                               // the unit's dQ is complete after these MMAs
          finish_tile();
          if (!ok) break;
          mma_commit_w(dq_ready);
        }
        if (next) {
          if (last) ok = mbar_wait_w(qdo_full, (k + 1) & 1, abort_flag, p.status, p.wait_ns);
          if (ok) ok = mbar_wait_w(kv_full((J + 1) % KS), ((J + 1) / KS) & 1, abort_flag, p.status, p.wait_ns);
          if (!ok) break;
          issue_s(J + 1, jn < n_rt);
        }
        ok = mbar_wait_w(dp_free, J & 1, abort_flag, p.status, p.wait_ns);
        if (!ok) break;
        if (next) {
          issue_dp(J + 1, jn < n_rt);
          if (jn + 1 == Tn) mma_commit_w(qdo_empty);
        }
        if (!last) {
          finish_tile();
          if (!ok) break;
        }
      }
      if (!ok) break;
      u = un;
      x = xn;
    }
    mma_commit_w(mma_done);
    drain_wait(mma_done, 0, p.status);
  } else if (warp >= 4) {
    // ======================= element-wise: dS = P o (dP - delta), P = exp2(S c2 - lse log2 e).
    // Thread = TMEM lane = row of the M tile; warpgroup w owns key columns 32w .. 32w+31.
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int c0 = 32 * w;
    const bool dq_v8 = (reinterpret_cast<uintptr_t>(p.dq) & 31u) == 0;
    pdl_wait();                 // O and lse come from the forward kernel, the kernel before
    bool ok = true;
    int J = 0;
    for (int k = 0; ok; ++k) {
      const int u = unit_of_cta(k, cta, G);
      if (u >= n_units) break;
      const Unit x = decode_unit(u, p, n_rt);
      const int head = x.h0 + (r >> 6);
      const int64_t t_pos = (int64_t)x.n * kQBlock + (r & 63);
      const int64_t row = ((int64_t)x.b * p.Hq + head) * p.S + t_pos;
      const float lse2 = p.lse[row] * kLog2e;
      // delta = sum_d dO o O of this row (FlashAttention-form backward).  Warpgroup w takes columns
      // 32w .. 32w+31: O from global memory (loads issued before the wait for the Q/dO tile), dO
      // from the 128B-swizzled tile loaded for dP (row r: 8-row atom r/8, 16-byte chunk c of a
      // 64-column half at position c ^ (r mod 8)).  The four partial sums meet in TMEM column
      // 384 + 32w (the first column of this warpgroup's dQ, already read out for the previous
      // unit and not rewritten before this unit's first dS K MMA) and every thread adds them in
      // order; the first warpgroup stores delta for the dK/dV kernel.
      uint4 ov[4];
      {
        const uint4* orow = reinterpret_cast<const uint4*>(p.o + row * kD + c0);
#pragma unroll
        for (int c = 0; c < 4; ++c) ov[c] = orow[c];
      }
      ok = __all_sync(0xffffffffu, mbar_wait(qdo_full, k & 1, abort_flag, p.status, p.wait_ns));
      if (!ok) break;
      float part;
      {
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * w + c;                       // 16-byte chunk of the 128-column row
          const uint32_t off = (uint32_t)(chunk >> 3) * kQHalf + (uint32_t)(r >> 3) * 1024u +
                               (uint32_t)(r & 7) * 128u + ((uint32_t)((chunk & 7) ^ (r & 7)) << 4);
          const uint4 dv4 = *reinterpret_cast<const uint4*>(smem + L::kDO + off);
          const uint32_t a[4] = {ov[c].x, ov[c].y, ov[c].z, ov[c].w}, d4[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc0 = fmaf(__uint_as_float(a[e] << 16), __uint_as_float(d4[e] << 16), acc0);
            acc1 = fmaf(__uint_as_float(a[e] & 0xffff0000u), __uint_as_float(d4[e] & 0xffff0000u), acc1);
          }
        }
        part = acc0 + acc1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(qdo_empty);                 // this warp is done with dO
      tmem_st1(tmem + lane_off + 384 + c0, __float_as_uint(part));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(delta_bar);
      ok = __all_sync(0xffffffffu, mbar_wait(delta_bar, k & 1, abort_flag, p.status, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      float dl;
      {
        uint32_t pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                       : "=r"(pv[i])
                       : "r"(tmem + lane_off + 384 + 32 * i));
        tmem_wait_ld();
        dl = ((__uint_as_float(pv[0]) + __uint_as_float(pv[1])) + __uint_as_float(pv[2])) + __uint_as_float(pv[3]);
      }
      if (w == 0) p.delta[row] = dl;
      for (int j = 0; j < x.T; ++j, ++J) {
        // P of this warpgroup's 32 keys from S (masked keys -> 0) while dP is still in the tensor
        // pipe; then dP, which frees the dP columns for the next tile's dP
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(J & 1), (J >> 1) & 1, abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + (J & 1) * 128 + c0;
        int nvalid;   // valid key columns of this tile for this row
        if (j < n_rt) {
          nvalid = min(BN, n_hist - j * BN);
        } else {
          const int64_t u0 = (int64_t)(j - n_rt) * BN;
          nvalid = (int)max((int64_t)0, min((int64_t)BN, t_pos - u0 + 1));
        }
        float pr[32];
        {
          uint32_t sv[32];
          tmem_ld32(tS, sv);
          tmem_wait_ld();
          auto pexp = [&](int e) { return ex2(fmaf(__uint_as_float(sv[e]), p.c2, -lse2)); };
          if (nvalid >= c0 + 32) {
#pragma unroll
            for (int e = 0; e < 32; ++e) pr[e] = pexp(e);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) pr[e] = (c0 + e < nvalid) ? pexp(e) : 0.f;
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(dp_full, J & 1, abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        uint32_t dv[32], pk[16];
        tmem_ld32(tmem + lane_off + 256 + c0, dv);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dp_free);
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pk[e >> 1] = pack_bf16(pr[e] * (__uint_as_float(dv[e]) - dl), pr[e + 1] * (__uint_as_float(dv[e + 1]) - dl));
        // packed bf16 dS stays inside this warpgroup's own (already read) column range
        tmem_st16(tS, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full(J & 1));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dq_ready, k & 1, abort_flag, p.status, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[32], pk[16];
      tmem_ld32(tmem + lane_off + 384 + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        pk[e >> 1] = pack_bf16(__uint_as_float(v[e]) * p.scale, __uint_as_float(v[e + 1]) * p.scale);
      // The row's 32 columns: 64 bytes at a 64-byte offset from dq.  With dq 32-byte aligned they
      // go out as two 32-byte stores (whole sectors); the interface only promises 16-byte
      // alignment, and then as four 16-byte stores.
      __nv_bfloat16* dst = p.dq + row * kD + c0;
      if (dq_v8) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16 * h), "r"(pk[8 * h]),
                       "r"(pk[8 * h + 1]), "r"(pk[8 * h + 2]), "r"(pk[8 * h + 3]), "r"(pk[8 * h + 4]),
                       "r"(pk[8 * h + 5]), "r"(pk[8 * h + 6]), "r"(pk[8 * h + 7])
                       : "memory");
      } else {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  pdl_wait();   // completes only after the kernel before, even when it gave up early
}

}  // namespace dq

// ======================================================================================== dK, dV
namespace dkdv {

constexpr int BM = 128;                     // keys per CTA (M dimension)
constexpr int BQ = 64;                      // queries per step
constexpr int NS = 4;                       // Q / dO / stats stages
constexpr uint32_t kKTile = BM * 256;       // 32 KB
constexpr uint32_t kKHalf = BM * 128;       // 16 KB
constexpr uint32_t kQTileB = BQ * 256;      // 16 KB
constexpr uint32_t kQHalfB = BQ * 128;      // 8 KB
constexpr uint32_t kStatBytes = 2 * BQ * 4; // lse[64], delta[64]

struct Params {
  int B, Hq, Hkv, G;
  int cs;               // CTAs per cluster (1 or 2): the query heads of one KV head are split over them
  int hpc;              // query heads per CTA (G = cs * hpc), accumulated in TMEM one after another
  int nblk, nkt;
  int64_t S;
  float c2, scale;
  const float* lse;
  const float* delta;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* xchg;          // cs == 2: per cluster, two [32 chunks of 4 columns x 2][64 rows] float32 areas
  int* status;
  uint64_t wait_ns;     // limit of every bounded mbarrier wait (drains excepted)
};

struct Smem {
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kKTile;
  static constexpr uint32_t kQ = kV + kKTile;
  static constexpr uint32_t kDO = kQ + NS * kQTileB;
  static constexpr uint32_t kStat = kDO + NS * kQTileB;
  static constexpr uint32_t kBar = kStat + NS * kStatBytes;
  // kv_full, q_full[NS], q_empty[NS], sd_full[2], pd_full[2], done, mma_done
  static constexpr int kNumBars = 1 + 2 * NS + 4 + 2;
  static constexpr uint32_t kMisc = kBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = kMisc + 16;
};

// Exchange area of one direction of one cluster: 64 key rows x 256 float32 (dV | dK), stored as
// [64 float4 chunks][64 rows] so that a warp's 32 rows of one chunk are 512 contiguous bytes.
constexpr size_t kXchgFloats = 64 * 256;
__device__ __forceinline__ size_t xchg_off(int chunk, int row) { return ((size_t)chunk * 64 + row) * 4; }

__global__ void __launch_bounds__(640, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                   const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                   const Params p) {
  using L = Smem;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBar;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const uint32_t kv_full = BAR(0);
  auto q_full = [&](int s) { return BAR(1 + s); };
  auto q_empty = [&](int s) { return BAR(1 + NS + s); };
  auto sd_full = [&](int b) { return BAR(1 + 2 * NS + b); };
  auto pd_full = [&](int b) { return BAR(3 + 2 * NS + b); };
  const uint32_t done = BAR(5 + 2 * NS);
  const uint32_t mma_done = BAR(6 + 2 * NS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- unit decode: key tile m (heavy = early first), batch x KV head, rank in the cluster
  // (the cluster's cs CTAs are consecutive blocks and share one key tile)
  const int crank = (int)cluster_rank();
  const int c = blockIdx.x / p.cs;
  const int bkh = c % (p.B * p.Hkv);
  const int m = c / (p.B * p.Hkv);
  const int b = bkh / p.Hkv, kh = bkh % p.Hkv;
  const int head0 = kh * p.G + crank * p.hpc;
  const int n0 = 2 * m;                       // first query block that sees this key tile
  const int Tq = p.nblk - n0;                 // query steps per head
  const int NJ = p.hpc * Tq;                  // steps of this CTA: head-major, then query block

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(sd_full(x), 1);
      mbar_init(pd_full(x), 256);
    }
    mbar_init(done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();
  uint32_t va[32], vb[32];   // element-wise threads after the main loop: 64 accumulator columns
  bool ew_ok = false;

  if (warp == 0) {
    // ======================= TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * kKTile);
      const int32_t krow = (int32_t)((int64_t)bkh * p.S + (int64_t)m * BM);
      tma_load_2d(sbase + L::kK, &tm_ks, 0, krow, kv_full);
      tma_load_2d(sbase + L::kK + kKHalf, &tm_ks, 64, krow, kv_full);
      tma_load_2d(sbase + L::kV, &tm_vs, 0, krow, kv_full);
      tma_load_2d(sbase + L::kV + kKHalf, &tm_vs, 64, krow, kv_full);
      // lse and delta (loaded with each Q/dO step) come from the forward and dQ kernels
      pdl_wait();
      int issued[NS] = {0, 0, 0, 0};
      for (int j = 0; j < NJ; ++j) {
        const int s = j % NS;
        const int t = j / Tq, i = j - t * Tq;
        if (!mbar_wait(q_empty(s), ((j / NS) & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
        mbar_arrive_expect_tx(q_full(s), 2 * kQTileB + kStatBytes);
        const int64_t row = ((int64_t)b * p.Hq + head0 + t) * p.S + (int64_t)(n0 + i) * BQ;
        tma_load_2d(sbase + L::kQ + s * kQTileB, &tm_q, 0, (int32_t)row, q_full(s));
        tma_load_2d(sbase + L::kQ + s * kQTileB + kQHalfB, &tm_q, 64, (int32_t)row, q_full(s));
        tma_load_2d(sbase + L::kDO + s * kQTileB, &tm_do, 0, (int32_t)row, q_full(s));
        tma_load_2d(sbase + L::kDO + s * kQTileB + kQHalfB, &tm_do, 64, (int32_t)row, q_full(s));
        bulk_load(sbase + L::kStat + s * kStatBytes, p.lse + row, BQ * 4, q_full(s));
        bulk_load(sbase + L::kStat + s * kStatBytes + BQ * 4, p.delta + row, BQ * 4, q_full(s));
        ++issued[s];
      }
      drain_wait(kv_full, 0, p.status);
      for (int s = 0; s < NS; ++s)
        if (issued[s]) drain_wait(q_full(s), (issued[s] - 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer: the whole warp runs the loop (warp-uniform descriptors
    // and waits) and one elected lane issues each tcgen05 instruction.  K and V are fixed for the
    // CTA, so their descriptor arrays are built once; Q / dO stage descriptors come from prebuilt
    // bases.
    {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BQ, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(BM, kD, true);
      uint64_t kd[8], vd[8];
      kmajor_descs(kd, sbase + L::kK, kKHalf, 1024);
      kmajor_descs(vd, sbase + L::kV, kKHalf, 1024);
      // stage st is st * kQTileB bytes after stage 0 (descriptor units of 16 bytes)
      const uint64_t q0 = smem_desc_sw128(sbase + L::kQ, 16, 1024);
      const uint64_t do0 = smem_desc_sw128(sbase + L::kDO, 16, 1024);
      const uint64_t qmn0 = smem_desc_sw128(sbase + L::kQ, kQHalfB, 1024);
      const uint64_t domn0 = smem_desc_sw128(sbase + L::kDO, kQHalfB, 1024);
      auto issue_sd = [&](int j, int x) {
        const uint64_t soff = (uint64_t)((j % NS) * (kQTileB >> 4));
        uint64_t bb[8];
        kmajor_from_base(bb, q0 + soff, kQHalfB >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + x * 128, kd[ks], bb[ks], idesc_s, ks > 0);
        kmajor_from_base(bb, do0 + soff, kQHalfB >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem + x * 128 + 64, vd[ks], bb[ks], idesc_s, ks > 0);
      };
      auto issue_grad = [&](int j, int x) {
        const uint64_t soff = (uint64_t)((j % NS) * (kQTileB >> 4));
        // dV += P^T dO ; dK += dS^T Q  (B operands MN-major: 64-dim halves 8 KB apart, 8 rows 1 KB apart).
        // P^T / dS^T of queries 32h..32h+31 sit in columns 32h..32h+15 of their region.
        uint64_t b1[4], b2[4];
        mnmajor_from_base<4>(b1, domn0 + soff, 2048u >> 4);
        mnmajor_from_base<4>(b2, qmn0 + soff, 2048u >> 4);
#pragma unroll
        for (int ks = 0; ks < BQ / 16; ++ks) {
          const uint32_t acol = (ks >> 1) * 32 + (ks & 1) * 8;
          mma_ts_w(tmem + 256, tmem + x * 128 + acol, b1[ks], idesc_g, (j > 0 || ks > 0));
          mma_ts_w(tmem + 384, tmem + x * 128 + 64 + acol, b2[ks], idesc_g, (j > 0 || ks > 0));
        }
      };
      bool ok = mbar_wait_w(kv_full, 0, abort_flag, p.status, p.wait_ns);
      for (int j = 0; ok && j < 2 && j < NJ; ++j) {
        ok = mbar_wait_w(q_full(j % NS), (j / NS) & 1, abort_flag, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_sd(j, j & 1);
        mma_commit_w(sd_full(j & 1));
      }
      for (int j = 0; ok && j < NJ; ++j) {
        const int x = j & 1;
        ok = mbar_wait_w(pd_full(x), (j >> 1) & 1, abort_flag, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_grad(j, x);
        mma_commit_w(q_empty(j % NS));
        if (j + 2 < NJ) {
          ok = mbar_wait_w(q_full((j + 2) % NS), ((j + 2) / NS) & 1, abort_flag, p.status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_sd(j + 2, x);
          mma_commit_w(sd_full(x));
        }
      }
      if (ok) mma_commit_w(done);
      mma_commit_w(mma_done);
      drain_wait(mma_done, 0, p.status);
    }
  } else if (warp >= 4) {
    // ======================= element-wise: P^T, dS^T.  Warpgroup w4 = 0..3 takes the steps
    // j = w4 mod 2 and the 32 query columns 32*(w4/2) .. of each (thread = TMEM lane = key row).
    const int w4 = (warp - 4) >> 2;
    const int x = w4 & 1, hc = w4 >> 1;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // key row within the tile
    const int64_t u = (int64_t)m * BM + r;      // key position in the segment
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + x * 128;
    const uint32_t tP = tS + 64;
    const float* stat_base = reinterpret_cast<const float*>(smem + L::kStat);
    bool ok = true;
    for (int j = x; j < NJ; j += 2) {
      const int s = j % NS;
      const int i = j % Tq;
      ok = mbar_wait(sd_full(x), (j >> 1) & 1, abort_flag, p.status, p.wait_ns);
      if (ok) ok = mbar_wait(q_full(s), (j / NS) & 1, abort_flag, p.status, p.wait_ns);   // stats landed
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* lse = stat_base + s * (kStatBytes / 4);
      const float* dlt = lse + BQ;
      const int64_t t0 = (int64_t)(n0 + i) * BQ;
      const bool diag = i < 2;                  // only the first two steps overlap the key tile
      // one TMEM round trip per step: both loads in flight, one wait, compute, both stores
      uint32_t sv[32], dv[32], pp[16], pd[16];
      tmem_ld32(tS + 32 * hc, sv);
      tmem_ld32(tP + 32 * hc, dv);
      tmem_wait_ld();
      const int q0 = 32 * hc;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse + q0 + e);
        const float4 d4 = *reinterpret_cast<const float4*>(dlt + q0 + e);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
        float pr[4], dsr[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          float pv = ex2(fmaf(__uint_as_float(sv[e + f]), p.c2, -lv[f] * kLog2e));
          if (diag && u > t0 + q0 + e + f) pv = 0.f;
          pr[f] = pv;
          dsr[f] = pv * (__uint_as_float(dv[e + f]) - dd[f]);
        }
        pp[e >> 1] = pack_bf16(pr[0], pr[1]);
        pp[(e >> 1) + 1] = pack_bf16(pr[2], pr[3]);
        pd[e >> 1] = pack_bf16(dsr[0], dsr[1]);
        pd[(e >> 1) + 1] = pack_bf16(dsr[2], dsr[3]);
      }
      // packed bf16 stays inside this warpgroup's own (already read) column range
      tmem_st16(tS + 32 * hc, pp);
      tmem_st16(tP + 32 * hc, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pd_full(x));
    }
    // ---- epilogue: warpgroups 0,1 own dV columns 0-63 / 64-127, warpgroups 2,3 the same of dK;
    // after `done` every MMA has completed and each thread takes its 64 columns of the float32 sums
    // over this CTA's heads into registers.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, p.status, p.wait_ns));
    if (ok) {
      tc_fence_after();
      const uint32_t tacc = tmem + lane_off + (w4 >= 2 ? 384 : 256) + 64 * (w4 & 1);
      tmem_ld32(tacc, va);
      tmem_ld32(tacc + 32, vb);
      tmem_wait_ld();
    }
    ew_ok = ok;
  }
  // ---- reduction over the query heads of this KV head and store.  In a cluster of two, CTA
  // `crank` writes key rows [64 crank, 64 crank + 64): each thread holding a row of the other half
  // stores its 64 float32 sums into the cluster's exchange area for the peer (L2-resident; a
  // transfer through distributed shared memory measured several times slower), then a release /
  // acquire cluster barrier, then each owner adds the row the peer left for it and stores bf16.  A
  // sum of two terms does not depend on their order, so the result is reproducible.  Every thread
  // takes part in the barriers on the error path too; a CTA that gave up leaves arbitrary rows and
  // the status word says so.
  const int nrows = BM / p.cs;
  const int r0 = crank * nrows;
  const int er = (warp & 3) * 32 + lane;                  // element-wise thread: key row (TMEM lane)
  const int ew4 = (warp - 4) >> 2;
  const int c16 = (ew4 >= 2 ? 32 : 0) + 16 * (ew4 & 1);   // first float4 chunk of its 64 columns
  const bool mine = er >= r0 && er < r0 + nrows;
  float* xc = p.xchg + (size_t)c * 2 * kXchgFloats;        // this cluster's two areas
  if (p.cs == 2 && warp >= 4 && ew_ok && !mine) {
    float* to = xc + (size_t)(crank ^ 1) * kXchgFloats;
    const int rl = er - (crank ^ 1) * nrows;
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      __stcg(reinterpret_cast<float4*>(to + xchg_off(c16 + e / 4, rl)),
             make_float4(__uint_as_float(va[e]), __uint_as_float(va[e + 1]), __uint_as_float(va[e + 2]),
                         __uint_as_float(va[e + 3])));
      __stcg(reinterpret_cast<float4*>(to + xchg_off(c16 + 8 + e / 4, rl)),
             make_float4(__uint_as_float(vb[e]), __uint_as_float(vb[e + 1]), __uint_as_float(vb[e + 2]),
                         __uint_as_float(vb[e + 3])));
    }
    __threadfence();
  }
  tc_fence_before();
  if (p.cs == 2) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (warp >= 4 && ew_ok && mine && (int64_t)m * BM + er < p.S) {
    // the row's 64 bf16 columns go into this warp's 4 KB slot of the (now unused) K/V stage area in
    // the 128-byte swizzled layout of a {64 columns, 32 rows} box, and the warp stores its 32 rows
    // with one TMA store (the rows past the segment end are whole warps, S being a multiple of 64)
    const bool is_dk = ew4 >= 2;
    const float mul = is_dk ? p.scale : 1.f;
    const float* from = xc + (size_t)crank * kXchgFloats;
    const int rl = er - r0;
    const uint32_t slot = sbase + L::kK + (uint32_t)(warp - 4) * 4096u;
    const uint32_t row_addr = slot + (uint32_t)lane * 128u;
    auto stage32 = [&](const uint32_t(&v)[32], int cbase, int chunk0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * q + e]);
        if (p.cs == 2) {
          const float4 x0 = __ldcg(reinterpret_cast<const float4*>(from + xchg_off(cbase + 2 * q, rl)));
          const float4 x1 = __ldcg(reinterpret_cast<const float4*>(from + xchg_off(cbase + 2 * q + 1, rl)));
          f[0] += x0.x; f[1] += x0.y; f[2] += x0.z; f[3] += x0.w;
          f[4] += x1.x; f[5] += x1.y; f[6] += x1.z; f[7] += x1.w;
        }
        const uint32_t chunk = (uint32_t)(chunk0 + q);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + ((chunk ^ (uint32_t)(lane & 7)) << 4)),
                     "r"(pack_bf16(f[0] * mul, f[1] * mul)), "r"(pack_bf16(f[2] * mul, f[3] * mul)),
                     "r"(pack_bf16(f[4] * mul, f[5] * mul)), "r"(pack_bf16(f[6] * mul, f[7] * mul))
                     : "memory");
      }
    };
    stage32(va, c16, 0);
    stage32(vb, c16 + 8, 4);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int32_t row0 = (int32_t)((int64_t)bkh * p.S + (int64_t)m * BM + (warp & 3) * 32);
      tma_store_2d(is_dk ? &tm_dk : &tm_dv, 64 * (ew4 & 1), row0, slot);
      bulk_commit_group();
      bulk_wait_read_all();   // the shared-memory source must be read before the CTA exits
    }
    __syncwarp();
  }
  pdl_wait();   // completes only after the kernel before, even when it gave up early
}

}  // namespace dkdv
}  // namespace tcbwd

// ------------------------------------------------------------------ host side
cudaError_t launch_bwd_dq_tc(const void* q, const void* kh, const void* vh, const void* ks, const void* vs,
                             const int32_t* gi, const float* lse, const void* o, const void* d_o, float* delta,
                             void* dq, int B, int Hq, int Hkv, int64_t H, int64_t S, int64_t Hs, int kg, int nsg,
                             float scale, int* status, uint64_t wait_ns, cudaStream_t st) {
  namespace K = tcbwd::dq;
  CUtensorMap mq, mdo, mkh, mvh, mks, mvs;
  // with no history the history maps are never used: map the segment instead (maps need rows > 0)
  const void* kh_m = Hs ? kh : ks;
  const void* vh_m = Hs ? vh : vs;
  const uint64_t hrows = (uint64_t)B * Hkv * (Hs ? Hs : S);
  if (!make_map_bf16_rows(&mq, q, (uint64_t)B * Hq * S, 64) || !make_map_bf16_rows(&mdo, d_o, (uint64_t)B * Hq * S, 64) ||
      !make_map_bf16_groups(&mkh, kh_m, hrows) || !make_map_bf16_groups(&mvh, vh_m, hrows) ||
      !make_map_bf16_rows(&mks, ks, (uint64_t)B * Hkv * S, K::BN) ||
      !make_map_bf16_rows(&mvs, vs, (uint64_t)B * Hkv * S, K::BN))
    return cudaErrorInvalidValue;
  const int G = Hq / Hkv;
  K::Params p{B, Hq, Hkv, G, kg, (int)(S / kQBlock), nsg, H, S, Hs, scale * tcbwd::kLog2e, scale, gi, lse,
              static_cast<const __nv_bfloat16*>(o), delta, static_cast<__nv_bfloat16*>(dq), status, wait_ns};
  // persistent: one CTA per SM (or per unit, when there are fewer units than SMs)
  const int64_t units = (int64_t)B * Hkv * p.nblk * (G / 2);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int64_t grid = units < sms ? units : sms;
  const size_t smem = K::Smem::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(K::dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(K::dq_tc_kernel, dim3((unsigned)grid), dim3(128 + 32 * K::kEWWarps), smem, st, 1, mq, mdo, mkh,
                       mvh, mks, mvs, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// CTAs per cluster of the dK/dV kernel.  With one CTA per (batch, KV head, key tile) every CTA
// sums all G query heads in TMEM and no reduction is needed; when that gives fewer CTAs than the GPU
// has SMs (and G is even) the heads are split over a cluster of two.  (Clusters of four CTAs of one
// SM each leave SMs of the graphics processing clusters idle and measured slower.)
int dkdv_cluster_size(int B, int Hkv, int G, int nkt) {
  if (G % 2 != 0) return 1;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  return ((int64_t)B * Hkv * nkt >= sms) ? 1 : 2;
}

// Bytes of the exchange area the dK/dV kernel uses when it pairs CTAs (0 when it does not).
size_t dkdv_xchg_bytes(int B, int Hq, int Hkv, int64_t S) {
  const int nkt = (int)((S + tcbwd::dkdv::BM - 1) / tcbwd::dkdv::BM);
  if (dkdv_cluster_size(B, Hkv, Hq / Hkv, nkt) != 2) return 0;
  return (size_t)B * Hkv * nkt * 2 * tcbwd::dkdv::kXchgFloats * sizeof(float);
}

// xchg: the exchange area (dkdv_xchg_bytes), or nullptr, in which case no CTAs are paired.
cudaError_t launch_bwd_dkdv_tc(const void* q, const void* ks, const void* vs, const float* lse, const void* d_o,
                               const float* delta, void* dk, void* dv, float* xchg, int B, int Hq, int Hkv, int64_t S,
                               float scale, int* status, uint64_t wait_ns, cudaStream_t st) {
  namespace K = tcbwd::dkdv;
  CUtensorMap mq, mdo, mks, mvs, mdk, mdv;
  if (!make_map_bf16_rows(&mq, q, (uint64_t)B * Hq * S, K::BQ) ||
      !make_map_bf16_rows(&mdo, d_o, (uint64_t)B * Hq * S, K::BQ) ||
      !make_map_bf16_rows(&mks, ks, (uint64_t)B * Hkv * S, K::BM) ||
      !make_map_bf16_rows(&mvs, vs, (uint64_t)B * Hkv * S, K::BM) ||
      !make_map_bf16_rows(&mdk, dk, (uint64_t)B * Hkv * S, 32) || !make_map_bf16_rows(&mdv, dv, (uint64_t)B * Hkv * S, 32))
    return cudaErrorInvalidValue;
  const int G = Hq / Hkv;
  const int nkt = (int)((S + K::BM - 1) / K::BM);
  const int cs = xchg ? dkdv_cluster_size(B, Hkv, G, nkt) : 1;
  K::Params p{B, Hq, Hkv, G, cs, G / cs, (int)(S / kQBlock), nkt, S, scale * tcbwd::kLog2e, scale, lse, delta,
              static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), xchg, status, wait_ns};
  const int64_t grid = (int64_t)B * Hkv * nkt * cs;
  const size_t smem = K::Smem::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(K::dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(K::dkdv_tc_kernel, dim3((unsigned)grid), dim3(640), smem, st, (unsigned)cs, mq, mdo, mks, mvs, mdk,
                       mdv, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hga
