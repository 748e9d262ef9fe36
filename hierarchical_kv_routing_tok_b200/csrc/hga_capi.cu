// C ABI of the routed-HGA library (declarations and contract in include/hga.h).
// Validates every argument on the host, then enqueues the kernels on the
// caller's stream.  No allocation, no synchronisation (except hga_read_status).
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "hga.h"
#include "common.cuh"

namespace hga {
cudaError_t launch_summaries(bool bf16, const void* k_hist, float* group_sum, float* chunk_sum, int64_t BHkv,
                             int64_t Hs, int64_t c0, int64_t c1, cudaStream_t stream);
size_t route_split_bytes(int64_t units, int64_t nblk, int nch, int nsc);
cudaError_t launch_route_split(bool bf16, const void* q, const void* q_prev, bool causal, const float* group_sum,
                               const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, int B, int Hq,
                               int Hkv, int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, void* scratch,
                               cudaStream_t stream);
cudaError_t launch_route(bool bf16, const void* q, const void* q_prev, bool causal, const float* group_sum,
                         const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, int B, int Hq, int Hkv,
                         int64_t S, int nch, int nch_stride, int nsc, int kc, int kg, cudaStream_t stream);
size_t route_smem_bytes(bool bf16, int nch, int kc, int kg);
cudaError_t launch_route_chunks(bool bf16, const void* q, const void* q_prev, bool causal, const float* chunk_sum,
                                int32_t* chunk_idx, float* qb, int B, int Hq, int Hkv, int64_t S, int nch,
                                int nch_stride, int nsc, int kc, cudaStream_t stream);
cudaError_t launch_route_groups_cached(const float* qb, const int32_t* chunk_idx, const int32_t* slot_of,
                                       const float* gcache, int cap, int32_t* group_idx, int B, int Hkv, int64_t S,
                                       int nch_stride, int kc, int kg, int* status, cudaStream_t stream);
size_t gcache_plan_smem_bytes(int nchs, int cap);
cudaError_t launch_gcache_plan(const int32_t* chunk_idx, int BHkv, int nidx, int nchs, int cap, int step,
                               int32_t* slot_of, int32_t* chunk_of, int32_t* stamp, int32_t* miss_chunk,
                               int32_t* miss_slot, int32_t* counts, int* status, cudaStream_t st);
cudaError_t launch_gcache_fetch(const float* gsum, int64_t ngrs, const int32_t* miss_chunk, const int32_t* miss_slot,
                                const int32_t* counts, int BHkv, int cap, float* gcache, cudaStream_t st);
cudaError_t launch_attn_fwd_simt(bool bf16, const void* q, const void* kh, const void* vh, const void* ks,
                                 const void* vs, const int32_t* gi, void* o, float* lse, int B, int Hq, int Hkv,
                                 int64_t H, int64_t S, int64_t Hs, int kg, int nsg, float scale, int* status,
                                 cudaStream_t st);
bool attn_fwd_tc_supported(int Hq, int Hkv);
cudaError_t launch_attn_fwd_tc(const void* q, const void* kh, const void* vh, const void* ks, const void* vs,
                               const int32_t* gi, void* o, float* lse, int B, int Hq, int Hkv, int64_t H, int64_t S,
                               int64_t Hs, int kg, int nsg, float scale, int* status, uint64_t wait_ns,
                               cudaStream_t st);
cudaError_t launch_bwd_dq_tc(const void* q, const void* kh, const void* vh, const void* ks, const void* vs,
                             const int32_t* gi, const float* lse, const void* o, const void* d_o, float* delta,
                             void* dq, int B, int Hq, int Hkv, int64_t H, int64_t S, int64_t Hs, int kg, int nsg,
                             float scale, int* status, uint64_t wait_ns, cudaStream_t st);
size_t dkdv_xchg_bytes(int B, int Hq, int Hkv, int64_t S);
cudaError_t launch_bwd_dkdv_tc(const void* q, const void* ks, const void* vs, const float* lse, const void* d_o,
                               const float* delta, void* dk, void* dv, float* xchg, int B, int Hq, int Hkv, int64_t S,
                               float scale, int* status, uint64_t wait_ns, cudaStream_t st);
cudaError_t launch_bwd_delta_simt(bool bf16, const void* o, const void* d_o, float* delta, int B, int Hq,
                                  int64_t S, cudaStream_t st);
cudaError_t launch_bwd_dkdv_simt(bool bf16, const void* q, const void* ks, const void* vs, const float* lse,
                                 const void* d_o, const float* delta, void* dk, void* dv, int B, int Hq, int Hkv,
                                 int64_t H, int64_t S, int kg, float scale, cudaStream_t st);
cudaError_t launch_bwd_dq_simt(bool bf16, const void* q, const void* kh, const void* vh, const void* ks,
                               const void* vs, const int32_t* gi, const float* lse, const void* d_o,
                               const float* delta, void* dq, int B, int Hq, int Hkv, int64_t H, int64_t S,
                               int64_t Hs, int kg, int nsg, float scale, int* status, cudaStream_t st);
size_t tier_plan_smem_bytes(int ngr);
cudaError_t launch_tier_plan(const int32_t* group_idx, int BHkv, int nblk, int kg, int nsg, int ngr, int cap,
                             int32_t* used_groups, int32_t* n_used, int32_t* compact_idx, int* status,
                             cudaStream_t st);
cudaError_t launch_tier_gather(bool bf16, const void* kh, const void* vh, const int32_t* used_groups,
                               const int32_t* n_used, int BHkv, int64_t H, int cap, void* kc, void* vc,
                               cudaStream_t st);
}  // namespace hga

namespace {

constexpr int64_t kMaxChunks = 32768;             // routing keeps one score per chunk in smem
constexpr size_t kMaxRouteSmem = 200 * 1024;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_config(const hga_config_t* c) {
  if (!c) return HGA_ERR_ARG;
  if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv != 0) return HGA_ERR_ARG;
  if (c->dtype != HGA_F32 && c->dtype != HGA_BF16) return HGA_ERR_ARG;
  if (c->D != hga::kD || c->chunk != hga::kChunk || c->group != hga::kGroup || c->qblock != hga::kQBlock)
    return HGA_ERR_UNSUPPORTED;
  if (c->hist_len < 0 || c->hist_len % c->chunk != 0) return HGA_ERR_ARG;
  if (c->hist_capacity != 0 && (c->hist_capacity < c->hist_len || c->hist_capacity % c->chunk != 0))
    return HGA_ERR_ARG;
  if (c->seg_len < c->qblock || c->seg_len % c->qblock != 0) return HGA_ERR_ARG;
  const int64_t nch = c->hist_len / c->chunk;
  if (nch > kMaxChunks) return HGA_ERR_UNSUPPORTED;
  if (nch == 0) {
    // no history yet (the first segment of a sequence): local attention only, nothing to route
    if (c->top_chunks != 0 || c->top_groups != 0 || c->n_sink_tokens != 0) return HGA_ERR_ARG;
  } else {
    // the sink window: whole chunks at the start of the history, at least one chunk left to route
    if (c->n_sink_tokens < 0 || c->n_sink_tokens % c->chunk != 0 || c->n_sink_tokens >= c->hist_len)
      return HGA_ERR_ARG;
    const int64_t nsc = c->n_sink_tokens / c->chunk;
    if (c->top_chunks < 1 || c->top_chunks > nch - nsc) return HGA_ERR_ARG;
    if (c->top_groups < 1 || (int64_t)c->top_groups > (int64_t)c->top_chunks * (c->chunk / c->group))
      return HGA_ERR_ARG;
  }
  if (!(c->softmax_scale >= 0.f) || isinf(c->softmax_scale)) return HGA_ERR_ARG;
  if (c->wait_limit_ns < 0) return HGA_ERR_ARG;
  // grid dimensions are 32-bit
  if ((int64_t)c->B * c->Hq * (c->seg_len / c->qblock) > INT32_MAX) return HGA_ERR_UNSUPPORTED;
  if ((int64_t)c->B * c->Hkv * nch > (int64_t)INT32_MAX) return HGA_ERR_UNSUPPORTED;   // one CTA per chunk
  // history rows are addressed with 32-bit tensor-map coordinates
  const int64_t hs = c->hist_capacity ? c->hist_capacity : c->hist_len;
  if ((int64_t)c->B * c->Hkv * hs > (int64_t)INT32_MAX) return HGA_ERR_UNSUPPORTED;
  if (nch && hga::route_smem_bytes(c->dtype == HGA_BF16, (int)nch, c->top_chunks, c->top_groups) > kMaxRouteSmem)
    return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p) return HGA_ERR_ARG;
  for (const void* p : ps)
    if (!aligned16(p)) return HGA_ERR_ALIGN;
  return HGA_OK;
}

// Rows per (batch, KV head) of the history and summary buffers (the history's capacity).
int64_t hist_rows(const hga_config_t* c) { return c->hist_capacity ? c->hist_capacity : c->hist_len; }

// Groups of the sink window, attended by every query ahead of the routed groups.
int sink_groups(const hga_config_t* c) { return (int)(c->n_sink_tokens / c->group); }

// int32 index arrays are read and written with 4-byte accesses: non-null and 4-byte aligned.
int check_idx(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p) return HGA_ERR_ARG;
  for (const void* p : ps)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return HGA_ERR_ALIGN;
  return HGA_OK;
}

// History K/V and routed group indices of the attention calls; with no history (hist_len == 0)
// none of them is read and they may be NULL.
int check_history(const hga_config_t* c, const void* k_hist, const void* v_hist, const int32_t* group_idx) {
  if (c->hist_len == 0) return HGA_OK;
  int rc = check_ptrs({k_hist, v_hist});
  return rc ? rc : check_idx({group_idx});
}

// Limit of the tensor-core kernels' bounded on-chip waits: wait_limit_ns, or 2 s when it is 0.
uint64_t wait_limit(const hga_config_t* c) {
  return c->wait_limit_ns > 0 ? (uint64_t)c->wait_limit_ns : 2000000000ull;
}

float eff_scale(const hga_config_t* c) {
  return c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / sqrtf((float)c->D);
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? HGA_OK : HGA_ERR_CUDA; }

// HGA_ATTN_PATH=cuda_cores selects the CUDA-core attention kernels for every dtype (the
// tensor-core kernels are the default for bf16); used to cross-check the two implementations.
bool force_cuda_cores() {
  const char* v = getenv("HGA_ATTN_PATH");
  return v && strcmp(v, "cuda_cores") == 0;
}

// The workspace starts with the status word.
int* status_of(void* workspace) { return static_cast<int*>(workspace); }

// The tensor-core attention kernels handle bf16 with an even number of query heads per KV head.
bool use_tc(const hga_config_t* c) {
  return c->dtype == HGA_BF16 && hga::attn_fwd_tc_supported(c->Hq, c->Hkv) && !force_cuda_cores();
}

// Workspace layout: [status word | delta rows (float32) | dK/dV exchange area].  The exchange area
// is used only by the tensor-core dK/dV kernel when it pairs CTAs (few (batch, KV head, key tile)
// units for the GPU's SMs); a workspace that ends before it (the no-allocation entry point's fixed
// scratch) runs that kernel unpaired.
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t delta_bytes(const hga_config_t* c) { return (size_t)c->B * c->Hq * c->seg_len * sizeof(float); }
float* delta_of(void* workspace) {
  return reinterpret_cast<float*>(static_cast<char*>(workspace) + hga::kStatusBytes);
}
size_t base_workspace_bytes(const hga_config_t* c) { return hga::kStatusBytes + round256(delta_bytes(c)); }
size_t xchg_bytes(const hga_config_t* c) {
  return use_tc(c) ? hga::dkdv_xchg_bytes(c->B, c->Hq, c->Hkv, c->seg_len) : 0;
}
// Scratch of the three-launch routing of long histories (block queries and chunk scores; 0 when the
// history is short enough for the single launch).  Routing and the dK/dV kernel never run at once on
// a workspace, so the two share the region after the status word and the delta rows.
size_t route_bytes(const hga_config_t* c) {
  const int64_t nblk = c->seg_len / c->qblock;
  return hga::route_split_bytes((int64_t)c->B * c->Hkv * nblk, nblk, (int)(c->hist_len / c->chunk),
                                (int)(c->n_sink_tokens / c->chunk));
}
size_t full_workspace_bytes(const hga_config_t* c) {
  const size_t x = xchg_bytes(c), r = route_bytes(c);
  return base_workspace_bytes(c) + (x > r ? x : r);
}
float* xchg_of(void* workspace, const hga_config_t* c, size_t ws_bytes) {
  const size_t x = xchg_bytes(c);
  if (x == 0 || ws_bytes < base_workspace_bytes(c) + x) return nullptr;
  return reinterpret_cast<float*>(static_cast<char*>(workspace) + base_workspace_bytes(c));
}

// dK/dV with a workspace of ws_bytes (status word and delta rows).
int bwd_dkdv_ws(const hga_config_t* cfg, const void* q, const void* k_seg, const void* v_seg, const float* lse,
                const void* d_o, void* dk_seg, void* dv_seg, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_ptrs({q, k_seg, v_seg, lse, d_o, dk_seg, dv_seg});
  if (rc) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ws_bytes < base_workspace_bytes(cfg)) return HGA_ERR_WORKSPACE;
  if (use_tc(cfg))
    return from_cuda(hga::launch_bwd_dkdv_tc(q, k_seg, v_seg, lse, d_o, delta_of(workspace), dk_seg, dv_seg,
                                             xchg_of(workspace, cfg, ws_bytes), cfg->B, cfg->Hq, cfg->Hkv,
                                             cfg->seg_len, eff_scale(cfg), status_of(workspace), wait_limit(cfg),
                                             st));
  return from_cuda(hga::launch_bwd_dkdv_simt(cfg->dtype == HGA_BF16, q, k_seg, v_seg, lse, d_o, delta_of(workspace),
                                             dk_seg, dv_seg, cfg->B, cfg->Hq, cfg->Hkv, cfg->hist_len, cfg->seg_len,
                                             cfg->top_groups, eff_scale(cfg), st));
}

// Groups of the compact history cache of a tiered step: every group a step can route to (the
// sink groups plus k_g per query block, at most the whole history), rounded up to whole chunks, and
// at least enough whole chunks for the sink and k_g routed groups (so the cache is a valid history
// for a configuration whose routing budget is ceil(k_g / 8) chunks).
int64_t tier_cap_groups(const hga_config_t* c) {
  const int64_t gpc = c->chunk / c->group, ngr = c->hist_len / c->group, nsg = c->n_sink_tokens / c->group;
  const int64_t nblk = c->seg_len / c->qblock;
  int64_t cap = nsg + nblk * c->top_groups;
  if (cap > ngr) cap = ngr;
  const int64_t least = nsg + gpc * ((c->top_groups + gpc - 1) / gpc);
  if (cap < least) cap = least;
  cap = (cap + gpc - 1) / gpc * gpc;
  return cap < ngr ? cap : ngr;
}

// Device-accessible address of a buffer of `bytes` bytes that is either device memory or pinned
// host memory mapped into the device's address space (both ends checked); nullptr otherwise.
const void* device_view(const void* p, size_t bytes) {
  const char* ends[2] = {static_cast<const char*>(p), static_cast<const char*>(p) + (bytes ? bytes - 1 : 0)};
  const void* dev = nullptr;
  for (int i = 0; i < 2; ++i) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ends[i]) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if ((a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeHost && a.type != cudaMemoryTypeManaged) ||
        a.devicePointer == nullptr)
      return nullptr;
    if (i == 0) dev = a.devicePointer;
  }
  return dev;
}

}  // namespace

// The whole backward with a workspace of ws_bytes (also used by the no-allocation entry point).
int hga_internal_attn_bwd_ws(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist,
                             const void* k_seg, const void* v_seg, const int32_t* group_idx, const void* o,
                             const float* lse, const void* d_o, void* dq, void* dk_seg, void* dv_seg, void* workspace,
                             size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, k_seg, v_seg, o, lse, d_o, dq, dk_seg, dv_seg}))) return rc;
  if ((rc = check_history(cfg, k_hist, v_hist, group_idx))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  // dQ first: it also forms delta = rowsum(dO o O) into the workspace, which dK/dV then reads
  if ((rc = hga_attn_bwd_dq(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, workspace, stream)))
    return rc;
  return bwd_dkdv_ws(cfg, q, k_seg, v_seg, lse, d_o, dk_seg, dv_seg, workspace, ws_bytes, stream);
}

extern "C" {

int hga_version(void) { return HGA_VERSION; }

const char* hga_strerror(int code) {
  switch (code) {
    case HGA_OK: return "ok";
    case HGA_ERR_ARG: return "invalid argument (shape, budget or null pointer)";
    case HGA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case HGA_ERR_UNSUPPORTED: return "configuration not supported by this build";
    case HGA_ERR_CUDA: return "CUDA launch or copy failed";
    case HGA_ERR_TIMEOUT: return "device-side bounded wait expired";
    case HGA_ERR_WORKSPACE: return "workspace missing";
    case HGA_ERR_TOO_LARGE: return "problem larger than the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

int hga_workspace_size(const hga_config_t* cfg, size_t* bytes_out) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!bytes_out) return HGA_ERR_ARG;
  *bytes_out = full_workspace_bytes(cfg);
  return HGA_OK;
}

int hga_route_launches(const hga_config_t* cfg, int with_workspace, int32_t* launches_out) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!launches_out) return HGA_ERR_ARG;
  *launches_out = cfg->hist_len == 0 ? 0 : (with_workspace && route_bytes(cfg) > 0) ? 3 : 1;
  return HGA_OK;
}

int hga_build_summaries(const hga_config_t* cfg, const void* k_hist, float* group_sum, float* chunk_sum,
                        void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({k_hist, group_sum, chunk_sum}))) return rc;
  (void)workspace;
  return from_cuda(hga::launch_summaries(cfg->dtype == HGA_BF16, k_hist, group_sum, chunk_sum,
                                         (int64_t)cfg->B * cfg->Hkv, hist_rows(cfg), 0, cfg->hist_len / cfg->chunk,
                                         static_cast<cudaStream_t>(stream)));
}

int hga_append_summaries(const hga_config_t* cfg, const void* k_hist, float* group_sum, float* chunk_sum,
                         int64_t first_token, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({k_hist, group_sum, chunk_sum}))) return rc;
  if (first_token < 0 || first_token > cfg->hist_len || first_token % cfg->chunk != 0) return HGA_ERR_ARG;
  (void)workspace;
  return from_cuda(hga::launch_summaries(cfg->dtype == HGA_BF16, k_hist, group_sum, chunk_sum,
                                         (int64_t)cfg->B * cfg->Hkv, hist_rows(cfg), first_token / cfg->chunk,
                                         cfg->hist_len / cfg->chunk, static_cast<cudaStream_t>(stream)));
}

int hga_route(const hga_config_t* cfg, const void* q, const float* group_sum, const float* chunk_sum,
              int32_t* chunk_idx, int32_t* group_idx, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, group_sum, chunk_sum}))) return rc;
  if (cfg->hist_len == 0) return HGA_OK;        // nothing to route
  if ((rc = check_idx({chunk_idx, group_idx}))) return rc;
  const int nch = (int)(cfg->hist_len / cfg->chunk), nsc = (int)(cfg->n_sink_tokens / cfg->chunk);
  if (workspace && route_bytes(cfg) > 0) {
    if (!aligned16(workspace)) return HGA_ERR_ALIGN;
    return from_cuda(hga::launch_route_split(cfg->dtype == HGA_BF16, q, nullptr, false, group_sum, chunk_sum, chunk_idx,
                                             group_idx, cfg->B, cfg->Hq, cfg->Hkv, cfg->seg_len, nch,
                                             (int)(hist_rows(cfg) / cfg->chunk), nsc, cfg->top_chunks,
                                             cfg->top_groups,
                                             static_cast<char*>(workspace) + base_workspace_bytes(cfg),
                                             static_cast<cudaStream_t>(stream)));
  }
  return from_cuda(hga::launch_route(cfg->dtype == HGA_BF16, q, nullptr, false, group_sum, chunk_sum, chunk_idx,
                                     group_idx, cfg->B, cfg->Hq, cfg->Hkv, cfg->seg_len, nch,
                                     (int)(hist_rows(cfg) / cfg->chunk), nsc, cfg->top_chunks, cfg->top_groups,
                                     static_cast<cudaStream_t>(stream)));
}

int hga_route_causal(const hga_config_t* cfg, const void* q, const void* q_prev, const float* group_sum,
                     const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, group_sum, chunk_sum}))) return rc;
  if (q_prev && !aligned16(q_prev)) return HGA_ERR_ALIGN;
  if (cfg->hist_len == 0) return HGA_OK;        // nothing to route
  if ((rc = check_idx({chunk_idx, group_idx}))) return rc;
  const int nch = (int)(cfg->hist_len / cfg->chunk), nsc = (int)(cfg->n_sink_tokens / cfg->chunk);
  if (workspace && route_bytes(cfg) > 0) {
    if (!aligned16(workspace)) return HGA_ERR_ALIGN;
    return from_cuda(hga::launch_route_split(cfg->dtype == HGA_BF16, q, q_prev, true, group_sum, chunk_sum, chunk_idx,
                                             group_idx, cfg->B, cfg->Hq, cfg->Hkv, cfg->seg_len, nch,
                                             (int)(hist_rows(cfg) / cfg->chunk), nsc, cfg->top_chunks,
                                             cfg->top_groups,
                                             static_cast<char*>(workspace) + base_workspace_bytes(cfg),
                                             static_cast<cudaStream_t>(stream)));
  }
  return from_cuda(hga::launch_route(cfg->dtype == HGA_BF16, q, q_prev, true, group_sum, chunk_sum, chunk_idx,
                                     group_idx, cfg->B, cfg->Hq, cfg->Hkv, cfg->seg_len, nch,
                                     (int)(hist_rows(cfg) / cfg->chunk), nsc, cfg->top_chunks, cfg->top_groups,
                                     static_cast<cudaStream_t>(stream)));
}

int hga_attn_fwd(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist, const void* k_seg,
                 const void* v_seg, const int32_t* group_idx, void* o, float* lse, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, k_seg, v_seg, o, lse}))) return rc;
  if ((rc = check_history(cfg, k_hist, v_hist, group_idx))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  const bool bf16 = cfg->dtype == HGA_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_tc(cfg))
    return from_cuda(hga::launch_attn_fwd_tc(q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, cfg->B, cfg->Hq,
                                             cfg->Hkv, cfg->hist_len, cfg->seg_len, hist_rows(cfg), cfg->top_groups,
                                             sink_groups(cfg), eff_scale(cfg), status_of(workspace), wait_limit(cfg),
                                             st));
  return from_cuda(hga::launch_attn_fwd_simt(bf16, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, cfg->B,
                                             cfg->Hq, cfg->Hkv, cfg->hist_len, cfg->seg_len, hist_rows(cfg),
                                             cfg->top_groups, sink_groups(cfg), eff_scale(cfg), status_of(workspace),
                                             st));
}

int hga_attn_bwd_preprocess(const hga_config_t* cfg, const void* o, const void* d_o, void* workspace,
                            void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({o, d_o}))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  return from_cuda(hga::launch_bwd_delta_simt(cfg->dtype == HGA_BF16, o, d_o, delta_of(workspace), cfg->B, cfg->Hq,
                                              cfg->seg_len, static_cast<cudaStream_t>(stream)));
}

int hga_attn_bwd_dkdv(const hga_config_t* cfg, const void* q, const void* k_seg, const void* v_seg, const float* lse,
                      const void* d_o, void* dk_seg, void* dv_seg, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  return bwd_dkdv_ws(cfg, q, k_seg, v_seg, lse, d_o, dk_seg, dv_seg, workspace, full_workspace_bytes(cfg), stream);
}

int hga_attn_bwd_dq(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist, const void* k_seg,
                    const void* v_seg, const int32_t* group_idx, const void* o, const float* lse, const void* d_o,
                    void* dq, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, k_seg, v_seg, o, lse, d_o, dq}))) return rc;
  if ((rc = check_history(cfg, k_hist, v_hist, group_idx))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_tc(cfg))   // the tensor-core kernel forms delta of its own rows as it starts
    return from_cuda(hga::launch_bwd_dq_tc(q, k_hist, v_hist, k_seg, v_seg, group_idx, lse, o, d_o,
                                           delta_of(workspace), dq, cfg->B, cfg->Hq, cfg->Hkv, cfg->hist_len,
                                           cfg->seg_len, hist_rows(cfg), cfg->top_groups, sink_groups(cfg),
                                           eff_scale(cfg), status_of(workspace), wait_limit(cfg), st));
  if ((rc = hga_attn_bwd_preprocess(cfg, o, d_o, workspace, stream))) return rc;
  return from_cuda(hga::launch_bwd_dq_simt(cfg->dtype == HGA_BF16, q, k_hist, v_hist, k_seg, v_seg, group_idx, lse,
                                           d_o, delta_of(workspace), dq, cfg->B, cfg->Hq, cfg->Hkv, cfg->hist_len,
                                           cfg->seg_len, hist_rows(cfg), cfg->top_groups, sink_groups(cfg),
                                           eff_scale(cfg), status_of(workspace), st));
}

int hga_attn_bwd(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist, const void* k_seg,
                 const void* v_seg, const int32_t* group_idx, const void* o, const float* lse, const void* d_o,
                 void* dq, void* dk_seg, void* dv_seg, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  return hga_internal_attn_bwd_ws(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, dk_seg, dv_seg,
                                  workspace, full_workspace_bytes(cfg), stream);
}

int hga_tier_cache_config(const hga_config_t* cfg, hga_config_t* cache_cfg) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!cache_cfg) return HGA_ERR_ARG;
  *cache_cfg = *cfg;
  cache_cfg->hist_len = tier_cap_groups(cfg) * cfg->group;
  cache_cfg->hist_capacity = 0;
  cache_cfg->top_chunks = (cfg->top_groups + (cfg->chunk / cfg->group) - 1) / (cfg->chunk / cfg->group);
  return check_config(cache_cfg);
}

int hga_tier_plan(const hga_config_t* cfg, const int32_t* group_idx, int32_t* used_groups, int32_t* n_used,
                  int32_t* compact_idx, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_idx({group_idx, used_groups, n_used, compact_idx}))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  const int64_t ngr = cfg->hist_len / cfg->group;
  if (hga::tier_plan_smem_bytes((int)ngr) > 200 * 1024) return HGA_ERR_UNSUPPORTED;
  return from_cuda(hga::launch_tier_plan(group_idx, cfg->B * cfg->Hkv, (int)(cfg->seg_len / cfg->qblock),
                                         cfg->top_groups, sink_groups(cfg), (int)ngr, (int)tier_cap_groups(cfg),
                                         used_groups, n_used, compact_idx, status_of(workspace),
                                         static_cast<cudaStream_t>(stream)));
}

int hga_tier_gather(const hga_config_t* cfg, const void* k_hist, const void* v_hist, const int32_t* used_groups,
                    const int32_t* n_used, void* k_cache, void* v_cache, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({k_hist, v_hist, k_cache, v_cache}))) return rc;
  if ((rc = check_idx({used_groups, n_used}))) return rc;
  const size_t esz = cfg->dtype == HGA_BF16 ? 2 : 4;
  const size_t hist_bytes = (size_t)cfg->B * cfg->Hkv * hist_rows(cfg) * cfg->D * esz;
  const void* kh = device_view(k_hist, hist_bytes);
  const void* vh = device_view(v_hist, hist_bytes);
  if (!kh || !vh) return HGA_ERR_ARG;        // pageable host memory cannot be read by the device
  return from_cuda(hga::launch_tier_gather(cfg->dtype == HGA_BF16, kh, vh, used_groups, n_used, cfg->B * cfg->Hkv,
                                           hist_rows(cfg), (int)tier_cap_groups(cfg), k_cache, v_cache,
                                           static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- group-summary cache
namespace {
constexpr int kMaxCacheSlots = 4096;

// cap_chunks: slots per (batch, KV head), 1 .. min(4096, the history's capacity in chunks).
int check_cache(const hga_config_t* c, int32_t cap) {
  const int64_t nchs = hist_rows(c) / c->chunk;
  if (cap < 1 || cap > kMaxCacheSlots || cap > nchs) return HGA_ERR_ARG;
  if (hga::gcache_plan_smem_bytes((int)nchs, cap) > 200 * 1024) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}
}  // namespace

int hga_route_chunks(const hga_config_t* cfg, const void* q, const float* chunk_sum, int32_t* chunk_idx, float* qb,
                     void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_ptrs({q, chunk_sum}))) return rc;
  (void)workspace;
  if (cfg->hist_len == 0) return HGA_OK;        // nothing to route
  if ((rc = check_idx({chunk_idx}))) return rc;
  if ((rc = check_ptrs({qb}))) return rc;
  return from_cuda(hga::launch_route_chunks(cfg->dtype == HGA_BF16, q, nullptr, false, chunk_sum, chunk_idx, qb,
                                            cfg->B, cfg->Hq, cfg->Hkv, cfg->seg_len, (int)(cfg->hist_len / cfg->chunk),
                                            (int)(hist_rows(cfg) / cfg->chunk), (int)(cfg->n_sink_tokens / cfg->chunk),
                                            cfg->top_chunks, static_cast<cudaStream_t>(stream)));
}

int hga_gcache_plan(const hga_config_t* cfg, int32_t cap_chunks, const int32_t* chunk_idx, int32_t* slot_of,
                    int32_t* chunk_of, int32_t* stamp, int32_t step, int32_t* miss_chunk, int32_t* miss_slot,
                    int32_t* counts, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (cfg->hist_len == 0) return HGA_OK;
  if ((rc = check_cache(cfg, cap_chunks))) return rc;
  if ((rc = check_idx({chunk_idx, slot_of, chunk_of, stamp, miss_chunk, miss_slot, counts}))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  return from_cuda(hga::launch_gcache_plan(chunk_idx, cfg->B * cfg->Hkv,
                                           (int)(cfg->seg_len / cfg->qblock) * cfg->top_chunks,
                                           (int)(hist_rows(cfg) / cfg->chunk), cap_chunks, step, slot_of, chunk_of,
                                           stamp, miss_chunk, miss_slot, counts, status_of(workspace),
                                           static_cast<cudaStream_t>(stream)));
}

int hga_gcache_fetch(const hga_config_t* cfg, int32_t cap_chunks, const float* group_sum_src, const int32_t* miss_chunk,
                     const int32_t* miss_slot, const int32_t* counts, float* gcache, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (cfg->hist_len == 0) return HGA_OK;
  if ((rc = check_cache(cfg, cap_chunks))) return rc;
  if ((rc = check_ptrs({group_sum_src, gcache}))) return rc;
  if ((rc = check_idx({miss_chunk, miss_slot, counts}))) return rc;
  const size_t bytes = (size_t)cfg->B * cfg->Hkv * (hist_rows(cfg) / cfg->group) * cfg->D * sizeof(float);
  const void* src = device_view(group_sum_src, bytes);
  if (!src) return HGA_ERR_ARG;                 // pageable host memory cannot be read by the device
  return from_cuda(hga::launch_gcache_fetch(static_cast<const float*>(src), hist_rows(cfg) / cfg->group, miss_chunk,
                                            miss_slot, counts, cfg->B * cfg->Hkv, cap_chunks, gcache,
                                            static_cast<cudaStream_t>(stream)));
}

int hga_route_groups_cached(const hga_config_t* cfg, const float* qb, const int32_t* chunk_idx,
                            const int32_t* slot_of, int32_t cap_chunks, const float* gcache, int32_t* group_idx,
                            void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (cfg->hist_len == 0) return HGA_OK;
  if ((rc = check_cache(cfg, cap_chunks))) return rc;
  if ((rc = check_ptrs({qb, gcache}))) return rc;
  if ((rc = check_idx({chunk_idx, slot_of, group_idx}))) return rc;
  if (!workspace) return HGA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HGA_ERR_ALIGN;
  return from_cuda(hga::launch_route_groups_cached(qb, chunk_idx, slot_of, gcache, cap_chunks, group_idx, cfg->B,
                                                   cfg->Hkv, cfg->seg_len, (int)(hist_rows(cfg) / cfg->chunk),
                                                   cfg->top_chunks, cfg->top_groups, status_of(workspace),
                                                   static_cast<cudaStream_t>(stream)));
}

int hga_read_status(void* workspace, void* stream, int32_t* status_out) {
  if (!workspace || !status_out) return HGA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return HGA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(v), st) != cudaSuccess) return HGA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HGA_ERR_CUDA;
  *status_out = v;
  return HGA_OK;
}

}  // extern "C"
