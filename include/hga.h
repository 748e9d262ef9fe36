/*
 * hga.h -- C ABI of the B200 (sm_100a) library for routed Hierarchical Global
 * Attention (HGA): the attention step of one transformer layer over a
 * detached history plus an active, differentiable segment.
 *
 * Method: "Long-Context Fine-Tuning with Limited VRAM" (arXiv 2607.15105).
 *   - gist.science "Technical Summary", section 2.1 "Hierarchical Global
 *     Attention": chunk selection over per-chunk summaries, group selection
 *     inside the chosen chunks, exact-token attention over the selected
 *     groups only; routing runs without gradient.
 *   - same page, section 2.2: the history K/V are detached at the segment
 *     boundary (segment-wise backward), so only the active segment gets
 *     gradients.
 *   - pith.science review, Figure 1 / Figure 2 captions and the
 *     free-parameter ledger: 64-token chunks, 8-token groups, summaries for
 *     every closed chunk, routed tokens alongside the local window.
 *
 * Readings where the pages are silent (the same ones the test oracle takes):
 * a summary is the arithmetic mean of the keys it covers; the routing query
 * of a block is the mean of its queries over the block's positions and the
 * query heads of one KV head (one routing per batch x KV head x block); the
 * score is the raw dot product; only history chunks are routable; group
 * selection is one top-k over all groups of the chosen chunks; ties go to the
 * lower index; index lists are sorted ascending; the local window is the whole
 * causal prefix of the active segment; the fixed sink window (section 2.1,
 * "alongside fixed sink and local windows") is the first n_sink_tokens history
 * tokens, whole chunks, attended by every query and never routed; one softmax
 * spans sink, routed and local keys; softmax scale 1/sqrt(D) unless given.
 *
 * Conventions for every entry point
 *   - Memory: the caller allocates and owns every buffer, including the
 *     workspace.  All tensor pointers are DEVICE pointers, 16-byte aligned
 *     (int32 index arrays: 4-byte aligned; a 32-byte aligned dq lets the
 *     bf16 backward store whole 32-byte sectors, which is faster, and gives
 *     the same result), contiguous, head-major: q, o, d_o, dq: [B, Hq, S, D]; k/v history:
 *     [B, Hkv, H, D]; k/v segment, dk/dv segment: [B, Hkv, S, D].  Query head
 *     h uses KV head h / (Hq / Hkv).  Element type: float32 or bfloat16 as
 *     set by cfg->dtype (summaries, LSE are always float32; indices int32).
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).
 *     Every call only enqueues work and returns without synchronising.
 *   - Return value: HGA_OK, or a negative HGA_ERR_* code.  Argument checks
 *     happen before anything is launched; on an error nothing is launched
 *     and no output is touched.  HGA_ERR_CUDA reports a launch failure.
 *   - Workspace: at least hga_workspace_size() bytes of device memory, zero-
 *     filled once before its first use (cudaMemset).  Layout: a 256-byte
 *     sticky status word (must start at zero; read and cleared by
 *     hga_read_status()), then the backward's delta rows (B*Hq*S float32,
 *     written before they are read), then, only for the bf16 tensor-core path
 *     when B*Hkv*ceil(S/128) is below the GPU's SM count, an exchange area of
 *     128 KB per such (batch, KV head, 128-key tile) unit in which the dK/dV
 *     kernel's CTA pairs hand each other float32 row sums (written before they
 *     are read).  Kernels that wait on on-chip barriers give up after
 *     a bounded time and record HGA_ERR_TIMEOUT there instead of hanging; an
 *     attention kernel given a group index outside [0, H/8) reads that group
 *     as zeros (never out of bounds) and records HGA_ERR_ARG there; so does a
 *     routed index inside the sink window.
 *   - Aliasing: outputs must not overlap inputs or each other.
 *   - Thread safety: the library keeps no mutable host state; calls on
 *     different streams with different workspaces may run concurrently.
 */
#ifndef HGA_H_
#define HGA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HGA_VERSION 3

/* Symbols of the shared library (built with hidden default visibility). */
#if defined(__GNUC__)
#define HGA_API __attribute__((visibility("default")))
#else
#define HGA_API
#endif

enum hga_status {
  HGA_OK = 0,
  HGA_ERR_ARG = -1,         /* bad shape, budget or null pointer            */
  HGA_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned             */
  HGA_ERR_UNSUPPORTED = -3, /* valid for the method, not built (D != 128 ...) */
  HGA_ERR_CUDA = -4,        /* kernel launch failed                         */
  HGA_ERR_TIMEOUT = -5,     /* a device-side bounded wait expired           */
  HGA_ERR_WORKSPACE = -6,   /* workspace pointer missing                    */
  HGA_ERR_TOO_LARGE = -7    /* beyond the fixed scratch of hga_attn_bwd_noalloc */
};

enum hga_dtype { HGA_F32 = 0, HGA_BF16 = 1 };

/* Problem description.  chunk = 64, group = 8, qblock = 64 and D = 128 are
 * the only built values (pith.science free-parameter ledger: chunk 64,
 * group 8).  hist_len must be a multiple of chunk (only closed chunks exist),
 * seg_len a positive multiple of qblock.  hist_len = 0 (the first segment of a
 * sequence, no history yet) requires top_chunks = top_groups = n_sink_tokens
 * = 0: routing does nothing and attention covers the causal segment prefix
 * only; k_hist, v_hist and group_idx are then not read and may be NULL.
 * hist_capacity: rows per (batch, KV head) of the history buffers k_hist /
 * v_hist [B, Hkv, hist_capacity, D] and of the summary buffers [B, Hkv,
 * hist_capacity / group, D] and [B, Hkv, hist_capacity / chunk, D], of which
 * the first hist_len tokens are the history (0 = hist_len; otherwise a
 * multiple of chunk, >= hist_len): a history that grows segment by segment
 * lives in one allocation.
 * n_sink_tokens: 0 <= n_sink_tokens < hist_len, a multiple of chunk; the
 * first n_sink_tokens history tokens are attended by every query and their
 * chunks are not routable, so 1 <= top_chunks <= (hist_len - n_sink_tokens) /
 * chunk; 1 <= top_groups <= top_chunks * (chunk / group).  group_idx passed to
 * the attention calls holds routed groups only (all >= n_sink_tokens / group).
 * softmax_scale = 0 selects 1 / sqrt(D).
 * wait_limit_ns: how long a tensor-core kernel's on-chip pipeline wait may
 * last before the kernel gives up, records HGA_ERR_TIMEOUT in the status word,
 * lets its own copies and MMAs land, releases its tensor memory and returns
 * (its outputs are then undefined); 0 selects 2 s, negative is HGA_ERR_ARG.  A
 * limit below 1 ms makes those waits poll the clock on every try (used to
 * exercise the expiry path: a limit shorter than a tile load's latency makes
 * the call time out). */
typedef struct hga_config {
  int32_t B, Hq, Hkv, D;
  int64_t hist_len, seg_len;
  int32_t chunk, group, qblock;
  int32_t top_chunks, top_groups;
  int32_t n_sink_tokens;
  int32_t dtype;
  float softmax_scale;
  int64_t hist_capacity;
  int64_t wait_limit_ns;
} hga_config_t;

/* Bytes of workspace the calls below need for this configuration. */
HGA_API int hga_workspace_size(const hga_config_t* cfg, size_t* bytes_out);

/* Kernels that one hga_route or hga_route_causal call launches for this
 * configuration, given a workspace (with_workspace != 0) or not: 0 when
 * hist_len = 0; 3 with a workspace and at least 512 routable chunks (chunks
 * outside the sink window), as long as the S/64 block queries of a (batch, KV
 * head) fit in 200 KB of shared memory; else 1.  For counting launches (a CUDA
 * graph, a profiler's kernel filter); no device work. */
HGA_API int hga_route_launches(const hga_config_t* cfg, int with_workspace, int32_t* launches_out);

/* Summaries (Technical Summary 2.1, chunk and group selection; review,
 * Figure 1): group_sum[b,kh,j,:] = mean of history keys 8j..8j+7;
 * chunk_sum[b,kh,i,:] = mean of history keys 64i..64i+63.
 *   k_hist     [B, Hkv, H, D]        cfg->dtype        (in)
 *   group_sum  [B, Hkv, H/8, D]      float32           (out)
 *   chunk_sum  [B, Hkv, H/64, D]     float32           (out) */
HGA_API int hga_build_summaries(const hga_config_t* cfg, const void* k_hist, float* group_sum,
                        float* chunk_sum, void* workspace, void* stream);

/* As hga_build_summaries for the chunks of history tokens [first_token,
 * hist_len) only (first_token a multiple of chunk): at a segment boundary the
 * closed segment's keys are appended to the history and only their summaries
 * are computed; every summary depends on its own keys only, so the result
 * equals a full rebuild bit for bit. */
HGA_API int hga_append_summaries(const hga_config_t* cfg, const void* k_hist, float* group_sum,
                                 float* chunk_sum, int64_t first_token, void* workspace,
                                 void* stream);

/* Two-level routing (Technical Summary 2.1): for each (b, kv head kh, block
 * n) the block query qb = mean of q over the block's 64 positions and the
 * query heads of kh; chunk scores qb . chunk_sum over all history chunks,
 * keep the top_chunks best; group scores qb . group_sum over the 8 groups of
 * each kept chunk, keep the top_groups best.  Scores in float32; ties to
 * the lower index; both lists written sorted ascending.  No gradient.
 *   q          [B, Hq, S, D]               cfg->dtype  (in)
 *   group_sum, chunk_sum                   float32     (in, from above)
 *   chunk_idx  [B, Hkv, S/64, top_chunks]  int32       (out)
 *   group_idx  [B, Hkv, S/64, top_groups]  int32       (out)
 *   workspace  hga_workspace_size(cfg) bytes, 16-byte aligned, or NULL.
 * With a workspace and a long history (hga_route_launches) the routing runs in
 * three launches: the block queries; every chunk summary of a (batch, KV head)
 * scored against all of its block queries in one pass (each summary read once
 * per (batch, KV head), not once per block); then each block's selection and
 * the group level.  The scores come from the same float32 operations in the
 * same order as in the single launch, so the indices are the same bit for bit.
 * The scratch shares the workspace region of the backward's dK/dV exchange
 * area: the routing and a backward call must not run at the same time on one
 * workspace.  Without a workspace: one launch. */
HGA_API int hga_route(const hga_config_t* cfg, const void* q, const float* group_sum,
              const float* chunk_sum, int32_t* chunk_idx, int32_t* group_idx,
              void* workspace, void* stream);

/* Strictly causal routing: as hga_route, except that block n is routed with the
 * block query of block n-1 (block 0 with that of q_prev, the previous segment's
 * last query block [B, Hq, qblock, D], same dtype; q_prev = NULL routes block 0
 * with a zero query, so ties give it the lowest routable indices).  The routing of
 * block n then depends on no token at or after the start of block n, which closes
 * the within-block side channel ("Technical Summary" section 5, "Causal Leakage":
 * a strictly causal variant is named there as future work).  The attention calls
 * are unchanged. */
HGA_API int hga_route_causal(const hga_config_t* cfg, const void* q, const void* q_prev,
                             const float* group_sum, const float* chunk_sum, int32_t* chunk_idx,
                             int32_t* group_idx, void* workspace, void* stream);

/* Forward (Technical Summary 2.1 "Exact-Token Attention"; review Figure 2):
 * query (b, h, t) of block n = t/64 attends to the exact history tokens
 * 8j..8j+7 of every j in group_idx[b, h/G, n, :] and to the segment tokens
 * 0..t, with one softmax over both sets:
 *   o = softmax(scale * q K^T) V,   lse = log sum exp(scale * q K^T).
 *   q [B,Hq,S,D]; k_hist, v_hist [B,Hkv,H,D]; k_seg, v_seg [B,Hkv,S,D]
 *   group_idx [B,Hkv,S/64,top_groups] int32, entries in [0, H/8)
 *   o [B,Hq,S,D] (cfg->dtype, out); lse [B,Hq,S] float32 (out, natural log) */
HGA_API int hga_attn_fwd(const hga_config_t* cfg, const void* q, const void* k_hist,
                 const void* v_hist, const void* k_seg, const void* v_seg,
                 const int32_t* group_idx, void* o, float* lse, void* workspace,
                 void* stream);

/* Backward of the forward above for L with dL/do = d_o (Technical Summary
 * 2.1: routing has no gradient; 2.2: history detached).  Produces
 *   dq over routed and local keys; dk_seg, dv_seg from the local (segment)
 *   pairs only, summed over the G query heads of each KV head.
 * No gradient is produced for k_hist / v_hist.  o and lse are the forward's
 * outputs.  dq [B,Hq,S,D], dk_seg, dv_seg [B,Hkv,S,D] in cfg->dtype (out).
 * Uses the workspace scratch described above (delta, dK/dV exchange area). */
HGA_API int hga_attn_bwd(const hga_config_t* cfg, const void* q, const void* k_hist,
                 const void* v_hist, const void* k_seg, const void* v_seg,
                 const int32_t* group_idx, const void* o, const float* lse,
                 const void* d_o, void* dq, void* dk_seg, void* dv_seg, void* workspace,
                 void* stream);

/* The steps of hga_attn_bwd as separate calls, on one stream and one workspace
 * (the same computation):
 *   preprocess: delta[b,h,t] = sum_d d_o * o  -> workspace scratch
 *               (the FlashAttention-form backward the pages cite);
 *   dq:         dq over routed and local keys; it also forms delta itself and
 *               leaves it in the workspace (so dq then dkdv needs no
 *               preprocess -- that is the order hga_attn_bwd uses);
 *   dkdv:       dk_seg, dv_seg from the local causal pairs (needs delta: from
 *               preprocess or from an earlier dq on the same workspace).
 * Arguments as for hga_attn_bwd. */
HGA_API int hga_attn_bwd_preprocess(const hga_config_t* cfg, const void* o, const void* d_o,
                                    void* workspace, void* stream);
HGA_API int hga_attn_bwd_dkdv(const hga_config_t* cfg, const void* q, const void* k_seg,
                              const void* v_seg, const float* lse, const void* d_o,
                              void* dk_seg, void* dv_seg, void* workspace, void* stream);
HGA_API int hga_attn_bwd_dq(const hga_config_t* cfg, const void* q, const void* k_hist,
                            const void* v_hist, const void* k_seg, const void* v_seg,
                            const int32_t* group_idx, const void* o, const float* lse,
                            const void* d_o, void* dq, void* workspace, void* stream);

/* Backward without any allocation: the same computation and kernels as
 * hga_attn_bwd, for callers that cannot allocate device memory -- e.g. a host
 * runtime that has handed the whole device to its own memory pool, or code that
 * must not call cudaMalloc/cudaFree because those may synchronise the device.
 * The paper has no counterpart of this entry point; it exists for such callers.
 *
 * Scratch: instead of a caller workspace it uses one fixed device array of
 * 256 + 4 * HGA_NOALLOC_MAX_ROWS bytes (4 MiB + 256 B) that every GPU loading
 * the library holds until the process exits.  Of it this entry uses the status
 * word and the B*Hq*S delta rows only; there is no dK/dV exchange area, so the
 * dK/dV kernel always runs with unpaired CTAs here (same result up to float32
 * summation order, slower when B*Hkv*ceil(S/128) is below the SM count).
 * B * Hq * S must not exceed HGA_NOALLOC_MAX_ROWS, else HGA_ERR_TOO_LARGE is
 * returned and nothing runs.
 * The array's device address is looked up with the device current on the
 * first call in each CUDA context of a device (the first call on a device, and
 * the first after cudaDeviceReset); make that call before any stream capture.
 * Every call clears the array's status word and overwrites the rest, and all
 * calls share it: calls that overlap on the GPU (other streams, other threads)
 * race and corrupt each other's results -- serialise them.  The device-side
 * status of the last call (HGA_ERR_TIMEOUT, HGA_ERR_ARG, see Workspace above)
 * stays in the array's status word: read it with hga_noalloc_read_status.
 * Arguments as for hga_attn_bwd, without workspace. */
#define HGA_NOALLOC_MAX_ROWS (1 << 20)
HGA_API int hga_attn_bwd_noalloc(const hga_config_t* cfg, const void* q, const void* k_hist,
                                 const void* v_hist, const void* k_seg, const void* v_seg,
                                 const int32_t* group_idx, const void* o, const float* lse,
                                 const void* d_o, void* dq, void* dk_seg, void* dv_seg,
                                 void* stream);

/* As hga_read_status for the fixed scratch array of hga_attn_bwd_noalloc on the
 * current device: synchronises `stream`, copies the array's status word (the
 * device-side status of the last hga_attn_bwd_noalloc call on this device) to
 * *status_out and clears it.  Allocates nothing.  The paper has no counterpart
 * of this entry point either. */
HGA_API int hga_noalloc_read_status(void* stream, int32_t* status_out);

/* ---------------------------------------------------------------- tiered history
 * Tiered storage ("Technical Summary" 2.2, "Tiered Memory Hierarchy"; pith.science
 * review, Figure 2 caption): the detached history K/V stay in host memory, the
 * summaries in device memory, and a layer step brings into device memory only the
 * exact K/V of the groups its routing selected.  Per step, after hga_route:
 *   1. hga_tier_plan: per (batch, KV head) the ascending list of every history group
 *      any block routed to (sink groups included), and each block's routed indices
 *      rewritten as positions in that list;
 *   2. hga_tier_gather: those groups' K/V rows copied from the history into a
 *      compact cache [B, Hkv, cap*8, D] in device memory;
 *   3. hga_attn_fwd / hga_attn_bwd with the configuration from
 *      hga_tier_cache_config, the cache as k_hist / v_hist and the rewritten
 *      indices as group_idx.  Positions keep the order of the group indices, so
 *      the results equal those over the full history bit for bit.
 * The cache holds cap groups per (batch, KV head): cap = min(H/8, sink groups +
 * (S/64) * top_groups), raised to at least the sink plus ceil(top_groups/8)
 * chunks, rounded up to whole chunks (cache_cfg->hist_len = 8 * cap). */

/* *cache_cfg = cfg with hist_len = 8 * cap and top_chunks = ceil(top_groups / 8):
 * the configuration of the attention calls over the compact cache. */
HGA_API int hga_tier_cache_config(const hga_config_t* cfg, hga_config_t* cache_cfg);

/* group_idx [B, Hkv, S/64, top_groups] (device, from hga_route with cfg) ->
 * used_groups [B, Hkv, cap] (ascending; entries past n_used unspecified),
 * n_used [B*Hkv], compact_idx [B, Hkv, S/64, top_groups] (all device int32).
 * A routed index outside [n_sink_tokens/8, H/8) is left out of the list, maps to
 * position 0 and records HGA_ERR_ARG in the workspace status word.  Asynchronous
 * on `stream`; needs the workspace only for its status word. */
HGA_API int hga_tier_plan(const hga_config_t* cfg, const int32_t* group_idx,
                          int32_t* used_groups, int32_t* n_used, int32_t* compact_idx,
                          void* workspace, void* stream);

/* Copies the K and V rows of used_groups[b, kh, 0 .. n_used) from k_hist / v_hist
 * [B, Hkv, H, D] into k_cache / v_cache [B, Hkv, cap*8, D] (device), group
 * position p to cache rows 8p .. 8p+7.  k_hist / v_hist may be device memory or
 * pinned host memory mapped into the device address space (cudaHostAlloc, or
 * cudaHostRegister with cudaHostRegisterMapped): the SMs read it over the host
 * link.  Pageable host memory is rejected with HGA_ERR_ARG before any launch (the
 * device cannot read it).  Cache rows past 8 * n_used are not written.
 * Asynchronous on `stream`: a side stream lets the copy of one batch element
 * overlap the attention of another. */
HGA_API int hga_tier_gather(const hga_config_t* cfg, const void* k_hist, const void* v_hist,
                            const int32_t* used_groups, const int32_t* n_used, void* k_cache,
                            void* v_cache, void* stream);

/* ---------------------------------------------------------------- group-summary cache
 * The middle tier of the tiered storage ("Technical Summary" 2.1 "Group Selection":
 * group summaries are cached in device memory and the missing ones are fetched from
 * host memory; 2.2: the chunk summaries stay resident; pith.science review, Figure 1
 * caption): routing in two levels with the group summaries of a long history in host
 * memory and a device cache of cap_chunks slots per (batch, KV head), each slot
 * holding the 8 group summaries (8 x D float32, 4 KB) of one chunk.  Per step:
 *   1. hga_route_chunks: level 1 -> chunk_idx, and the block queries qb;
 *   2. hga_gcache_plan: hits refresh their slots; the chosen chunks without a slot take
 *      the least recently used slots holding no chosen chunk; writes the miss list;
 *   3. hga_gcache_fetch: copies the missed chunks' group summaries into their slots;
 *   4. hga_route_groups_cached: level 2 from the slots -> group_idx.
 * The summaries are the same float32 values, so chunk_idx and group_idx equal those of
 * hga_route bit for bit.  A cache of at least min(chunks outside the sink, (S/64) *
 * top_chunks) slots always holds a step's chosen chunks; a smaller one records
 * HGA_ERR_ARG in the workspace status word when a step needs more.
 * Cache state (device int32, owned by the caller, initialised once to -1 everywhere):
 *   slot_of  [B, Hkv, hist_capacity/64]  slot of each chunk (-1: not cached)
 *   chunk_of [B, Hkv, cap_chunks]        chunk held by each slot (-1: empty)
 *   stamp    [B, Hkv, cap_chunks]        step that last used each slot (-1: never)
 * Per-step buffers (device int32): miss_chunk, miss_slot [B, Hkv, cap_chunks];
 * counts [B*Hkv, 2] = (hits, misses) of the step.  qb [B, Hkv, S/64, D] float32;
 * gcache [B, Hkv, cap_chunks, 8, D] float32.  1 <= cap_chunks <= 4096. */

/* Level 1 of hga_route (chunk selection) only: chunk_idx as hga_route writes it, and
 * the block query of every (batch, KV head, block) into qb. */
HGA_API int hga_route_chunks(const hga_config_t* cfg, const void* q, const float* chunk_sum,
                             int32_t* chunk_idx, float* qb, void* workspace, void* stream);

/* The cache plan of one step (`step` increases by one per step and is stored in the
 * stamps).  Needs the workspace for its status word. */
HGA_API int hga_gcache_plan(const hga_config_t* cfg, int32_t cap_chunks, const int32_t* chunk_idx,
                            int32_t* slot_of, int32_t* chunk_of, int32_t* stamp, int32_t step,
                            int32_t* miss_chunk, int32_t* miss_slot, int32_t* counts,
                            void* workspace, void* stream);

/* Copies the 8 group summaries of every missed chunk from group_sum_src [B, Hkv,
 * hist_capacity/8, D] float32 -- pinned host memory mapped into the device address space
 * (the SMs read it over the host link) or device memory; pageable host memory is
 * rejected with HGA_ERR_ARG -- into their slots of gcache. */
HGA_API int hga_gcache_fetch(const hga_config_t* cfg, int32_t cap_chunks, const float* group_sum_src,
                             const int32_t* miss_chunk, const int32_t* miss_slot, const int32_t* counts,
                             float* gcache, void* stream);

/* Level 2 of hga_route (group selection) from the cache: group_idx as hga_route writes
 * it, from qb and chunk_idx of hga_route_chunks and the group summaries in gcache.  A
 * chosen chunk without a slot records HGA_ERR_ARG in the workspace status word. */
HGA_API int hga_route_groups_cached(const hga_config_t* cfg, const float* qb, const int32_t* chunk_idx,
                                    const int32_t* slot_of, int32_t cap_chunks, const float* gcache,
                                    int32_t* group_idx, void* workspace, void* stream);

/* Synchronises `stream`, copies the workspace status word to *status_out
 * (HGA_OK, HGA_ERR_TIMEOUT or HGA_ERR_ARG, see Workspace above) and clears it.  Returns HGA_ERR_CUDA if the
 * copy itself fails. */
HGA_API int hga_read_status(void* workspace, void* stream, int32_t* status_out);

/* Static text for a status code. */
HGA_API const char* hga_strerror(int code);

/* HGA_VERSION of the built library. */
HGA_API int hga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H_ */
