// Backward entry point that allocates nothing: the scratch that hga_attn_bwd keeps in the
// caller's workspace (status word + delta rows) lives here in a fixed device array instead.
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "hga.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kScratchBytes = hga::kStatusBytes + (size_t)HGA_NOALLOC_MAX_ROWS * sizeof(float);

// One copy per GPU that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_bwd_scratch on the current device, looked up once per device.
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return HGA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HGA_OK;
}

}  // namespace

int hga_internal_attn_bwd_ws(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist,
                             const void* k_seg, const void* v_seg, const int32_t* group_idx, const void* o,
                             const float* lse, const void* d_o, void* dq, void* dk_seg, void* dv_seg, void* workspace,
                             size_t ws_bytes, void* stream);

extern "C" int hga_attn_bwd_noalloc(const hga_config_t* cfg, const void* q, const void* k_hist, const void* v_hist,
                                    const void* k_seg, const void* v_seg, const int32_t* group_idx, const void* o,
                                    const float* lse, const void* d_o, void* dq, void* dk_seg, void* dv_seg,
                                    void* stream) {
  size_t need = 0;
  int rc = hga_workspace_size(cfg, &need);   // validates cfg
  if (rc) return rc;
  if ((int64_t)cfg->B * cfg->Hq * cfg->seg_len > (int64_t)HGA_NOALLOC_MAX_ROWS) return HGA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  // the status word must start at zero; delta is fully rewritten by the first kernel
  if (cudaMemsetAsync(scratch, 0, hga::kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HGA_ERR_CUDA;
  // the fixed array holds the status word and B*Hq*S delta rows: the whole workspace of this problem
  return hga_internal_attn_bwd_ws(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, dk_seg, dv_seg,
                                  scratch, kScratchBytes, stream);
}
