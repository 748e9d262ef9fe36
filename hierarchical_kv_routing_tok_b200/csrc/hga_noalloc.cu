// Backward entry point that allocates nothing: the scratch that hga_attn_bwd keeps in the
// caller's workspace (status word + delta rows) lives here in a fixed device array instead.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "hga.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kScratchBytes = hga::kStatusBytes + (size_t)HGA_NOALLOC_MAX_ROWS * sizeof(float);

// One copy per GPU that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

// Device address of g_bwd_scratch per device, with the id of the context it was looked up in: a
// new context on the device (after cudaDeviceReset the runtime makes a new primary context and
// loads the module again) has its own copy of the array, so the address is looked up again.
struct Cached {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_mu;
Cached g_cache[kMaxDevices] = {};

// Driver entry points, resolved through the runtime (the library does not link libcuda itself).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
template <typename F>
F driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(ptr);
}

// Device address of g_bwd_scratch in the current device's current context.
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return HGA_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return HGA_ERR_CUDA;
  if (!ctx) {
    // no context current on this thread yet: a runtime call on the device makes its primary
    // context current (the symbol lookup does, and allocates nothing)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess) return HGA_ERR_CUDA;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return HGA_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return HGA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_cache[dev].ptr || g_cache[dev].ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return HGA_ERR_CUDA;
    g_cache[dev] = Cached{id, p};
  }
  *out = g_cache[dev].ptr;
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
  const int64_t rows = (int64_t)cfg->B * cfg->Hq * cfg->seg_len;
  if (rows > (int64_t)HGA_NOALLOC_MAX_ROWS) return HGA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  // the status word must start at zero; delta is fully rewritten by the first kernel
  if (cudaMemsetAsync(scratch, 0, hga::kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HGA_ERR_CUDA;
  // the array serves as a workspace of exactly the status word and this problem's delta rows: it has
  // no dK/dV exchange area, so the dK/dV kernel never pairs CTAs through this entry (whatever room
  // the rest of the array would leave)
  const size_t ws_bytes = hga::kStatusBytes + (((size_t)rows * sizeof(float) + 255) & ~(size_t)255);
  return hga_internal_attn_bwd_ws(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, dk_seg, dv_seg,
                                  scratch, ws_bytes, stream);
}

extern "C" int hga_noalloc_read_status(void* stream, int32_t* status_out) {
  if (!status_out) return HGA_ERR_ARG;
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  return hga_read_status(scratch, stream, status_out);
}
