// Device helpers shared by the HGA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace hga {

constexpr int kD = 128;       // head dimension built
constexpr int kChunk = 64;    // tokens per chunk
constexpr int kGroup = 8;     // tokens per group
constexpr int kQBlock = 64;   // queries per routing block
constexpr int kStatusBytes = 256;

// Load 4 consecutive elements as float4 (p is 8-byte aligned for bf16, 16 for f32).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float4 f;
  f.x = __uint_as_float(u.x << 16);
  f.y = __uint_as_float(u.x & 0xffff0000u);
  f.z = __uint_as_float(u.y << 16);
  f.w = __uint_as_float(u.y & 0xffff0000u);
  return f;
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// 16-byte vector of elements: 8 bf16 or 4 f32, expanded to floats.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization (see
// launch_dependent) may start while the kernel before it in the stream is still running: its CTAs
// take SMs as that kernel's CTAs leave them, once every CTA of that kernel has called pdl_trigger().
// Each of its threads must call pdl_wait() before reading anything an earlier kernel wrote; the
// wait returns once the kernel before has completed and its memory is visible (at once when the
// kernel was launched normally).  A kernel whose every CTA waits completes only after its
// predecessor, so the order of a whole chain of such launches is kept.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch `kernel` as a dependent of the previous kernel in `st` (programmatic stream
// serialization), optionally in clusters of `cluster` CTAs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                    unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  unsigned na = 0;
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = cluster;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Record a device-side failure code in the workspace status word (first one wins).
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// History group read by slot `slot` of a block's history key list: the nsg groups of the sink
// window (groups 0..nsg-1) come first, then the block's kg routed groups gi[0..kg).  Slots past the
// list (tile padding) read group 0.  A routed index outside [nsg, ngr) is never dereferenced: it
// records HGA_ERR_ARG (-1) in the status word and -1 is returned.
__device__ __forceinline__ int32_t routed_group(const int32_t* gi, int slot, int nsg, int kg, int64_t ngr,
                                                int* status) {
  if (slot < nsg) return slot;
  const int r = slot - nsg;
  if (r >= kg) return 0;
  const int32_t g = gi[r];
  if (g < nsg || (int64_t)g >= ngr) {
    set_status(status, -1);
    return -1;
  }
  return g;
}

}  // namespace hga
