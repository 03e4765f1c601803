// Shared device-side definitions for the libla2 kernels (one translation unit).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la2 {

// Device error word. The first bounded wait that gives up stores its code
// here; la2_check() reads and clears it. Value 0 means no error.
__device__ int g_error_code = 0;
__device__ int g_error_where = 0;

enum DeviceError : int {
  DEV_ERR_NONE = 0,
  DEV_ERR_TIMEOUT = 5,
};

__device__ __forceinline__ void record_error(int code, int where) {
  if (atomicCAS(&g_error_code, 0, code) == 0) g_error_where = where;
}

__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// Grouped K/V heads (GQA; MQA with one K/V head). With H query heads and
// Hkv = H / G K/V heads, query sequence bh = b*H + h reads K/V sequence
// b*Hkv + h/G. G = 1 is the plain layout (every query head has its own K/V).
__host__ __device__ __forceinline__ int64_t kv_seq(int64_t bh, int32_t H, int32_t G) {
  if (G <= 1) return bh;
  const int64_t b = bh / H;
  const int32_t h = static_cast<int32_t>(bh - b * H);
  return b * (H / G) + h / G;
}
// First query sequence of K/V sequence `kv` (the group is kv's G consecutive heads).
__host__ __device__ __forceinline__ int64_t q_seq0(int64_t kv, int32_t H, int32_t G) {
  if (G <= 1) return kv;
  const int32_t Hkv = H / G;
  const int64_t b = kv / Hkv;
  const int32_t j = static_cast<int32_t>(kv - b * Hkv);
  return b * H + static_cast<int64_t>(j) * G;
}

// Programmatic dependent launch: let the next kernel of the stream start its
// launch now (its CTAs still wait in pdl_wait for this grid), and wait until
// the previous kernel of the stream has completed and its memory is visible.
// Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kern` with programmatic stream serialization. Every kernel
// launched this way calls pdl_wait() before its first global-memory access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

}  // namespace la2
