// Shared device/host helpers for libddt (status codes, bf16 conversion,
// ordered-float keys). Internal header: not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/ddt.h"

#define DDT_FULL_MASK 0xffffffffu

namespace ddt {

// Launch-error check used right after every kernel launch in the API layer.
inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t u) {
  return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Monotone map float -> uint32 (larger float => larger key); -0 maps like +0.
// Finite inputs only (NaN is a precondition violation upstream).
__device__ __forceinline__ uint32_t float_order_key(float x) {
  uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Host state the library keeps per device ordinal (below this bound).
constexpr int kMaxDevices = 128;

// Streaming multiprocessors of the current device, looked up once per device
// (148 on a B200; 148 also when the query fails).
inline int sm_count() {
  static std::mutex mu;
  static int counts[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (counts[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    counts[dev] = c;
  }
  return counts[dev];
}

// Wall-clock limit of every bounded wait inside a kernel, in nanoseconds
// (process-wide; read when a kernel is launched). ddt_set_wait_limit_ns sets it.
uint64_t wait_limit_ns();

// Programmatic dependent launch: a kernel launched with the PDL attribute may
// start while its predecessor on the stream is still running; it must wait
// before touching anything the predecessor writes. Both are no-ops without
// the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with the programmatic-stream-serialization attribute set.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
