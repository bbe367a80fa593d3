// Shared device/host helpers for libddt (status codes, bf16 conversion,
// ordered-float keys). Internal header: not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

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

}  // namespace ddt
