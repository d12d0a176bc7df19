// Shared device/host helpers of the CUDA library (not used by the oracle).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/fsq.h"

namespace fsq {

// B200: 148 SMs.  Launch planning uses this constant so that workspace sizes
// depend only on the call's arguments (and can be computed without a device).
constexpr int kNumSMs = 148;

// 1/ln(2): scores are kept in the log2 domain so the softmax uses exp2.
constexpr float kLog2e = 1.4426950408889634f;

struct Thresholds {
  float th[15];
};

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(((uint32_t)v) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Nibble = number of thresholds at or below u (0..15); level = nibble - 8.
__device__ __forceinline__ uint32_t fsq_nibble(float u, const Thresholds &t) {
  uint32_t n = 0;
#pragma unroll
  for (int k = 0; k < 15; ++k) n += (u >= t.th[k]) ? 1u : 0u;
  return n;
}

// Workspace header: the device error word lives in the first 4 bytes.
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void record_error(uint32_t *err, int status) {
  atomicCAS(err, 0u, (uint32_t)(-status));
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace fsq
