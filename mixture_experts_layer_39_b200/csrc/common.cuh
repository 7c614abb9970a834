// Shared device helpers for the MoE expert-layer kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Segments of the routed-row space start at multiples of this many rows
// (bf16 operands), or of kSegAlignMx rows when the expert GEMMs run in MXFP8
// (so every 32-token scale block and every 128-token K-block of the weight
// gradients lies inside one expert).
constexpr int kSegAlign = 32;
constexpr int kSegAlignMx = 128;

struct DeviceCtl {
  int status;  // first recorded moe_status_t code, 0 when clean
  int detail;  // kernel-specific detail of the first error (which wait, which index)
};

__device__ __forceinline__ void report(DeviceCtl* ctl, int code, int detail) {
  if (ctl == nullptr) return;
  if (atomicCAS(&ctl->status, 0, code) == 0) atomicExch(&ctl->detail, detail);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two fp32 -> packed bf16x2 (round to nearest even), low half = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace moe
