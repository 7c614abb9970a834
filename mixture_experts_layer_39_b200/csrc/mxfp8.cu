// MXFP8 blockwise quantisation: E4M3 elements, one E8M0 scale per 32
// consecutive elements.
//
// The pages only name the format ("MXFP8 for selected operations; the gain
// comes from the feed-forward network and expert data movement", Olmo-core 3
// introduction page, section 3).  The rule used is the OCP MX v1.0 one:
// scale exponent = floor(log2(amax)) - 8 (8 = largest E4M3 exponent),
// clamped to [-127, 127]; element = round-to-nearest-even(v / 2^e),
// saturated to +-448.  floor(log2(amax)) is read from the fp32 exponent
// field of amax (an fp32 subnormal amax gives the clamp value -127), and
// v / 2^e is an exact multiply by 2^-e, so the only rounding is the E4M3
// conversion (cvt with .satfinite through cuda_fp8.h).
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int mx_scale_exp(float amax) {
  const int field = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);
  const int e = field - 127 - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ float pow2_neg(int e) {  // 2^-e for e in [-127, 126]
  return __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// axis 1: one thread per 32-element block of a row.
__global__ void mx_rowwise_kernel(const uint4* __restrict__ in, int64_t rows, int64_t cols,
                                  uint4* __restrict__ q, uint8_t* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int64_t nblk = cols / 32;
  const int64_t total = rows * nblk;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __ldg(in + b * 4 + i);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * i + 0] = bf16_lo(w[i].x); v[8 * i + 1] = bf16_hi(w[i].x);
      v[8 * i + 2] = bf16_lo(w[i].y); v[8 * i + 3] = bf16_hi(w[i].y);
      v[8 * i + 4] = bf16_lo(w[i].z); v[8 * i + 5] = bf16_hi(w[i].z);
      v[8 * i + 6] = bf16_lo(w[i].w); v[8 * i + 7] = bf16_hi(w[i].w);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_scale_exp(amax);
    const float inv = pow2_neg(e);
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a = e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv);
      const uint32_t c = e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv);
      p[i] = a | (c << 16);
    }
    q[b * 2] = make_uint4(p[0], p[1], p[2], p[3]);
    q[b * 2 + 1] = make_uint4(p[4], p[5], p[6], p[7]);
    scales[b] = static_cast<uint8_t>(e + 127);
  }
}

// axis 0: one thread per (32-row block, pair of adjacent columns).  Scales go
// to [rows/32, cols] (scale_mode 0) or, for the GEMM operand layout, to
// [groups, cols, rows_per_group/32] (scale_mode 1: a column's scales along
// the contraction axis are contiguous inside each group of rows).
__global__ void mx_colwise_kernel(const uint32_t* __restrict__ in, int64_t rows, int64_t cols,
                                  uint16_t* __restrict__ q, uint8_t* __restrict__ scales,
                                  int scale_mode, int64_t rows_per_group) {
  pdl_wait();
  pdl_trigger();
  const int64_t cpairs = cols / 2;
  const int64_t total = (rows / 32) * cpairs;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rb = i / cpairs, cp = i - rb * cpairs;
    float a[32], b[32];
    float am0 = 0.f, am1 = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t w = __ldg(in + (rb * 32 + r) * cpairs + cp);
      a[r] = bf16_lo(w);
      b[r] = bf16_hi(w);
      am0 = fmaxf(am0, fabsf(a[r]));
      am1 = fmaxf(am1, fabsf(b[r]));
    }
    const int e0 = mx_scale_exp(am0), e1 = mx_scale_exp(am1);
    const float i0 = pow2_neg(e0), i1 = pow2_neg(e1);
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint16_t lo = e4m3x2(a[r] * i0, 0.f) & 0xFF;
      const uint16_t hi = e4m3x2(b[r] * i1, 0.f) & 0xFF;
      q[(rb * 32 + r) * cpairs + cp] = static_cast<uint16_t>(lo | (hi << 8));
    }
    if (scale_mode == 0) {
      reinterpret_cast<uint16_t*>(scales)[rb * cpairs + cp] =
          static_cast<uint16_t>((e0 + 127) | ((e1 + 127) << 8));
    } else {
      const int64_t bpg = rows_per_group / 32;  // scale blocks per group
      const int64_t g = rb / bpg, rl = rb - g * bpg;
      scales[(g * cols + 2 * cp) * bpg + rl] = static_cast<uint8_t>(e0 + 127);
      scales[(g * cols + 2 * cp + 1) * bpg + rl] = static_cast<uint8_t>(e1 + 127);
    }
  }
}

}  // namespace

cudaError_t launch_mxfp8_quantize(const __nv_bfloat16* in, int64_t rows, int64_t cols, int axis,
                                  uint8_t* q, uint8_t* scales, cudaStream_t st) {
  if (axis == 1) {
    const int64_t total = rows * (cols / 32);
    const unsigned grid = static_cast<unsigned>(ceil_div64(total, 256) < 65535 ? ceil_div64(total, 256) : 65535);
    (void)launch_pdl(mx_rowwise_kernel, grid, 256, 0, st, reinterpret_cast<const uint4*>(in), rows, cols,
                                            reinterpret_cast<uint4*>(q), scales);
  } else {
    const int64_t total = (rows / 32) * (cols / 2);
    const unsigned grid = static_cast<unsigned>(ceil_div64(total, 256) < 65535 ? ceil_div64(total, 256) : 65535);
    (void)launch_pdl(mx_colwise_kernel, grid, 256, 0, st, reinterpret_cast<const uint32_t*>(in), rows, cols,
                                            reinterpret_cast<uint16_t*>(q), scales, 0, rows);
  }
  return cudaGetLastError();
}

cudaError_t launch_mxfp8_quantize_cols_t(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                         int64_t rows_per_group, uint8_t* q, uint8_t* scales,
                                         cudaStream_t st) {
  const int64_t total = (rows / 32) * (cols / 2);
  const unsigned grid = static_cast<unsigned>(ceil_div64(total, 256) < 65535 ? ceil_div64(total, 256) : 65535);
  (void)launch_pdl(mx_colwise_kernel, grid, 256, 0, st, reinterpret_cast<const uint32_t*>(in), rows, cols,
                                          reinterpret_cast<uint16_t*>(q), scales, 1, rows_per_group);
  return cudaGetLastError();
}

}  // namespace moe
