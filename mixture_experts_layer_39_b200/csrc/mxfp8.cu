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

#include <type_traits>

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

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t v) {
  __nv_bfloat162 r;
  memcpy(&r, &v, sizeof(r));
  return r;
}

__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) {
  uint32_t r;
  memcpy(&r, &v, sizeof(r));
  return r;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Byte of the scale of (MN index r, 32-element contraction block kb) in the
// tensor cores' scale-atom order: atoms of 512 bytes for 128 MN indices x 4
// blocks (128 contraction elements), atom (r/128, kb/4) at index
// (r/128) * n_kb4 + kb/4 (n_kb4 = contraction length / 128), and inside an
// atom byte (r%32)*16 + ((r/32)%4)*4 + kb%4.  The GEMMs copy one atom per
// stage with one TMA load and hand it to tcgen05.cp unchanged.
__device__ __forceinline__ int64_t atom_byte(int64_t r, int64_t kb, int64_t n_kb4) {
  return ((r >> 7) * n_kb4 + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

// axis 1: one thread per 32-element block of a row.  Scales go to
// [rows, cols/32] (atoms = false) or, for the GEMM operands, in atom order
// (atoms = true; rows and cols multiples of 128).
__global__ void mx_rowwise_kernel(const uint4* __restrict__ in, int64_t rows, int64_t cols,
                                  uint4* __restrict__ q, uint8_t* __restrict__ scales,
                                  bool atoms) {
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
    if (atoms) {
      const int64_t r = b / nblk;
      scales[atom_byte(r, b - r * nblk, nblk >> 2)] = static_cast<uint8_t>(e + 127);
    } else {
      scales[b] = static_cast<uint8_t>(e + 127);
    }
  }
}

// axis 0: one thread per (32-row block, W adjacent columns), W = 4 where the
// row width and the buffers' alignment allow 8-byte loads, else 2.  Each row
// of the block is one vector load and one vector store of W codes; the two
// columns of a bf16 pair are converted by one paired E4M3 conversion (each
// element rounds on its own, so pairing changes no code).  Scales go to
// [rows/32, cols].
template <int W>
__global__ void mx_colwise_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows, int64_t cols,
                                  uint8_t* __restrict__ q, uint8_t* __restrict__ scales) {
  static_assert(W == 2 || W == 4, "two or four columns per thread");
  constexpr int NP = W / 2;  // bf16 pairs per row slice
  using In = typename std::conditional<NP == 2, uint2, uint32_t>::type;
  using Out = typename std::conditional<NP == 2, uint32_t, uint16_t>::type;
  pdl_wait();
  pdl_trigger();
  const int64_t cgroups = cols / W;
  const int64_t total = (rows / 32) * cgroups;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rb = i / cgroups, cg = i - rb * cgroups;
    const In* src = reinterpret_cast<const In*>(in) + rb * 32 * cgroups + cg;
    uint32_t w[32][NP];
#pragma unroll
    for (int r = 0; r < 32; ++r, src += cgroups) {
      const In v = __ldg(src);
      if constexpr (NP == 2) {
        w[r][0] = v.x;
        w[r][1] = v.y;
      } else {
        w[r][0] = v;
      }
    }
    // amax on the packed pairs: a max is exact in bf16, and like fmaxf
    // __hmax2 returns the other operand when one is NaN.
    __nv_bfloat162 m[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) m[j] = __float2bfloat162_rn(0.f);
#pragma unroll
    for (int r = 0; r < 32; ++r)
#pragma unroll
      for (int j = 0; j < NP; ++j) m[j] = __hmax2(m[j], __habs2(as_bf162(w[r][j])));
    int e[W];
    float inv[W];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      const uint32_t mb = as_u32(m[j]);
      e[2 * j] = mx_scale_exp(bf16_lo(mb));
      e[2 * j + 1] = mx_scale_exp(bf16_hi(mb));
    }
#pragma unroll
    for (int c = 0; c < W; ++c) inv[c] = pow2_neg(e[c]);
    Out* dst = reinterpret_cast<Out*>(q) + rb * 32 * cgroups + cg;
#pragma unroll
    for (int r = 0; r < 32; ++r, dst += cgroups) {
      uint32_t p = 0;
#pragma unroll
      for (int j = 0; j < NP; ++j)
        p |= static_cast<uint32_t>(e4m3x2(bf16_lo(w[r][j]) * inv[2 * j],
                                          bf16_hi(w[r][j]) * inv[2 * j + 1]))
             << (16 * j);
      *dst = static_cast<Out>(p);
    }
    uint32_t sc = 0;
#pragma unroll
    for (int c = 0; c < W; ++c) sc |= static_cast<uint32_t>(e[c] + 127) << (8 * c);
    reinterpret_cast<Out*>(scales)[rb * cgroups + cg] = static_cast<Out>(sc);
  }
}

// Both orientations of one operand in one pass (GEMM layouts, atom-ordered
// scales).  A block of 128 threads takes a tile of 32 rows x 128 columns:
// thread t loads 16 bytes (8 columns, c8 = t % 16) of rows t/16 + 8i,
// i = 0..3.
//   row-wise : blocks of 32 columns span 4 neighbouring lanes, whose maxima
//              meet by two shuffles; codes to q_row, scales along the row;
//   column-wise: the tile's 32 rows are one block of every column; each
//              thread's 4-row maxima meet in shared memory, thread t takes
//              column t's amax and writes its scale; codes to q_col.
// The tile's 32 rows never straddle a group (rows_per_group is a multiple of
// 128), so the column blocks of each group take their own run of atoms.
// Capped at 64 registers a thread, eight blocks (64 KB of loads in flight)
// fit on an SM, against five at the uncapped 92: 0.79 of the measured copy
// rate on operand-sized inputs, against 0.67.
__global__ void __launch_bounds__(128, 8)
    mx_both_kernel(const uint4* __restrict__ in, int64_t rows, int64_t cols, int64_t rows_per_group,
                   uint2* __restrict__ q_row, uint8_t* __restrict__ s_row, uint2* __restrict__ q_col,
                   uint8_t* __restrict__ s_col) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_part[8][128];
  __shared__ int s_ecol[128];
  const int t = threadIdx.x, c8 = t & 15, r0 = t >> 4;
  const int64_t tiles_c = cols / 128;
  const int64_t n_tiles = (rows / 32) * tiles_c;
  const int64_t vec_row = cols / 8;  // 16-byte vectors per row
  const int64_t n_kb4_row = cols / 128, bpg = rows_per_group / 32;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t tr = tile / tiles_c, tc = tile - tr * tiles_c;
    const int64_t row0 = tr * 32, col0 = tc * 128;
    float v[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w = __ldg(in + (row0 + r0 + 8 * i) * vec_row + (col0 >> 3) + c8);
      unpack8(w, v[i]);
    }
    // ---- row-wise: block (row, 32 columns) over lanes 4j..4j+3 of this row
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[i][j]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      const int e = mx_scale_exp(m);
      const float inv = pow2_neg(e);
      uint32_t p[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        p[h] = static_cast<uint32_t>(e4m3x2(v[i][4 * h] * inv, v[i][4 * h + 1] * inv)) |
               (static_cast<uint32_t>(e4m3x2(v[i][4 * h + 2] * inv, v[i][4 * h + 3] * inv)) << 16);
      const int64_t r = row0 + r0 + 8 * i;
      q_row[r * (cols / 8) + (col0 >> 3) + c8] = make_uint2(p[0], p[1]);
      if ((c8 & 3) == 0)
        s_row[atom_byte(r, (col0 >> 5) + (c8 >> 2), n_kb4_row)] = static_cast<uint8_t>(e + 127);
    }
    // ---- column-wise: the 32 rows of the tile are one block of each column
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) m = fmaxf(m, fabsf(v[i][j]));
      s_part[r0][8 * c8 + j] = m;
    }
    __syncthreads();
    {
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) m = fmaxf(m, s_part[k][t]);
      const int e = mx_scale_exp(m);
      s_ecol[t] = e;
      const int64_t g = row0 / rows_per_group, rl = (row0 - g * rows_per_group) >> 5;
      s_col[g * cols * bpg + atom_byte(col0 + t, rl, bpg >> 2)] = static_cast<uint8_t>(e + 127);
    }
    __syncthreads();
    float inv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) inv[j] = pow2_neg(s_ecol[8 * c8 + j]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t p[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        p[h] = static_cast<uint32_t>(e4m3x2(v[i][4 * h] * inv[4 * h], v[i][4 * h + 1] * inv[4 * h + 1])) |
               (static_cast<uint32_t>(e4m3x2(v[i][4 * h + 2] * inv[4 * h + 2],
                                             v[i][4 * h + 3] * inv[4 * h + 3])) << 16);
      q_col[(row0 + r0 + 8 * i) * (cols / 8) + (col0 >> 3) + c8] = make_uint2(p[0], p[1]);
    }
    __syncthreads();  // s_part / s_ecol are rewritten by the next tile
  }
}

// Picks four columns per thread when every vector access stays aligned.
cudaError_t launch_colwise(const __nv_bfloat16* in, int64_t rows, int64_t cols, uint8_t* q,
                           uint8_t* scales, cudaStream_t st) {
  const bool wide = cols % 4 == 0 && (reinterpret_cast<uintptr_t>(in) & 7) == 0 &&
                    (reinterpret_cast<uintptr_t>(q) & 3) == 0 &&
                    (reinterpret_cast<uintptr_t>(scales) & 3) == 0;
  const int64_t total = (rows / 32) * (cols / (wide ? 4 : 2));
  const unsigned grid = static_cast<unsigned>(ceil_div64(total, 256) < 65535 ? ceil_div64(total, 256) : 65535);
  if (wide)
    (void)launch_pdl(mx_colwise_kernel<4>, grid, 256, 0, st, in, rows, cols, q, scales);
  else
    (void)launch_pdl(mx_colwise_kernel<2>, grid, 256, 0, st, in, rows, cols, q, scales);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rowwise(const __nv_bfloat16* in, int64_t rows, int64_t cols, uint8_t* q,
                           uint8_t* scales, bool atoms, cudaStream_t st) {
  const int64_t total = rows * (cols / 32);
  const unsigned grid = static_cast<unsigned>(ceil_div64(total, 256) < 65535 ? ceil_div64(total, 256) : 65535);
  (void)launch_pdl(mx_rowwise_kernel, grid, 256, 0, st, reinterpret_cast<const uint4*>(in), rows,
                   cols, reinterpret_cast<uint4*>(q), scales, atoms);
  return cudaGetLastError();
}

cudaError_t launch_mxfp8_quantize(const __nv_bfloat16* in, int64_t rows, int64_t cols, int axis,
                                  uint8_t* q, uint8_t* scales, cudaStream_t st) {
  if (axis == 1) return launch_rowwise(in, rows, cols, q, scales, false, st);
  return launch_colwise(in, rows, cols, q, scales, st);
}

cudaError_t launch_mxfp8_quantize_atoms(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                        uint8_t* q, uint8_t* scales, cudaStream_t st) {
  return launch_rowwise(in, rows, cols, q, scales, true, st);
}

cudaError_t launch_mxfp8_quantize_both(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                       int64_t rows_per_group, uint8_t* q_row, uint8_t* s_row,
                                       uint8_t* q_col, uint8_t* s_col, int num_sms,
                                       cudaStream_t st) {
  // two waves of the eight resident blocks per SM, each block walking tiles
  const int64_t tiles = (rows / 32) * (cols / 128);
  const int64_t cap = static_cast<int64_t>(num_sms > 0 ? num_sms : 148) * 16;
  const unsigned grid = static_cast<unsigned>(tiles < cap ? (tiles > 0 ? tiles : 1) : cap);
  (void)launch_pdl(mx_both_kernel, grid, 128, 0, st, reinterpret_cast<const uint4*>(in), rows, cols,
                   rows_per_group, reinterpret_cast<uint2*>(q_row), s_row,
                   reinterpret_cast<uint2*>(q_col), s_col);
  return cudaGetLastError();
}

}  // namespace moe
