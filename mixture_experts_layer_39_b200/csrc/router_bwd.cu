// Router backward: gradient through the selected softmax probabilities.
//
// The top-k choice is piecewise constant, so only the chosen probabilities
// carry gradient.  With g = d(loss)/d(gate weight) (adjusted for the
// optional renormalisation), dp[t, idx[t,j]] = g[t,j] and the softmax
// backward gives dL = p * (dp - <p, dp>).  Then
//   dX_router = dL W_r,  dW_r = dL^T x,  db = sum_t dL.
// For small E these run on CUDA cores; for E a multiple of 128 the two
// products run on the tcgen05 grouped GEMM (see gemm.cu) and this file only
// produces dL (bf16) and the db partial sums.
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

// NE: compile-time bound on E for the fused dX_router loop (E <= NE <= 32*NPL).
template <int NPL, bool FUSE_DX, int NE = 32 * NPL>
__global__ void __launch_bounds__(kWarps * 32)
    router_bwd_dl_kernel(const float* __restrict__ dw, const float* __restrict__ probs,
                         const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ w_r,
                         int T, int d, int E, int k, int renorm, float* __restrict__ dl_f32,
                         __nv_bfloat16* __restrict__ dl_bf16, float* __restrict__ dx_router,
                         float* __restrict__ db_partial, int stage_w) {
  __shared__ float s_db[kWarps][32 * NPL];
  extern __shared__ uint4 s_wdyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* s_w = nullptr;
  if constexpr (FUSE_DX) {
    if (stage_w) {  // W_r staged once per block
      const uint4* src = reinterpret_cast<const uint4*>(w_r);
      for (int i = threadIdx.x; i < E * (d >> 3); i += blockDim.x) s_wdyn[i] = __ldg(src + i);
      __syncthreads();
      s_w = s_wdyn;
    }
  }
  float db[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) db[i] = 0.f;
  const int nvec = d >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < T; t += stride) {
    int id[8];
    float g[8];
    float psel_sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      id[j] = j < k ? __ldg(idx + t * k + j) : -1;
      g[j] = j < k ? __ldg(dw + t * k + j) : 0.f;
      if (id[j] < 0 || id[j] >= E) id[j] = -1;
    }
    if (renorm) {
      float ps[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ps[j] = id[j] >= 0 ? __ldg(probs + t * E + id[j]) : 0.f;
        psel_sum += ps[j];
      }
      const float inv = 1.0f / psel_sum;
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) dot += g[j] * ps[j] * inv;
#pragma unroll
      for (int j = 0; j < 8; ++j) g[j] = (g[j] - dot) * inv;
    }
    float p[NPL], dp[NPL];
    float pdp = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      p[i] = e < E ? __ldg(probs + t * E + e) : 0.f;
      dp[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) if (id[j] == e) dp[i] += g[j];
      pdp += p[i] * dp[i];
    }
    pdp = warp_sum(pdp);
    float dl[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      dl[i] = p[i] * (dp[i] - pdp);
      if (e < E) {
        db[i] += dl[i];
        if (dl_f32 != nullptr) dl_f32[t * E + e] = dl[i];
        if (dl_bf16 != nullptr) dl_bf16[t * E + e] = __float2bfloat16_rn(dl[i]);
      }
    }
    if constexpr (FUSE_DX) {
      // dX_router[t, :] = sum_e dL[e] W_r[e, :]; every lane gets all of dL
      // once, then owns 8 columns per 256 (W_r from shared memory)
      float dle[NE];
#pragma unroll
      for (int e = 0; e < NE; ++e) dle[e] = __shfl_sync(0xffffffffu, dl[e >> 5], e & 31);
      const uint4* wv = s_w != nullptr ? s_w : reinterpret_cast<const uint4*>(w_r);
      float4* out = reinterpret_cast<float4*>(dx_router + t * d);
      for (int v = lane; v < nvec; v += 32) {
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          if (e < E) {
            const uint4 q = wv[static_cast<int64_t>(e) * nvec + v];
            const float g = dle[e];
            acc[0] = fmaf(g, bf16_lo(q.x), acc[0]); acc[1] = fmaf(g, bf16_hi(q.x), acc[1]);
            acc[2] = fmaf(g, bf16_lo(q.y), acc[2]); acc[3] = fmaf(g, bf16_hi(q.y), acc[3]);
            acc[4] = fmaf(g, bf16_lo(q.z), acc[4]); acc[5] = fmaf(g, bf16_hi(q.z), acc[5]);
            acc[6] = fmaf(g, bf16_lo(q.w), acc[6]); acc[7] = fmaf(g, bf16_hi(q.w), acc[7]);
          }
        }
        out[2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
  // per-block partial of db (fixed order: warps, then blocks in a later pass)
#pragma unroll
  for (int i = 0; i < NPL; ++i) s_db[warp][lane + 32 * i] = db[i];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kWarps * 32) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += s_db[w][e];
    db_partial[static_cast<int64_t>(blockIdx.x) * E + e] = s;
  }
}

// dW_r partial over a chunk of tokens, CUDA cores (E <= 64): each thread
// owns CPT consecutive columns and all E experts of them; blocks tile
// (column slice, token chunk).
constexpr int kChunk = 64;
constexpr int kDwThreads = 128;

template <int NE, int CPT>
__global__ void __launch_bounds__(kDwThreads)
    router_dw_small_kernel(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ x, int T,
                           int d, int E, float* __restrict__ partial) {
  __shared__ float s_dl[kChunk * NE];  // 16 KB at NE = 64
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kChunk;
  const int nt = T - t0 < kChunk ? static_cast<int>(T - t0) : kChunk;
  for (int i = threadIdx.x; i < nt * E; i += blockDim.x) {
    const int tt = i / E, e = i - tt * E;
    s_dl[tt * NE + e] = dl[(t0 + tt) * E + e];
  }
  __syncthreads();
  const int64_t col = (static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x) * CPT;
  if (col >= d) return;
  float acc[NE][CPT];
#pragma unroll
  for (int e = 0; e < NE; ++e)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[e][c] = 0.f;
#pragma unroll 4
  for (int tt = 0; tt < nt; ++tt) {
    float xv[CPT];
    const __nv_bfloat16* xr = x + (t0 + tt) * d + col;
    if constexpr (CPT == 4) {
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(xr));
      xv[0] = bf16_lo(q.x); xv[1] = bf16_hi(q.x); xv[2] = bf16_lo(q.y); xv[3] = bf16_hi(q.y);
    } else if constexpr (CPT == 2) {
      const uint32_t q = __ldg(reinterpret_cast<const unsigned int*>(xr));
      xv[0] = bf16_lo(q); xv[1] = bf16_hi(q);
    } else {
#pragma unroll
      for (int c = 0; c < CPT; ++c) xv[c] = __bfloat162float(xr[c]);
    }
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      if (e < E) {
        const float g = s_dl[tt * NE + e];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[e][c] = fmaf(g, xv[c], acc[e][c]);
      }
    }
  }
  float* out = partial + static_cast<int64_t>(blockIdx.y) * E * d;
#pragma unroll
  for (int e = 0; e < NE; ++e)
    if (e < E)
#pragma unroll
      for (int c = 0; c < CPT; ++c) out[static_cast<int64_t>(e) * d + col + c] = acc[e][c];
}

// out[i] = bf16(sum_p partial[p][i]).  A block owns 32 float4 columns; its
// 8 warps take the partials p = w, w+8, ... and are summed in a fixed order.
__global__ void __launch_bounds__(256)
    reduce_partials_bf16_kernel(const float4* __restrict__ partial, int n_part, int64_t n4,
                                __nv_bfloat16* __restrict__ out) {
  __shared__ float4 s_part[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (i < n4) {
#pragma unroll 4
    for (int p = warp; p < n_part; p += 8) {
      const float4 v = __ldg(partial + static_cast<int64_t>(p) * n4 + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  }
  s_part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && i < n4) {
    float4 r = s_part[0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      r.x += s_part[w][lane].x; r.y += s_part[w][lane].y;
      r.z += s_part[w][lane].z; r.w += s_part[w][lane].w;
    }
    uint2 packed = make_uint2(pack_bf16x2(r.x, r.y), pack_bf16x2(r.z, r.w));
    reinterpret_cast<uint2*>(out)[i] = packed;
  }
}

// out[e] = sum_p partial[p][e]: one warp per e, lanes stride over p, then a
// fixed-order butterfly.
__global__ void reduce_rows_f32_kernel(const float* __restrict__ partial, int n_part, int E,
                                       float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= E) return;
  float s = 0.f;
  for (int p = lane; p < n_part; p += 32) s += partial[static_cast<int64_t>(p) * E + e];
  s = warp_sum(s);
  if (lane == 0) out[e] = s;
}

}  // namespace

int router_bwd_blocks(int num_sms) { return num_sms * 4; }
int router_dw_small_chunk() { return kChunk; }

cudaError_t launch_router_bwd_dl(const float* dw, const float* probs, const int32_t* idx,
                                 const __nv_bfloat16* w_r, int T, int d, int E, int k, bool renorm,
                                 bool fuse_dx, float* dl_f32, __nv_bfloat16* dl_bf16,
                                 float* dx_router, float* db_partial, int nblocks,
                                 DeviceCtl* ctl, cudaStream_t st) {
  (void)ctl;
  const size_t w_bytes = static_cast<size_t>(E) * d * 2;
  const bool stage = fuse_dx && w_bytes <= 96 * 1024;
  const size_t smem = stage ? w_bytes : 0;
  auto go = [&](auto kern) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return cudaErrorInvalidValue;
    kern<<<nblocks, kWarps * 32, smem, st>>>(dw, probs, idx, w_r, T, d, E, k, renorm ? 1 : 0,
                                             dl_f32, dl_bf16, dx_router, db_partial,
                                             stage ? 1 : 0);
    return cudaGetLastError();
  };
  if (fuse_dx) {
    if (E <= 8) return go(router_bwd_dl_kernel<1, true, 8>);
    if (E <= 16) return go(router_bwd_dl_kernel<1, true, 16>);
    if (E <= 32) return go(router_bwd_dl_kernel<1, true, 32>);
    if (E <= 64) return go(router_bwd_dl_kernel<2, true, 64>);
    return cudaErrorInvalidValue;
  }
  if (E <= 128) return go(router_bwd_dl_kernel<4, false>);
  if (E <= 256) return go(router_bwd_dl_kernel<8, false>);
  if (E <= 512) return go(router_bwd_dl_kernel<16, false>);
  if (E <= 1024) return go(router_bwd_dl_kernel<32, false>);
  return cudaErrorInvalidValue;
}

cudaError_t launch_router_dw_small(const float* dl, const __nv_bfloat16* x, int T, int d, int E,
                                   float* partial, cudaStream_t st) {
  const unsigned gy = static_cast<unsigned>(ceil_div64(T, kChunk));
  auto go = [&](auto kern, int cpt) {
    const unsigned gx = static_cast<unsigned>(ceil_div64(d, kDwThreads * cpt));
    kern<<<dim3(gx, gy), kDwThreads, 0, st>>>(dl, x, T, d, E, partial);
    return cudaGetLastError();
  };
  if (E <= 8) return go(router_dw_small_kernel<8, 4>, 4);
  if (E <= 16) return go(router_dw_small_kernel<16, 2>, 2);
  if (E <= 32) return go(router_dw_small_kernel<32, 1>, 1);
  if (E <= 64) return go(router_dw_small_kernel<64, 1>, 1);
  return cudaErrorInvalidValue;
}

cudaError_t launch_reduce_partials_bf16(const float* partial, int n_part, int64_t n,
                                        __nv_bfloat16* out, cudaStream_t st) {
  const int64_t n4 = n / 4;  // n = E * d, a multiple of 256
  reduce_partials_bf16_kernel<<<static_cast<unsigned>(ceil_div64(n4, 32)), 256, 0, st>>>(
      reinterpret_cast<const float4*>(partial), n_part, n4, out);
  return cudaGetLastError();
}

cudaError_t launch_reduce_rows_f32(const float* partial, int n_part, int E, float* out,
                                   cudaStream_t st) {
  reduce_rows_f32_kernel<<<static_cast<unsigned>(ceil_div64(E, 8)), 256, 0, st>>>(partial, n_part,
                                                                                 E, out);
  return cudaGetLastError();
}

}  // namespace moe
