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

template <int NPL, bool FUSE_DX>
__global__ void __launch_bounds__(kWarps * 32)
    router_bwd_dl_kernel(const float* __restrict__ dw, const float* __restrict__ probs,
                         const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ w_r,
                         int T, int d, int E, int k, int renorm, float* __restrict__ dl_f32,
                         __nv_bfloat16* __restrict__ dl_bf16, float* __restrict__ dx_router,
                         float* __restrict__ db_partial) {
  __shared__ float s_db[kWarps][32 * NPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
      // dX_router[t, :] = sum_e dL[e] W_r[e, :]; lane owns 8 columns per 256
      const uint4* wv = reinterpret_cast<const uint4*>(w_r);
      float4* out = reinterpret_cast<float4*>(dx_router + t * d);
      for (int v = lane; v < nvec; v += 32) {
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          for (int src = 0; src < 32; ++src) {
            const int e = 32 * i + src;
            const float dle = __shfl_sync(0xffffffffu, dl[i], src);
            if (e >= E) break;
            const uint4 q = __ldg(wv + static_cast<int64_t>(e) * nvec + v);
            acc[0] = fmaf(dle, bf16_lo(q.x), acc[0]); acc[1] = fmaf(dle, bf16_hi(q.x), acc[1]);
            acc[2] = fmaf(dle, bf16_lo(q.y), acc[2]); acc[3] = fmaf(dle, bf16_hi(q.y), acc[3]);
            acc[4] = fmaf(dle, bf16_lo(q.z), acc[4]); acc[5] = fmaf(dle, bf16_hi(q.z), acc[5]);
            acc[6] = fmaf(dle, bf16_lo(q.w), acc[6]); acc[7] = fmaf(dle, bf16_hi(q.w), acc[7]);
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
// owns CPT consecutive columns and all E experts of them.
constexpr int kChunk = 128;

template <int NE, int CPT>
__global__ void __launch_bounds__(256)
    router_dw_small_kernel(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ x, int T,
                           int d, int E, float* __restrict__ partial) {
  __shared__ float s_dl[kChunk * NE];
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kChunk;
  const int nt = T - t0 < kChunk ? static_cast<int>(T - t0) : kChunk;
  for (int i = threadIdx.x; i < nt * E; i += blockDim.x) {
    const int tt = i / E, e = i - tt * E;
    s_dl[tt * NE + e] = dl[(t0 + tt) * E + e];
  }
  __syncthreads();
  const int64_t col = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) * CPT;
  if (col >= d) return;
  float acc[NE][CPT];
#pragma unroll
  for (int e = 0; e < NE; ++e)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[e][c] = 0.f;
  for (int tt = 0; tt < nt; ++tt) {
    float xv[CPT];
    const __nv_bfloat16* xr = x + (t0 + tt) * d + col;
#pragma unroll
    for (int c = 0; c < CPT; ++c) xv[c] = __bfloat162float(xr[c]);
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

__global__ void reduce_partials_bf16_kernel(const float* __restrict__ partial, int n_part,
                                            int64_t n, __nv_bfloat16* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int p = 0; p < n_part; ++p) s += partial[static_cast<int64_t>(p) * n + i];
    out[i] = __float2bfloat16_rn(s);
  }
}

__global__ void reduce_rows_f32_kernel(const float* __restrict__ partial, int n_part, int E,
                                       float* __restrict__ out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  float s = 0.f;
  for (int p = 0; p < n_part; ++p) s += partial[static_cast<int64_t>(p) * E + e];
  out[e] = s;
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
  auto go = [&](auto kern) {
    kern<<<nblocks, kWarps * 32, 0, st>>>(dw, probs, idx, w_r, T, d, E, k, renorm ? 1 : 0, dl_f32,
                                          dl_bf16, dx_router, db_partial);
    return cudaGetLastError();
  };
  if (fuse_dx) {
    if (E <= 32) return go(router_bwd_dl_kernel<1, true>);
    if (E <= 64) return go(router_bwd_dl_kernel<2, true>);
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
    const unsigned gx = static_cast<unsigned>(ceil_div64(d, 256 * cpt));
    kern<<<dim3(gx, gy), 256, 0, st>>>(dl, x, T, d, E, partial);
    return cudaGetLastError();
  };
  if (E <= 8) return go(router_dw_small_kernel<8, 8>, 8);
  if (E <= 16) return go(router_dw_small_kernel<16, 4>, 4);
  if (E <= 32) return go(router_dw_small_kernel<32, 2>, 2);
  if (E <= 64) return go(router_dw_small_kernel<64, 1>, 1);
  return cudaErrorInvalidValue;
}

cudaError_t launch_reduce_partials_bf16(const float* partial, int n_part, int64_t n,
                                        __nv_bfloat16* out, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(n, 256) < 4096 ? ceil_div64(n, 256) : 4096);
  reduce_partials_bf16_kernel<<<grid, 256, 0, st>>>(partial, n_part, n, out);
  return cudaGetLastError();
}

cudaError_t launch_reduce_rows_f32(const float* partial, int n_part, int E, float* out,
                                   cudaStream_t st) {
  reduce_rows_f32_kernel<<<static_cast<unsigned>(ceil_div64(E, 256)), 256, 0, st>>>(partial, n_part,
                                                                                    E, out);
  return cudaGetLastError();
}

}  // namespace moe
