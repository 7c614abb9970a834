// Router forward: top-k softmax, one warp per token.
//
// "The router network computes a distribution over the experts for each
// token and keeps the k highest" -- discosf.com article on Olmo-core 3,
// sections 1.1 and 2.1.  Readings (the pages give no formula): softmax over
// all E experts in fp32; the k experts are chosen on the fp32 logit, ties
// to the lower expert index, slots ordered by descending logit; the gate
// weight is the chosen probability (renormalised over the k slots only when
// asked).  In the random-routing benchmark mode the ids come from the
// caller and the weights are still the router's probabilities.
#include <cfloat>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

// Selects the k best of `l[0..E)` held (redundantly) by every lane.
template <int NE>
__device__ __forceinline__ void topk_registers(const float (&l)[NE], int E, int k, int (&chosen)[8]) {
  uint64_t taken = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    float best = -FLT_MAX;
    int bi = -1;
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      if (e < E && !((taken >> e) & 1ull) && (bi < 0 || l[e] > best)) {
        best = l[e];
        bi = e;
      }
    }
    chosen[j] = bi;
    taken |= 1ull << bi;
  }
}

// Logits on CUDA cores for small E.  W_r is converted to fp32 once per
// block into shared memory (when it fits; else read as bf16 through L1);
// a warp takes TPW tokens at a time so every weight read serves TPW tokens,
// and each lane owns 8 consecutive features per 256.
template <int NE, int TPW, bool W_SMEM>
__global__ void __launch_bounds__(kWarps * 32)
    router_fused_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w_r,
                        const float* __restrict__ bias, const int32_t* __restrict__ route_in,
                        int T, int d, int E, int k, int renorm, int32_t* __restrict__ idx_out,
                        float* __restrict__ w_out, float* __restrict__ probs,
                        float* __restrict__ logits, DeviceCtl* ctl) {
  extern __shared__ float4 s_wf[];  // [E][d] fp32 when W_SMEM
  const int lane = threadIdx.x & 31;
  const int nvec = d >> 3;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const uint4* wv = reinterpret_cast<const uint4*>(w_r);
  if constexpr (W_SMEM) {
    for (int i = threadIdx.x; i < E * nvec; i += blockDim.x) {
      const uint4 q = __ldg(wv + i);
      s_wf[2 * i] = make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
      s_wf[2 * i + 1] = make_float4(bf16_lo(q.z), bf16_hi(q.z), bf16_lo(q.w), bf16_hi(q.w));
    }
    __syncthreads();
  }
  const int64_t groups = ceil_div64(T, TPW);
  for (int64_t grp = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); grp < groups;
       grp += static_cast<int64_t>(gridDim.x) * kWarps) {
    const int64_t t0 = grp * TPW;
    float acc[TPW][NE];
#pragma unroll
    for (int i = 0; i < TPW; ++i)
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[i][e] = 0.f;

    uint4 xq[TPW];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int64_t t = t0 + i < T ? t0 + i : T - 1;
      xq[i] = lane < nvec ? __ldg(xv + t * nvec + lane) : make_uint4(0, 0, 0, 0);
    }
    for (int v = lane; v < nvec; v += 32) {
      float xf[TPW][8];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        xf[i][0] = bf16_lo(xq[i].x); xf[i][1] = bf16_hi(xq[i].x);
        xf[i][2] = bf16_lo(xq[i].y); xf[i][3] = bf16_hi(xq[i].y);
        xf[i][4] = bf16_lo(xq[i].z); xf[i][5] = bf16_hi(xq[i].z);
        xf[i][6] = bf16_lo(xq[i].w); xf[i][7] = bf16_hi(xq[i].w);
      }
      if (v + 32 < nvec) {  // next features in flight while this slice is multiplied
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int64_t t = t0 + i < T ? t0 + i : T - 1;
          xq[i] = __ldg(xv + t * nvec + v + 32);
        }
      }
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        if (e < E) {
          float wf[8];
          if constexpr (W_SMEM) {
            const float4 a = s_wf[2 * (e * nvec + v)], b = s_wf[2 * (e * nvec + v) + 1];
            wf[0] = a.x; wf[1] = a.y; wf[2] = a.z; wf[3] = a.w;
            wf[4] = b.x; wf[5] = b.y; wf[6] = b.z; wf[7] = b.w;
          } else {
            const uint4 q = __ldg(wv + static_cast<int64_t>(e) * nvec + v);
            wf[0] = bf16_lo(q.x); wf[1] = bf16_hi(q.x);
            wf[2] = bf16_lo(q.y); wf[3] = bf16_hi(q.y);
            wf[4] = bf16_lo(q.z); wf[5] = bf16_hi(q.z);
            wf[6] = bf16_lo(q.w); wf[7] = bf16_hi(q.w);
          }
#pragma unroll
          for (int i = 0; i < TPW; ++i)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[i][e] = fmaf(xf[i][c], wf[c], acc[i][e]);
        }
      }
    }

#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int64_t t = t0 + i;
      if (t >= T) break;
      float l[NE];
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        l[e] = warp_sum(acc[i][e]);
        if (e < E && bias != nullptr) l[e] += __ldg(bias + e);
      }
      float m = -FLT_MAX;
#pragma unroll
      for (int e = 0; e < NE; ++e) if (e < E) m = fmaxf(m, l[e]);
      float sum = 0.f;
      float p[NE];
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        p[e] = e < E ? expf(l[e] - m) : 0.f;
        sum += p[e];
      }
      const float inv = 1.0f / sum;
#pragma unroll
      for (int e = 0; e < NE; ++e) p[e] *= inv;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        if (e < E && (e & 31) == lane) {
          probs[t * E + e] = p[e];
          if (logits != nullptr) logits[t * E + e] = l[e];
        }
      }
      int chosen[8];
      if (route_in == nullptr) {
        topk_registers<NE>(l, E, k, chosen);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) chosen[j] = j < k ? __ldg(route_in + t * k + j) : 0;
      }
      float wsel[8];
      float wsum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float pv = 0.f;
        if (j < k) {
          const int c = chosen[j];
          if (c >= 0 && c < E) {
#pragma unroll
            for (int e = 0; e < NE; ++e) if (e == c) pv = p[e];
          } else if (lane == 0) {
            report(ctl, MOE_ERR_DEVICE_CHECK, 100);
          }
        }
        wsel[j] = pv;
        wsum += pv;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && lane == j) {
          idx_out[t * k + j] = chosen[j];
          w_out[t * k + j] = renorm ? wsel[j] / wsum : wsel[j];
        }
      }
    }
  }
}

// Softmax + top-k from fp32 logits (large E); each lane holds NPL logits
// (expert lane + 32 i).  The winner of each round is found with a warp
// argmax on (logit desc, index asc).
template <int NPL>
__global__ void __launch_bounds__(kWarps * 32)
    softmax_topk_kernel(const float* __restrict__ logits_in, const float* __restrict__ bias,
                        const int32_t* __restrict__ route_in, int T, int E, int k, int renorm,
                        int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                        float* __restrict__ probs, float* __restrict__ logits_out,
                        DeviceCtl* ctl) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float l[NPL];
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      l[i] = logits_in[t * E + e] + (bias != nullptr ? __ldg(bias + e) : 0.f);
      m = fmaxf(m, l[i]);
    } else {
      l[i] = -FLT_MAX;
    }
  }
  m = warp_max(m);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) if (lane + 32 * i < E) s += expf(l[i] - m);
  s = warp_sum(s);
  const float inv = 1.0f / s;
  // selection first: logits_out may alias logits_in
  uint32_t taken = 0;
  int chosen[8];
  float wsel[8];
  float wsum = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    chosen[j] = 0;
    wsel[j] = 0.f;
    if (j >= k) continue;
    if (route_in == nullptr) {
      float bv = -FLT_MAX;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && (bi == 0x7fffffff || l[i] > bv)) {
          bv = l[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      chosen[j] = bi;
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      wsel[j] = expf(bv - m) * inv;
    } else {
      const int c = __ldg(route_in + t * k + j);
      chosen[j] = c;
      if (c >= 0 && c < E) {
        const float lc = logits_in[t * E + c] + (bias != nullptr ? __ldg(bias + c) : 0.f);
        wsel[j] = expf(lc - m) * inv;
      } else if (lane == 0) {
        report(ctl, MOE_ERR_DEVICE_CHECK, 101);
      }
    }
    wsum += wsel[j];
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      probs[t * E + e] = expf(l[i] - m) * inv;
      if (logits_out != nullptr) logits_out[t * E + e] = l[i];
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k && lane == j) {
      idx_out[t * k + j] = chosen[j];
      w_out[t * k + j] = renorm ? wsel[j] / wsum : wsel[j];
    }
  }
}

}  // namespace

cudaError_t launch_router_fused(const __nv_bfloat16* x, const __nv_bfloat16* w_r, const float* bias,
                                const int32_t* route_in, int T, int d, int E, int k, bool renorm,
                                int32_t* idx, float* w, float* probs, float* logits,
                                DeviceCtl* ctl, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t w_smem = static_cast<size_t>(E) * d * 4;
  auto go = [&](auto kern_smem, auto kern_l1, int tpw) {
    const int64_t groups = ceil_div64(T, tpw);
    const int64_t want = ceil_div64(groups, kWarps);
    if (w_smem <= 96 * 1024) {
      if (w_smem > 48 * 1024 &&
          cudaFuncSetAttribute(kern_smem, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(w_smem)) != cudaSuccess)
        return cudaErrorInvalidValue;
      const unsigned grid = static_cast<unsigned>(want < 2 * sms ? want : 2 * sms);
      kern_smem<<<grid, kWarps * 32, w_smem, st>>>(x, w_r, bias, route_in, T, d, E, k,
                                                   renorm ? 1 : 0, idx, w, probs, logits, ctl);
    } else {
      const unsigned grid = static_cast<unsigned>(want < 8 * sms ? want : 8 * sms);
      kern_l1<<<grid, kWarps * 32, 0, st>>>(x, w_r, bias, route_in, T, d, E, k, renorm ? 1 : 0,
                                            idx, w, probs, logits, ctl);
    }
    return cudaGetLastError();
  };
  if (E <= 8) return go(router_fused_kernel<8, 4, true>, router_fused_kernel<8, 4, false>, 4);
  if (E <= 16) return go(router_fused_kernel<16, 2, true>, router_fused_kernel<16, 2, false>, 2);
  if (E <= 32) return go(router_fused_kernel<32, 1, true>, router_fused_kernel<32, 1, false>, 1);
  if (E <= 64) return go(router_fused_kernel<64, 1, true>, router_fused_kernel<64, 1, false>, 1);
  return cudaErrorInvalidValue;
}

cudaError_t launch_softmax_topk(const float* logits_in, const float* bias, const int32_t* route_in,
                                int T, int E, int k, bool renorm, int32_t* idx, float* w,
                                float* probs, float* logits_out, DeviceCtl* ctl, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(T, kWarps));
  auto go = [&](auto kern) {
    kern<<<grid, kWarps * 32, 0, st>>>(logits_in, bias, route_in, T, E, k, renorm ? 1 : 0, idx, w,
                                       probs, logits_out, ctl);
    return cudaGetLastError();
  };
  if (E <= 32) return go(softmax_topk_kernel<1>);
  if (E <= 64) return go(softmax_topk_kernel<2>);
  if (E <= 128) return go(softmax_topk_kernel<4>);
  if (E <= 256) return go(softmax_topk_kernel<8>);
  if (E <= 512) return go(softmax_topk_kernel<16>);
  if (E <= 1024) return go(softmax_topk_kernel<32>);
  return cudaErrorInvalidValue;
}

}  // namespace moe
