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
  pdl_wait();
  pdl_trigger();
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

// Logits for E <= 16 on the warp-level bf16 tensor-core MMA (m16n8k16,
// fp32 accumulate).  For such E the contraction is a skinny [T, d] x [d, E]
// product bound by reading x once from HBM; the MMA only keeps the FMAs off
// the CUDA cores so that the loads stay in flight.
//
// A block owns 16 consecutive tokens; its 4 warps split d into quarters and
// their partial logits are summed in a fixed order through shared memory.
// Inside a 32-feature chunk, lane (g = lane/4, q = lane%4) loads the 16-byte
// vectors x[t0+g][8q..8q+7], x[t0+g+8][8q..8q+7] and W_r[n0+g][8q..8q+7].
// Because the contraction index may be relabelled freely (the same way in
// both operands), those vectors are used directly as fragments: their
// first halves feed one MMA and their second halves a second one.  The
// accumulator then holds, in lane (g, q), the logits of tokens g and g+8 for
// experts n0 + 2q and n0 + 2q + 1.
constexpr int kMmaWarps = 4;
constexpr int kMmaTokens = 16;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The best not-yet-taken expert of one token over the 4 lanes of a lane
// group: (higher logit, then lower index).  Each lane holds 2*NT logits.
template <int NT>
__device__ __forceinline__ void group_argmax(const float (&l)[2 * NT], const int (&eid)[2 * NT],
                                             uint32_t taken, int E, float& bv, int& bi) {
  bv = -FLT_MAX;
  bi = 0x7fffffff;
#pragma unroll
  for (int s = 0; s < 2 * NT; ++s) {
    if (eid[s] < E && !((taken >> s) & 1u) && (bi == 0x7fffffff || l[s] > bv)) {
      bv = l[s];
      bi = eid[s];
    }
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
      bv = ov;
      bi = oi;
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kMmaWarps * 32, NT == 1 ? 7 : 5)
    router_mma_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w_r,
                      const float* __restrict__ bias, const int32_t* __restrict__ route_in, int T,
                      int d, int E, int k, int renorm, int32_t* __restrict__ idx_out,
                      float* __restrict__ w_out, float* __restrict__ probs,
                      float* __restrict__ logits, DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  __shared__ float4 s_part[kMmaWarps][NT][32];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kMmaTokens;
  const int nvec = d >> 3;                 // 16-byte vectors per row
  const int chunks = d >> 5;               // 32-feature chunks per row
  const int per_warp = chunks / kMmaWarps; // d is a multiple of 128
  const int64_t ra = t0 + g < T ? t0 + g : T - 1;          // ragged tail: clamp the
  const int64_t rb = t0 + g + 8 < T ? t0 + g + 8 : T - 1;  // loads, skip the stores
  const uint4* xa = reinterpret_cast<const uint4*>(x) + ra * nvec + q;
  const uint4* xb = reinterpret_cast<const uint4*>(x) + rb * nvec + q;
  const uint4* wv[NT];
  bool wok[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    wok[nt] = nt * 8 + g < E;
    wv[nt] = reinterpret_cast<const uint4*>(w_r) + static_cast<int64_t>(wok[nt] ? nt * 8 + g : 0) * nvec + q;
  }

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

  constexpr int P = 4;  // chunks whose loads are issued together
  const int c_lo = warp * per_warp, c_hi = c_lo + per_warp;
  for (int c0 = c_lo; c0 < c_hi; c0 += P) {
    uint4 va[P], vb[P], vw[P][NT];
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if (c0 + j < c_hi) {
        const int o = (c0 + j) * 4;
        va[j] = ld_stream16(xa + o);
        vb[j] = ld_stream16(xb + o);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) vw[j][nt] = wok[nt] ? __ldg(wv[nt] + o) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if (c0 + j < c_hi) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_bf16_16816(acc[nt], va[j].x, vb[j].x, va[j].y, vb[j].y, vw[j][nt].x, vw[j][nt].y);
          mma_bf16_16816(acc[nt], va[j].z, vb[j].z, va[j].w, vb[j].w, vw[j][nt].z, vw[j][nt].w);
        }
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    s_part[warp][nt][lane] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
  __syncthreads();
  if (warp != 0) return;

  // ---- warp 0: sum the quarters (in warp order), softmax, top-k
  float lg[2][2 * NT];  // [token g / g+8][slot]; slot 2nt+i is expert 8nt + 2q + i
  int eid[2 * NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float4 s = s_part[0][nt][lane];
#pragma unroll
    for (int w = 1; w < kMmaWarps; ++w) {
      const float4 u = s_part[w][nt][lane];
      s.x += u.x; s.y += u.y; s.z += u.z; s.w += u.w;
    }
    lg[0][2 * nt] = s.x; lg[0][2 * nt + 1] = s.y;
    lg[1][2 * nt] = s.z; lg[1][2 * nt + 1] = s.w;
    eid[2 * nt] = nt * 8 + 2 * q;
    eid[2 * nt + 1] = nt * 8 + 2 * q + 1;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t t = t0 + g + 8 * h;
    float(&l)[2 * NT] = lg[h];
    float m = -FLT_MAX;
#pragma unroll
    for (int s = 0; s < 2 * NT; ++s) {
      if (eid[s] < E) {
        if (bias != nullptr) l[s] += __ldg(bias + eid[s]);
        m = fmaxf(m, l[s]);
      }
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float p[2 * NT];
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < 2 * NT; ++s) {
      p[s] = eid[s] < E ? expf(l[s] - m) : 0.f;
      sum += p[s];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int s = 0; s < 2 * NT; ++s) p[s] *= inv;

    int chosen[8];
    float wsel[8];
    float wsum = 0.f;
    uint32_t taken = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      chosen[j] = 0;
      wsel[j] = 0.f;
      if (j >= k) continue;
      int c;
      if (route_in == nullptr) {
        float bv;
        group_argmax<NT>(l, eid, taken, E, bv, c);
      } else {
        c = t < T ? __ldg(route_in + t * k + j) : 0;
        if ((c < 0 || c >= E) && q == 0 && t < T) report(ctl, MOE_ERR_DEVICE_CHECK, 100);
      }
      // the chosen expert's probability, from the lane that holds it
      float pv = 0.f;
#pragma unroll
      for (int s = 0; s < 2 * NT; ++s) {
        if (eid[s] == c) {
          pv = p[s];
          taken |= 1u << s;
        }
      }
      pv += __shfl_xor_sync(0xffffffffu, pv, 1);
      pv += __shfl_xor_sync(0xffffffffu, pv, 2);
      chosen[j] = c;
      wsel[j] = pv;
      wsum += pv;
    }
    if (t < T) {
#pragma unroll
      for (int s = 0; s < 2 * NT; ++s) {
        if (eid[s] < E) {
          probs[t * E + eid[s]] = p[s];
          if (logits != nullptr) logits[t * E + eid[s]] = l[s];
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && (j & 3) == q) {
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
    softmax_topk_kernel(const float* __restrict__ logits_in, int ld_in,
                        const float* __restrict__ bias,
                        const int32_t* __restrict__ route_in, int T, int E, int k, int renorm,
                        int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                        float* __restrict__ probs, float* __restrict__ logits_out,
                        DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float l[NPL];
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      l[i] = logits_in[t * ld_in + e] + (bias != nullptr ? __ldg(bias + e) : 0.f);
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
        const float lc = logits_in[t * ld_in + c] + (bias != nullptr ? __ldg(bias + c) : 0.f);
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
                                DeviceCtl* ctl, int sms, cudaStream_t st) {
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
      (void)launch_pdl(kern_smem, grid, kWarps * 32, w_smem, st, x, w_r, bias, route_in, T, d, E, k,
                                                   renorm ? 1 : 0, idx, w, probs, logits, ctl);
    } else {
      const unsigned grid = static_cast<unsigned>(want < 8 * sms ? want : 8 * sms);
      (void)launch_pdl(kern_l1, grid, kWarps * 32, 0, st, x, w_r, bias, route_in, T, d, E, k, renorm ? 1 : 0,
                                            idx, w, probs, logits, ctl);
    }
    return cudaGetLastError();
  };
  if (E <= 16) {
    const unsigned grid = static_cast<unsigned>(ceil_div64(T, kMmaTokens));
    if (E <= 8)
      (void)launch_pdl(router_mma_kernel<1>, grid, kMmaWarps * 32, 0, st, x, w_r, bias, route_in, T, d, E, k,
                                                            renorm ? 1 : 0, idx, w, probs, logits, ctl);
    else
      (void)launch_pdl(router_mma_kernel<2>, grid, kMmaWarps * 32, 0, st, x, w_r, bias, route_in, T, d, E, k,
                                                            renorm ? 1 : 0, idx, w, probs, logits, ctl);
    return cudaGetLastError();
  }
  if (E <= 32) return go(router_fused_kernel<32, 1, true>, router_fused_kernel<32, 1, false>, 1);
  if (E <= 64) return go(router_fused_kernel<64, 1, true>, router_fused_kernel<64, 1, false>, 1);
  return cudaErrorInvalidValue;
}

cudaError_t launch_softmax_topk(const float* logits_in, int ld_in, const float* bias,
                                const int32_t* route_in, int T, int E, int k, bool renorm,
                                int32_t* idx, float* w, float* probs, float* logits_out,
                                DeviceCtl* ctl, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(T, kWarps));
  auto go = [&](auto kern) {
    (void)launch_pdl(kern, grid, kWarps * 32, 0, st, logits_in, ld_in, bias, route_in, T, E, k, renorm ? 1 : 0, idx, w,
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
