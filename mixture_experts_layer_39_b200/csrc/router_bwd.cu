// Router backward: gradient through the selected softmax probabilities.
//
// The top-k choice is piecewise constant, so only the chosen probabilities
// carry gradient.  With g = d(loss)/d(gate weight) (adjusted for the
// optional renormalisation), dp[t, idx[t,j]] = g[t,j] and the softmax
// backward gives dL = p * (dp - <p, dp>).  Then
//   dX_router = dL W_r,  dW_r = dL^T x,  db = sum_t dL.
// For E <= 64 this file forms them: dX_router inside the permute backward,
// dW_r with mma.sync (E <= 16) or on CUDA cores (E <= 64).  Above 64 experts
// the two products run on the tcgen05 grouped GEMM (see gemm.cu) and this
// file only produces dL (bf16) and the db partial sums.
#include <type_traits>

#include "host_ctx.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

// dL[t, e] = p[t,e] (dp[t,e] - <p[t], dp[t]>) of one token, held by the warp
// in the lane layout e = lane + 32 i (i < NPL); dp is the gate-weight
// gradient scattered to the chosen experts (after the renormalisation's
// backward when the gate weights were renormalised), plus dprob_aux[e] for
// every expert when given (the load-balancing loss's gradient, the same for
// all tokens).  Ids outside [0, E) carry no gradient.  Every lane must call
// it (one warp reduction).
template <int NPL>
__device__ __forceinline__ void token_dlogits(const float* __restrict__ dw,
                                              const float* __restrict__ probs,
                                              const int32_t* __restrict__ idx,
                                              const float* __restrict__ dprob_aux, int64_t t,
                                              int E, int k, int renorm, int lane,
                                              float (&dl)[NPL]) {
  int id[8];
  float g[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    id[j] = j < k ? __ldg(idx + t * k + j) : -1;
    g[j] = j < k ? __ldg(dw + t * k + j) : 0.f;
    if (id[j] < 0 || id[j] >= E) id[j] = -1;
  }
  if (renorm) {
    float ps[8];
    float psel_sum = 0.f;
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
    if (dprob_aux != nullptr && e < E) dp[i] += __ldg(dprob_aux + e);
    pdp += p[i] * dp[i];
  }
  pdp = warp_sum(pdp);
#pragma unroll
  for (int i = 0; i < NPL; ++i) dl[i] = p[i] * (dp[i] - pdp);
}

// dX_router[t, 8v .. 8v+7] = sum_e dL[e] W_r[e, 8v .. 8v+7], experts in
// increasing order from zero (every caller sums in this same order).
template <int NE>
__device__ __forceinline__ void router_dx_slice(const uint4* __restrict__ wv, int nvec, int E, int v,
                                                const float (&dle)[NE], float (&acc)[8]) {
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
}

// NE: compile-time bound on E for the fused dX_router loop (E <= NE <= 32*NPL).
template <int NPL, bool FUSE_DX, int NE = 32 * NPL>
__global__ void __launch_bounds__(kWarps * 32)
    router_bwd_dl_kernel(const float* __restrict__ dw, const float* __restrict__ probs,
                         const int32_t* __restrict__ idx, const float* __restrict__ dprob_aux,
                         const __nv_bfloat16* __restrict__ w_r,
                         int T, int d, int E, int k, int renorm, float* __restrict__ dl_f32,
                         __nv_bfloat16* __restrict__ dl_bf16, int ld_bf16,
                         float* __restrict__ dx_router,
                         float* __restrict__ db_partial, int stage_w) {
  pdl_wait();
  pdl_trigger();
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
    float dl[NPL];
    token_dlogits<NPL>(dw, probs, idx, dprob_aux, t, E, k, renorm, lane, dl);
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        db[i] += dl[i];
        if (dl_f32 != nullptr) dl_f32[t * E + e] = dl[i];
        if (dl_bf16 != nullptr) dl_bf16[t * ld_bf16 + e] = __float2bfloat16_rn(dl[i]);
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
        router_dx_slice<NE>(wv, nvec, E, v, dle, acc);
        out[2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
  // per-block partial of db (fixed order: warps, then blocks in a later pass)
  if (db_partial == nullptr) return;
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

// dX[t] = bf16(sum_j dX_perm[row_map[t,j]] + dX_router[t]) with dX_router[t]
// = dL[t] W_r formed on the fly (E <= 64), so that the [T, d] fp32 dX_router
// never goes through HBM.  dL is recomputed per token from the gate-weight
// gradient (a few hundred bytes per token).  A warp takes TPW tokens so that
// every W_r vector it reads (through L1; W_r is at most 256 KB) serves TPW
// tokens; the dX_perm gathers bypass L1.  KMAX bounds k at compile time.  Sums run in the same order as the
// two-kernel path (router dX, then unpermute-reduce), so both give the same
// bits.
template <int NE, int TPW, int KMAX, bool SHARED>
__global__ void __launch_bounds__(kWarps * 32, 2)
    permute_router_bwd_kernel(const uint4* __restrict__ dxp, const int32_t* __restrict__ row_map,
                              const float* __restrict__ dw, const float* __restrict__ probs,
                              const int32_t* __restrict__ idx,
                              const float* __restrict__ dprob_aux,
                              const __nv_bfloat16* __restrict__ w_r,
                              const uint4* __restrict__ dxs, int T, int d, int E, int k,
                              int renorm, uint4* __restrict__ dx) {
  pdl_wait();
  pdl_trigger();
  constexpr int NPL = (NE + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5)) * TPW;
  if (t0 >= T) return;
  const int nvec = d >> 3;
  float dle[TPW][NE];
  int rows[TPW][KMAX];
#pragma unroll
  for (int h = 0; h < TPW; ++h) {
    const int64_t t = t0 + h < T ? t0 + h : t0;  // a missing second token repeats the first
    float dl[NPL];
    token_dlogits<NPL>(dw, probs, idx, dprob_aux, t, E, k, renorm, lane, dl);
#pragma unroll
    for (int e = 0; e < NE; ++e) dle[h][e] = __shfl_sync(0xffffffffu, dl[e >> 5], e & 31);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) rows[h][j] = j < k ? __ldg(row_map + t * k + j) : -1;
  }
  const uint4* wv = reinterpret_cast<const uint4*>(w_r);
  for (int v = lane; v < nvec; v += 32) {
    uint4 q[TPW][KMAX];
#pragma unroll
    for (int h = 0; h < TPW; ++h)
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (rows[h][j] >= 0) q[h][j] = ld_stream16(dxp + static_cast<int64_t>(rows[h][j]) * nvec + v);
    float r[TPW][8];
#pragma unroll
    for (int h = 0; h < TPW; ++h) router_dx_slice<NE>(wv, nvec, E, v, dle[h], r[h]);
#pragma unroll
    for (int h = 0; h < TPW; ++h) {
      if (t0 + h >= T) break;
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (rows[h][j] < 0) continue;
        float f[8];
        unpack8(q[h][j], f);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += f[c];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += r[h][c];
      if constexpr (SHARED) {  // the shared expert's input gradient, added last
        float f[8];
        unpack8(__ldg(dxs + (t0 + h) * nvec + v), f);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += f[c];
      }
      dx[(t0 + h) * nvec + v] = pack8(acc);
    }
  }
}

// dW_r partial sums over a chunk of tokens, CUDA cores (16 < E <= 64).  A block
// owns a slice of kDwCols columns of x and a chunk of tokens (a multiple of
// kDwTok); it streams the chunk through shared memory in stages of kDwTok
// tokens (the x slice and the matching dL rows), double-buffered with
// cp.async so that the next stage is in flight while this one is reduced.
// Each thread owns 2 consecutive columns and all E experts of them; tokens
// are accumulated in increasing order.  The grid holds about as many blocks
// as stay resident, so every partial row stands for a large chunk of tokens.
constexpr int kDwThreads = 256;
constexpr int kDwCols = 2 * kDwThreads;      // 512 columns = 1 KB of a bf16 row
constexpr int kDwTok = 32;                   // tokens per stage
constexpr int kDwStageX = kDwTok * kDwCols * 2;  // 32 KB of x per stage

__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(sdst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}

__device__ __forceinline__ void cp_async4b(void* sdst, const void* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(sdst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gsrc) : "memory");
}

template <int NE>
__global__ void __launch_bounds__(kDwThreads)
    router_dw_kernel(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ x, int T,
                     int d, int E, int group_len, float* __restrict__ partial) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t s_raw[];
  uint8_t* s_x = s_raw;                                              // [2][kDwTok][kDwCols] bf16
  float* s_dl = reinterpret_cast<float*>(s_raw + 2 * kDwStageX);      // [2][kDwTok][NE]
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kDwCols;
  const int width = d - col0 < kDwCols ? static_cast<int>(d - col0) : kDwCols;  // 256 or 512
  const int pieces = width / 8;                                       // 16-byte pieces per row
  const int64_t g0 = static_cast<int64_t>(blockIdx.y) * group_len;
  const int64_t g1 = g0 + group_len < T ? g0 + group_len : T;
  const int n_stages = g1 > g0 ? static_cast<int>(ceil_div64(g1 - g0, kDwTok)) : 0;

  auto issue = [&](int sidx) {
    const int64_t s0 = g0 + static_cast<int64_t>(sidx) * kDwTok;
    const int nt = g1 - s0 < kDwTok ? static_cast<int>(g1 - s0) : kDwTok;
    uint8_t* bx = s_x + (sidx & 1) * kDwStageX;
    for (int i = threadIdx.x; i < nt * pieces; i += kDwThreads) {
      const int tt = i / pieces, q = i - tt * pieces;
      cp_async16(bx + tt * (kDwCols * 2) + q * 16, x + (s0 + tt) * d + col0 + q * 8);
    }
    float* bd = s_dl + (sidx & 1) * (kDwTok * NE);
    for (int i = threadIdx.x; i < nt * E; i += kDwThreads) {
      const int tt = i / E, e = i - tt * E;
      cp_async4b(bd + tt * NE + e, dl + s0 * E + i);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  const int c = threadIdx.x * 2;  // this thread's first column in the slice
  const bool active = c < width;
  float acc[NE][2];
#pragma unroll
  for (int e = 0; e < NE; ++e) acc[e][0] = acc[e][1] = 0.f;
  if (n_stages > 0) issue(0);
  for (int sidx = 0; sidx < n_stages; ++sidx) {
    if (sidx + 1 < n_stages) {
      issue(sidx + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();  // every thread's copies of this stage have landed
    const int64_t s0 = g0 + static_cast<int64_t>(sidx) * kDwTok;
    const int nt = g1 - s0 < kDwTok ? static_cast<int>(g1 - s0) : kDwTok;
    const uint8_t* bx = s_x + (sidx & 1) * kDwStageX;
    const float* bd = s_dl + (sidx & 1) * (kDwTok * NE);
    if (active) {
#pragma unroll 4
      for (int tt = 0; tt < nt; ++tt) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(bx + tt * (kDwCols * 2) + c * 2);
        const float x0 = bf16_lo(w), x1 = bf16_hi(w);
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          if (e < E) {
            const float g = bd[tt * NE + e];
            acc[e][0] = fmaf(g, x0, acc[e][0]);
            acc[e][1] = fmaf(g, x1, acc[e][1]);
          }
        }
      }
    }
    __syncthreads();  // this buffer is refilled two stages later
  }
  if (!active) return;
  float* out = partial + static_cast<int64_t>(blockIdx.y) * E * d + col0 + c;
#pragma unroll
  for (int e = 0; e < NE; ++e)
    if (e < E)
      *reinterpret_cast<float2*>(out + static_cast<int64_t>(e) * d) = make_float2(acc[e][0], acc[e][1]);
}

// dW_r partial sums for E <= 16 on the tensor cores.  dW_r^T[col][e] =
// sum_t x[t][col] dL[t][e] is a product with M = columns, K = tokens and
// N = experts: bf16 mma.sync m16n8k16, x^T fragments loaded from shared
// memory with ldmatrix.trans, fp32 accumulation.  x is exact in bf16; dL is
// split into bf16 hi + lo parts (two MMAs), which keeps about 16 of its 24
// mantissa bits.  A block owns kDsCols (or d) columns and a chunk of tokens;
// a 3-deep ring of stages, each the chunk's next kDsTok rows of x (one
// cp.async.bulk per row, rows padded by 16 bytes so that ldmatrix is free of
// bank conflicts) and their dL rows, is filled by thread 0 and completes on
// an mbarrier per stage.  Warp w owns columns [256w, 256w + 256); tokens are
// accumulated in increasing order, so the result does not depend on timing.
constexpr int kDsThreads = 256;
constexpr int kDsCols = 2048;
constexpr int kDsTok = 16;  // tokens per stage = one MMA K step
constexpr int kDsStages = 3;
constexpr int kDsRow = kDsCols * 2 + 16;            // padded smem row, bytes
constexpr int kDsStageX = kDsTok * kDsRow;          // 65792 bytes
constexpr int kDsStageDl = kDsTok * 16 * 4;         // dL rows of up to 16 experts
constexpr size_t kDsSmem = kDsStages * (kDsStageX + kDsStageDl) + kDsStages * 8;

__device__ __forceinline__ void ds_mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void ds_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// global -> shared bulk copy completing on `bar` (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void ds_bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// bounded wait on a phase of `bar`; false after kDsWaitNs
constexpr uint64_t kDsWaitNs = 2000000000ull;
__device__ __forceinline__ bool ds_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok = 0;
  uint64_t t0 = 0;
  for (int i = 0;; ++i) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (i == 0) t0 = globaltimer_ns();
    else if (globaltimer_ns() - t0 > kDsWaitNs) return false;
  }
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 hi part of v, and the bf16 of what is left
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

template <int NE>
__global__ void __launch_bounds__(kDsThreads, 1)
    router_dw_stream_kernel(const float* __restrict__ dl, const __nv_bfloat16* __restrict__ x,
                            int T, int d, int E, int group_len, float* __restrict__ partial,
                            DeviceCtl* ctl) {
  static_assert(NE == 8 || NE == 16, "experts per n-tile");
  constexpr int NT = NE / 8;  // MMA n-tiles of 8 experts
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t s_raw[];
  uint8_t* s_x = s_raw;  // [stages][kDsTok][kDsRow]
  float* s_dl = reinterpret_cast<float*>(s_raw + kDsStages * kDsStageX);  // [stages][kDsTok][E]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_raw + kDsStages * (kDsStageX + kDsStageDl));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kDsCols;
  const int cols = d - col0 < kDsCols ? static_cast<int>(d - col0) : kDsCols;  // multiple of 128
  const int wcol = warp * 256;                    // this warp's first column
  const int mtiles = cols - wcol >= 256 ? 16 : (cols > wcol ? (cols - wcol) / 16 : 0);
  const int64_t g0 = static_cast<int64_t>(blockIdx.y) * group_len;
  const int64_t g1 = g0 + group_len < T ? g0 + group_len : T;
  const int n_stages = g1 > g0 ? static_cast<int>(ceil_div64(g1 - g0, kDsTok)) : 0;
  auto bar = [&](int st) { return static_cast<uint32_t>(__cvta_generic_to_shared(bars + st)); };
  auto issue = [&](int sidx) {  // thread 0
    const int st = sidx % kDsStages;
    const int64_t s0 = g0 + static_cast<int64_t>(sidx) * kDsTok;
    const int nt = g1 - s0 < kDsTok ? static_cast<int>(g1 - s0) : kDsTok;
    // dL rows: 16-byte multiples (the dL buffer is padded to 256 bytes)
    const uint32_t dl_bytes = (static_cast<uint32_t>(nt * E * 4) + 15u) & ~15u;
    ds_expect_tx(bar(st), static_cast<uint32_t>(nt * cols * 2) + dl_bytes);
    const uint32_t sx = static_cast<uint32_t>(__cvta_generic_to_shared(s_x + st * kDsStageX));
    for (int tt = 0; tt < nt; ++tt)
      ds_bulk_g2s(sx + tt * kDsRow, x + (s0 + tt) * d + col0, static_cast<uint32_t>(cols * 2),
                  bar(st));
    ds_bulk_g2s(static_cast<uint32_t>(__cvta_generic_to_shared(s_dl + st * (kDsStageDl / 4))),
                dl + s0 * E, dl_bytes, bar(st));
  };
  // rows a short last stage does not fill must hold finite values (their dL is 0)
  for (int i = tid; i < kDsStages * kDsStageX / 16; i += kDsThreads)
    reinterpret_cast<uint4*>(s_x)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    for (int st = 0; st < kDsStages; ++st) ds_mbar_init(bar(st), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zeros before the bulk writes
  __syncthreads();
  if (tid == 0)
    for (int sidx = 0; sidx < kDsStages && sidx < n_stages; ++sidx) issue(sidx);

  float acc[16][NT][4];
#pragma unroll
  for (int m = 0; m < 16; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;
  // ldmatrix: lane l addresses row (l & 7) of 8x8 matrix l >> 3:
  // matrices (cols 0-7, tokens 0-7), (cols 8-15, tokens 0-7), (0-7, 8-15), (8-15, 8-15)
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t lofs = static_cast<uint32_t>(((lm >> 1) * 8 + lr) * kDsRow + (wcol + (lm & 1) * 8) * 2);
  int done = 0;
  bool ok = true;
  for (int sidx = 0; sidx < n_stages; ++sidx) {
    const int st = sidx % kDsStages;
    ok = __syncthreads_and(ds_wait(bar(st), static_cast<uint32_t>((sidx / kDsStages) & 1)));
    if (!ok) break;
    const int64_t s0 = g0 + static_cast<int64_t>(sidx) * kDsTok;
    const int nt = g1 - s0 < kDsTok ? static_cast<int>(g1 - s0) : kDsTok;
    const float* bd = s_dl + st * (kDsStageDl / 4);
    // B fragments (K = tokens x N = experts): b0 = dL[2q, 2q+1][e], b1 = dL[2q+8, 2q+9][e],
    // e = 8n + g; hi and lo parts
    uint32_t bhi[NT][2], blo[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int e = 8 * n + g;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t0 = 2 * q + 8 * h;
        const float v0 = (e < E && t0 < nt) ? bd[t0 * E + e] : 0.f;
        const float v1 = (e < E && t0 + 1 < nt) ? bd[(t0 + 1) * E + e] : 0.f;
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(v0, h0, l0);
        split_bf16(v1, h1, l1);
        bhi[n][h] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        blo[n][h] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
      }
    }
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(s_x + st * kDsStageX)) + lofs;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if (m < mtiles) {
        uint32_t a[4];
        ldsm_x4_trans(sbase + m * 32, a);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          mma_16816(acc[m][n], a, bhi[n][0], bhi[n][1]);
          mma_16816(acc[m][n], a, blo[n][0], blo[n][1]);
        }
      }
    }
    done = sidx + 1;
    __syncthreads();  // every warp is done with this stage's buffers
    if (tid == 0 && sidx + kDsStages < n_stages) issue(sidx + kDsStages);
  }
  if (!ok) {
    // let this block's copies in flight land before it exits
    if (tid == 0) {
      report(ctl, MOE_ERR_TIMEOUT, 6);
      for (int sidx = done; sidx < n_stages && sidx < done + kDsStages; ++sidx)
        ds_wait(bar(sidx % kDsStages), static_cast<uint32_t>((sidx / kDsStages) & 1));
    }
    return;
  }
  // C fragments: c0 = (col g, expert 2q), c1 = (g, 2q+1), c2 = (g+8, 2q), c3 = (g+8, 2q+1)
  float* out = partial + static_cast<int64_t>(blockIdx.y) * E * d + col0 + wcol;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m < mtiles) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = 8 * n + 2 * q + (i & 1);
          const int c = 16 * m + g + 8 * (i >> 1);
          if (e < E) out[static_cast<int64_t>(e) * d + c] = acc[m][n][i];
        }
      }
    }
  }
}

template <int NE>
constexpr size_t dw_smem_bytes() {
  return 2 * kDwStageX + 2 * kDwTok * NE * sizeof(float);
}

// dw_out[i] = bf16(sum_p partial[p][i]) over n4_w float4 columns, and, when
// db_out is given, db_out[e] = sum_p db_part[p][e] over n_db rows of E
// floats (the extra columns of the last blocks).  A block owns 32 columns;
// its 32 warps take the rows p = w, w+32, ... and their sums are added in
// warp order, so the result does not depend on timing.
constexpr int kRedWarps = 32;

__global__ void __launch_bounds__(kRedWarps * 32)
    reduce_dw_kernel(const float4* __restrict__ partial, int n_part, int64_t stride4, int64_t n4_w,
                     const float* __restrict__ db_part, int n_db, int E,
                     __nv_bfloat16* __restrict__ dw_out, float* __restrict__ db_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float4 s_part[kRedWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  const int64_t n4 = n4_w + (db_out != nullptr ? (E + 3) / 4 : 0);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (i < n4_w) {
#pragma unroll 4
    for (int p = warp; p < n_part; p += kRedWarps) {
      const float4 v = __ldg(partial + static_cast<int64_t>(p) * stride4 + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  } else if (i < n4) {
    const int e0 = static_cast<int>(i - n4_w) * 4;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int p = warp; p < n_db; p += kRedWarps)
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (e0 + c < E) a[c] += __ldg(db_part + static_cast<int64_t>(p) * E + e0 + c);
    acc = make_float4(a[0], a[1], a[2], a[3]);
  }
  s_part[warp][lane] = acc;
  __syncthreads();
  if (warp != 0 || i >= n4) return;
  float4 r = s_part[0][lane];
#pragma unroll
  for (int w = 1; w < kRedWarps; ++w) {
    const float4 u = s_part[w][lane];
    r.x += u.x; r.y += u.y; r.z += u.z; r.w += u.w;
  }
  if (i < n4_w) {
    reinterpret_cast<uint2*>(dw_out)[i] = make_uint2(pack_bf16x2(r.x, r.y), pack_bf16x2(r.z, r.w));
  } else {
    const int e0 = static_cast<int>(i - n4_w) * 4;
    const float v[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (e0 + c < E) db_out[e0 + c] = v[c];
  }
}

}  // namespace

cudaError_t launch_permute_router_bwd(const __nv_bfloat16* dx_perm, const int32_t* row_map,
                                      const float* dw, const float* probs, const int32_t* idx,
                                      const float* dprob_aux, const __nv_bfloat16* w_r,
                                      const __nv_bfloat16* dx_shared, int T, int d, int E, int k,
                                      bool renorm, __nv_bfloat16* dx, cudaStream_t st) {
  auto go = [&](auto kern, int tpw) {
    const unsigned grid = static_cast<unsigned>(ceil_div64(T, static_cast<int64_t>(kWarps) * tpw));
    (void)launch_pdl(kern, grid, kWarps * 32, 0, st, reinterpret_cast<const uint4*>(dx_perm), row_map, dw, probs,
                                       idx, dprob_aux, w_r,
                                       reinterpret_cast<const uint4*>(dx_shared), T, d, E, k,
                                       renorm ? 1 : 0,
                                       reinterpret_cast<uint4*>(dx));
    return cudaGetLastError();
  };
  auto pick = [&](auto shared_tag) -> cudaError_t {
    constexpr bool S = decltype(shared_tag)::value;
    if (k <= 4) {
      if (E <= 8) return go(permute_router_bwd_kernel<8, 2, 4, S>, 2);
      if (E <= 16) return go(permute_router_bwd_kernel<16, 2, 4, S>, 2);
      if (E <= 32) return go(permute_router_bwd_kernel<32, 1, 4, S>, 1);
      if (E <= 64) return go(permute_router_bwd_kernel<64, 1, 4, S>, 1);
    } else {
      if (E <= 16) return go(permute_router_bwd_kernel<16, 1, 8, S>, 1);
      if (E <= 32) return go(permute_router_bwd_kernel<32, 1, 8, S>, 1);
      if (E <= 64) return go(permute_router_bwd_kernel<64, 1, 8, S>, 1);
    }
    return cudaErrorInvalidValue;
  };
  return dx_shared != nullptr ? pick(std::true_type{}) : pick(std::false_type{});
}

int router_bwd_blocks(int num_sms) { return num_sms * 4; }

cudaError_t launch_router_bwd_dl(const float* dw, const float* probs, const int32_t* idx,
                                 const float* dprob_aux, const __nv_bfloat16* w_r, int T, int d,
                                 int E, int k, bool renorm,
                                 bool fuse_dx, float* dl_f32, __nv_bfloat16* dl_bf16,
                                 int ld_bf16, float* dx_router, float* db_partial, int nblocks,
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
    (void)launch_pdl(kern, nblocks, kWarps * 32, smem, st, dw, probs, idx, dprob_aux, w_r, T, d, E, k,
                                             renorm ? 1 : 0,
                                             dl_f32, dl_bf16, ld_bf16, dx_router, db_partial,
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

namespace {
int dw_blocks_per_sm(int E) { return E <= 16 ? 3 : 2; }
}  // namespace

int router_dw_chunks(int num_sms, int T, int d, int E, int* group_len) {
  if (E <= 16) {  // streamed: one block per SM over all column slices, whole stages
    const int64_t col_blocks = ceil_div64(d, kDsCols);
    int64_t n = ceil_div64(num_sms, col_blocks);
    const int64_t most = ceil_div64(T, kDsTok);
    if (n > most) n = most;
    if (n < 1) n = 1;
    const int64_t len = ceil_div64(ceil_div64(T, n), kDsTok) * kDsTok;
    *group_len = static_cast<int>(len);
    return static_cast<int>(ceil_div64(T, len));
  }
  const int64_t col_blocks = ceil_div64(d, kDwCols);
  // as many blocks as stay resident, over all column blocks; chunks are
  // whole stages
  int64_t n = ceil_div64(static_cast<int64_t>(dw_blocks_per_sm(E)) * num_sms, col_blocks);
  const int64_t most = ceil_div64(T, kDwTok);
  if (n > most) n = most;
  if (n < 1) n = 1;
  const int64_t len = ceil_div64(ceil_div64(T, n), kDwTok) * kDwTok;
  *group_len = static_cast<int>(len);
  return static_cast<int>(ceil_div64(T, len));
}

cudaError_t launch_router_dw(const float* dl, const __nv_bfloat16* x, int T, int d, int E,
                             int n_chunks, int group_len, float* partial, DeviceCtl* ctl,
                             cudaStream_t st) {
  if (E <= 16) {
    auto kern = E <= 8 ? router_dw_stream_kernel<8> : router_dw_stream_kernel<16>;
    if (!set_max_dyn_smem(reinterpret_cast<const void*>(kern), kDsSmem))
      return cudaErrorInvalidValue;
    const unsigned gx = static_cast<unsigned>(ceil_div64(d, kDsCols));
    (void)launch_pdl(kern, dim3(gx, static_cast<unsigned>(n_chunks)), kDsThreads, kDsSmem, st, dl,
                     x, T, d, E, group_len, partial, ctl);
    return cudaGetLastError();
  }
  auto go = [&](auto kern, size_t smem) {
    // several 66-80 KB blocks per SM only fit with the largest shared-memory carve-out
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return cudaErrorInvalidValue;
    const unsigned gx = static_cast<unsigned>(ceil_div64(d, kDwCols));
    (void)launch_pdl(kern, dim3(gx, static_cast<unsigned>(n_chunks)), kDwThreads, smem, st, dl, x, T, d, E,
                                                                              group_len, partial);
    return cudaGetLastError();
  };
  if (E <= 32) return go(router_dw_kernel<32>, dw_smem_bytes<32>());
  if (E <= 64) return go(router_dw_kernel<64>, dw_smem_bytes<64>());
  return cudaErrorInvalidValue;
}

cudaError_t launch_reduce_dw(const float* partial, int n_part, int64_t n_w, const float* db_part,
                             int n_db, int E, __nv_bfloat16* dw_out, float* db_out,
                             cudaStream_t st) {
  // n_w = E * d is a multiple of 4 (d is a multiple of 128)
  const int64_t n4 = n_w / 4 + (db_out != nullptr ? (E + 3) / 4 : 0);
  (void)launch_pdl(reduce_dw_kernel, static_cast<unsigned>(ceil_div64(n4, 32)), kRedWarps * 32, 0, st,
      reinterpret_cast<const float4*>(partial), n_part, n_w / 4, n_w / 4, db_part, n_db, E, dw_out,
      db_out);
  return cudaGetLastError();
}


}  // namespace moe
