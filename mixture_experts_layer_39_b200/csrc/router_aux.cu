// Router load statistics and the load-balancing loss.
//
// The pages ask for a load-balancing auxiliary loss so that a few hot experts
// do not take most tokens, with a small weight tuned from the spread of
// expert load (discosf.com article on Olmo-core 3, sections 2.2 and 4.3), and
// for load balancing over the global batch (Olmo-core 3 introduction page,
// meetcoding.cn, section 4).  They give no formula.  Reading: the
// Switch-Transformer loss over the k routed slots,
//   f_e = n_e / (N k),  P_e = (sum_t p[t,e]) / N,  loss = alpha E sum_e f_e P_e,
// with f_e held constant (it is piecewise constant in the logits), so that
//   d loss / d p[t,e] = alpha E f_e / N   for every token t.
// The statistics [n | sum_t p] are sums, so a caller can add them over
// micro-batches and ranks (N = all their tokens) before forming the loss.
// Every sum runs in a fixed order.
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kStatWarps = 8;
constexpr int kStatTokensPerBlock = 64;

// partial[b][e] = sum of probs[t][e] over block b's chunk of tokens; warps
// take tokens w, w+8, ... of the chunk and their sums are added in warp order.
template <int NPL>
__global__ void __launch_bounds__(kStatWarps * 32)
    router_stats_partial_kernel(const float* __restrict__ probs, int T, int E, int chunk,
                                float* __restrict__ partial) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_sum[kStatWarps][32 * NPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t t1 = t0 + chunk < T ? t0 + chunk : T;
  float acc[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) acc[i] = 0.f;
  for (int64_t t = t0 + warp; t < t1; t += kStatWarps) {
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) acc[i] += __ldg(probs + t * E + e);
    }
  }
#pragma unroll
  for (int i = 0; i < NPL; ++i) s_sum[warp][lane + 32 * i] = acc[i];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kStatWarps * 32) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kStatWarps; ++w) s += s_sum[w][e];
    partial[static_cast<int64_t>(blockIdx.x) * E + e] = s;
  }
}

// stats[e] (+)= counts[e], stats[E + e] (+)= sum_b partial[b][e]: one warp per
// expert, lanes stride over the partials, then a fixed butterfly.
__global__ void __launch_bounds__(kStatWarps * 32)
    router_stats_final_kernel(const float* __restrict__ partial, int n_part,
                              const int32_t* __restrict__ counts, int E, int accumulate,
                              float* __restrict__ stats) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kStatWarps + (threadIdx.x >> 5);
  if (e >= E) return;
  float s = 0.f;
  for (int p = lane; p < n_part; p += 32) s += partial[static_cast<int64_t>(p) * E + e];
  s = warp_sum(s);
  if (lane == 0) {
    const float n = static_cast<float>(__ldg(counts + e));
    stats[e] = accumulate ? stats[e] + n : n;
    stats[E + e] = accumulate ? stats[E + e] + s : s;
  }
}

// loss = alpha E sum_e f_e P_e and dprob[e] = alpha E f_e / N; one block,
// the products summed in expert order by thread 0.
constexpr int kAuxThreads = 1024;

__global__ void __launch_bounds__(kAuxThreads)
    router_aux_loss_kernel(const float* __restrict__ stats, int E, int k, float n_tokens,
                           float alpha, float* __restrict__ loss, float* __restrict__ dprob) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_prod[kAuxThreads];
  const float slots = n_tokens * static_cast<float>(k);
  for (int e = threadIdx.x; e < E; e += kAuxThreads) {
    const float f = stats[e] / slots;
    const float P = stats[E + e] / n_tokens;
    s_prod[e] = f * P;
    if (dprob != nullptr) dprob[e] = alpha * static_cast<float>(E) * f / n_tokens;
  }
  __syncthreads();
  if (threadIdx.x == 0 && loss != nullptr) {
    float s = 0.f;
    for (int e = 0; e < E; ++e) s += s_prod[e];
    *loss = alpha * static_cast<float>(E) * s;
  }
}

}  // namespace

int router_stats_blocks(int num_sms, int T) {
  const int64_t by_tokens = ceil_div64(T, kStatTokensPerBlock);
  const int64_t most = 2ll * num_sms;
  return static_cast<int>(by_tokens < most ? by_tokens : most);
}

cudaError_t launch_router_load_stats(const float* probs, const int32_t* counts, int T, int E,
                                     int n_blocks, bool accumulate, float* partial, float* stats,
                                     cudaStream_t st) {
  const int chunk = static_cast<int>(ceil_div64(T, n_blocks));
  auto go = [&](auto kern) {
    (void)launch_pdl(kern, static_cast<unsigned>(n_blocks), kStatWarps * 32, 0, st, probs, T, E, chunk, partial);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (E <= 32) e = go(router_stats_partial_kernel<1>);
  else if (E <= 64) e = go(router_stats_partial_kernel<2>);
  else if (E <= 128) e = go(router_stats_partial_kernel<4>);
  else if (E <= 256) e = go(router_stats_partial_kernel<8>);
  else if (E <= 512) e = go(router_stats_partial_kernel<16>);
  else if (E <= 1024) e = go(router_stats_partial_kernel<32>);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  (void)launch_pdl(router_stats_final_kernel, static_cast<unsigned>(ceil_div64(E, kStatWarps)), kStatWarps * 32, 0, st, partial, n_blocks, counts, E, accumulate ? 1 : 0, stats);
  return cudaGetLastError();
}

cudaError_t launch_router_aux_loss(const float* stats, int E, int k, float n_tokens, float alpha,
                                   float* loss, float* dprob, cudaStream_t st) {
  if (E > kAuxThreads) return cudaErrorInvalidValue;
  (void)launch_pdl(router_aux_loss_kernel, 1, kAuxThreads, 0, st, stats, E, k, n_tokens, alpha, loss, dprob);
  return cudaGetLastError();
}

}  // namespace moe
