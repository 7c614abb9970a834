// Routing metadata, rowwise permute, combine and their backwards.
//
// "Routing metadata stays on the GPU, so the host never waits for a copy
// back" and "routed data is written straight into the expert's input
// buffer" -- Olmo-core 3 introduction page, section 2 (GPU-resident routing,
// rowwise expert parallelism).  "The routing result becomes a permutation
// index; tokens are regrouped per expert, processed, then restored to their
// original order" -- discosf.com article, section 2.1.
//
// Metadata is computed in two launches, deterministically, so that the row
// of every (token, slot) entry is exactly the stable expert-major order.
// The entries are cut into chunks of kChunkTokens tokens (k entries each).
//   count        : a warp per chunk counts its experts; the last block to
//                  finish (a ticket in the handle's control block, no
//                  waiting) scans, per expert, over the chunks (the base of
//                  each chunk) and then the padded segment offsets;
//   rank+scatter : a block of 4 warps per chunk: its first warp walks the
//                  chunk 32 entries at a time (the rank of an entry among
//                  equal experts in a batch comes from __match_any_sync, and
//                  the per-expert running base advances by the batch's
//                  count), then the 4 warps copy the chunk's tokens to their
//                  rows; blocks past the chunks zero each segment's pad rows.
//                  Small blocks keep about 7 resident per SM, so the chunks
//                  fill the SMs in one balanced wave.
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kRsWarps = 4;  // warps of a rank+scatter block

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block of kWarps warps; warp w counts chunk blockIdx.x * kWarps + w into
// sub[e * n_sub + c].  The last block to finish then turns sub into each
// chunk's base (exclusive scan over chunks, per expert), writes counts and
// the segments' offsets (starts rounded up to `align` rows) and resets the
// ticket for the next launch.
__global__ void __launch_bounds__(kWarps * 32)
    route_count_kernel(const int32_t* __restrict__ idx, int64_t n_entries, int k, int E,
                       int64_t n_sub, int align, int32_t* __restrict__ sub,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets, DeviceCtl* ctl) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_cnt[];  // kWarps x E (reused by the scan)
  __shared__ unsigned s_ticket;
  __shared__ int s_warp[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* cnt = s_cnt + warp * E;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  if (c < n_sub) {
    const int64_t per = static_cast<int64_t>(kChunkTokens) * k;
    const int64_t beg = c * per;
    const int64_t end = beg + per < n_entries ? beg + per : n_entries;
    for (int64_t i = beg + lane; i < end; i += 32) {
      const int e = __ldg(idx + i);
      if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
      else report(ctl, MOE_ERR_DEVICE_CHECK, 200);
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) sub[static_cast<int64_t>(e) * n_sub + c] = cnt[e];
  }
  // publish this block's counts, then take a ticket; the last one scans
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_ticket = atomicAdd(&ctl->ticket, 1u);
  __syncthreads();
  if (s_ticket != gridDim.x - 1) return;
  __threadfence();
  int* s_tot = s_cnt;  // E totals
  for (int e = warp; e < E; e += kWarps) {
    int32_t* row = sub + static_cast<int64_t>(e) * n_sub;
    int carry = 0;
    for (int64_t base = 0; base < n_sub; base += 32 * 4) {
      int v[4];
      int local = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = base + lane * 4 + u;
        v[u] = i < n_sub ? __ldcg(row + i) : 0;
        local += v[u];
      }
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int run = carry + incl - local;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = base + lane * 4 + u;
        if (i < n_sub) row[i] = run;
        run += v[u];
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      counts[e] = carry;
      s_tot[e] = carry;
    }
  }
  __syncthreads();
  // padded segment starts: thread t takes experts 4t .. 4t+3 (E <= 1024)
  int pad[4], local = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int e = threadIdx.x * 4 + u;
    pad[u] = e < E ? (s_tot[e] + align - 1) / align * align : 0;
    local += pad[u];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s_warp[w];
  int run = before + incl - local;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int e = threadIdx.x * 4 + u;
    if (e < E) offsets[e] = run;
    run += pad[u];
    if (e == E - 1) offsets[E] = run;
  }
  if (threadIdx.x == 0) ctl->ticket = 0u;
}

// Blocks [0, n_sub): chunk c -- warp 0 ranks its entries into row_map (and
// shared memory); then, with SCATTER, the block's warps copy each token's
// row of x to its k rows, two tokens per warp at a time.  Blocks past
// n_sub (SCATTER only): warp w of block n_sub + b zero-fills the pad rows
// of expert b * kRsWarps + w.  An entry with an id outside [0, E) gets row -1
// (the count kernel recorded MOE_ERR_DEVICE_CHECK) and is not copied.
template <bool SCATTER>
__global__ void __launch_bounds__(kRsWarps * 32)
    route_rank_scatter_kernel(const int32_t* __restrict__ idx, const uint4* __restrict__ x,
                              int T, int k, int E, int64_t n_sub,
                              const int32_t* __restrict__ sub_base,
                              const int32_t* __restrict__ offsets,
                              const int32_t* __restrict__ counts, int nvec,
                              int32_t* __restrict__ row_map, uint4* __restrict__ x_perm) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_base[];  // E running bases, then the chunk's rows
  int* s_rows = s_base + E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  if (c < n_sub) {
    const int64_t n_entries = static_cast<int64_t>(T) * k;
    const int64_t per = static_cast<int64_t>(kChunkTokens) * k;
    const int64_t beg = c * per;
    const int64_t end = beg + per < n_entries ? beg + per : n_entries;
    if (warp == 0) {
      for (int e = lane; e < E; e += 32)
        s_base[e] = __ldg(offsets + e) + sub_base[static_cast<int64_t>(e) * n_sub + c];
      __syncwarp();
      for (int64_t i0 = beg; i0 < end; i0 += 32) {
        const int64_t i = i0 + lane;
        const bool valid = i < end;
        const int e = valid ? __ldg(idx + i) : -1;
        const bool good = valid && e >= 0 && e < E;
        const int key = good ? e : -1 - lane;  // lanes without an expert match only themselves
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        int row = -1;
        if (good) row = s_base[e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (good && (peers & lanemask_lt()) == 0) s_base[e] += __popc(peers);
        __syncwarp();
        if (valid) {
          row_map[i] = row;
          s_rows[i - beg] = row;
        }
      }
    }
    if constexpr (SCATTER) {
      __syncthreads();
      const int64_t t0 = c * kChunkTokens;
      for (int tt = warp; tt < kChunkTokens; tt += 2 * kRsWarps) {
        // tokens tt and tt + kRsWarps of the chunk (each may be past T)
        int rows[2][8];
        bool live[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t t = t0 + tt + h * kRsWarps;
          live[h] = tt + h * kRsWarps < kChunkTokens && t < T;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            rows[h][j] = (live[h] && j < k) ? s_rows[(tt + h * kRsWarps) * k + j] : -1;
        }
        for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
          uint4 val[2][4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (live[h] && v0 + 32 * u < nvec)
                val[h][u] = __ldg(x + (t0 + tt + h * kRsWarps) * nvec + v0 + 32 * u);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (rows[h][j] < 0) continue;
              uint4* dst = x_perm + static_cast<int64_t>(rows[h][j]) * nvec;
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[h][u];
            }
        }
      }
    }
  } else if constexpr (SCATTER) {
    const int e = static_cast<int>((c - n_sub) * kRsWarps + warp);
    if (e >= E) return;
    const int64_t r0 = static_cast<int64_t>(__ldg(offsets + e)) + __ldg(counts + e);
    const int64_t r1 = __ldg(offsets + e + 1);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t r = r0; r < r1; ++r)
      for (int v = lane; v < nvec; v += 32) x_perm[r * nvec + v] = z;
  }
}

// row_src[r] = the token whose copy routed row r holds, for the expert GEMMs
// that gather their rows from x instead of reading x_perm.  Threads [0, T k)
// take one (token, slot) each; threads [T k, T k + m_cap) take routed row
// r = i - T k and write oob (a row index past x, which the gather loads read
// as zeros) when r is a pad row or lies past the last segment.  The two sets
// of rows are disjoint, so the kernel needs no ordering.
__global__ void __launch_bounds__(256)
    route_src_kernel(const int32_t* __restrict__ row_map, const int32_t* __restrict__ offsets,
                     const int32_t* __restrict__ counts, int T, int k, int E, int64_t m_cap,
                     int32_t oob, int32_t* __restrict__ row_src) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t tk = static_cast<int64_t>(T) * k;
  if (i < tk) {
    // an entry whose expert id was out of range has row -1 (the rank kernel
    // skipped it and the histogram recorded MOE_ERR_DEVICE_CHECK): no row
    const int32_t r = __ldg(row_map + i);
    if (r >= 0) row_src[r] = static_cast<int32_t>(i / k);
    return;
  }
  const int64_t r = i - tk;
  if (r >= m_cap) return;
  if (r >= __ldg(offsets + E)) {
    row_src[r] = oob;
    return;
  }
  int lo = 0, hi = E - 1;  // the segment holding r: the last e with offsets[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= r) lo = mid; else hi = mid - 1;
  }
  if (r >= static_cast<int64_t>(__ldg(offsets + lo)) + __ldg(counts + lo)) row_src[r] = oob;
}

// y[t] = bf16(sum_j w[t,j] * O[row_map[t,j]] + shared[t]), fp32 in slot order, the
// shared expert's output (when given) last.
template <bool SHARED>
__global__ void __launch_bounds__(kWarps * 32, 2)
    combine_kernel(const uint4* __restrict__ o, const int32_t* __restrict__ row_map,
                   const float* __restrict__ w, const uint4* __restrict__ shared, int T, int nvec,
                   int k, uint4* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[8];
  float wt[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    rows[j] = j < k ? __ldg(row_map + t * k + j) : -1;
    wt[j] = j < k ? __ldg(w + t * k + j) : 0.f;
  }
  for (int v0 = lane; v0 < nvec; v0 += 64) {
    float acc[2][8];
    uint4 q[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (rows[j] >= 0 && v0 + 32 * u < nvec)
          q[u][j] = __ldg(o + static_cast<int64_t>(rows[j]) * nvec + v0 + 32 * u);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[u][c] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (rows[j] < 0) continue;
        float f[8];
        unpack8(q[u][j], f);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[u][c] = fmaf(wt[j], f[c], acc[u][c]);
      }
      if (v0 + 32 * u >= nvec) continue;
      if constexpr (SHARED) {  // the shared expert's output, added last
        float f[8];
        unpack8(__ldg(shared + t * nvec + v0 + 32 * u), f);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[u][c] += f[c];
      }
      y[t * nvec + v0 + 32 * u] = pack8(acc[u]);
    }
  }
}

// dO[row_map[t,j]] = bf16(w * dY[t]); dw[t,j] = <dY[t], O[row_map[t,j]]>;
// warps past T zero the pad rows of dO.
__global__ void __launch_bounds__(kWarps * 32, 3)
    combine_bwd_kernel(const uint4* __restrict__ dy, const uint4* __restrict__ o,
                       const int32_t* __restrict__ row_map, const float* __restrict__ w,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts,
                       int T, int nvec, int k, int E, uint4* __restrict__ dO,
                       float* __restrict__ dw) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (gw < T) {
    const int64_t t = gw;
    int rows[8];
    float wt[8], part[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rows[j] = j < k ? __ldg(row_map + t * k + j) : -1;
      wt[j] = j < k ? __ldg(w + t * k + j) : 0.f;
      part[j] = 0.f;
    }
    for (int v = lane; v < nvec; v += 32) {
      float g[8];
      unpack8(__ldg(dy + t * nvec + v), g);
      uint4 q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (rows[j] >= 0) q[j] = __ldg(o + static_cast<int64_t>(rows[j]) * nvec + v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (rows[j] < 0) continue;
        float f[8], s[8];
        unpack8(q[j], f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          part[j] = fmaf(g[c], f[c], part[j]);
          s[c] = wt[j] * g[c];
        }
        dO[static_cast<int64_t>(rows[j]) * nvec + v] = pack8(s);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      const float r = warp_sum(part[j]);
      if (lane == 0) dw[t * k + j] = r;
    }
  } else if (gw < static_cast<int64_t>(T) + E) {
    const int e = static_cast<int>(gw - T);
    const int64_t r0 = static_cast<int64_t>(__ldg(offsets + e)) + __ldg(counts + e);
    const int64_t r1 = __ldg(offsets + e + 1);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t r = r0; r < r1; ++r)
      for (int v = lane; v < nvec; v += 32) dO[r * nvec + v] = z;
  }
}

// dX[t] = bf16(sum_j dX_perm[row_map[t,j]] + dX_router[t] + dX_shared[t]), fp32,
// rounded once (the last two terms when given).
template <bool SHARED>
__global__ void __launch_bounds__(kWarps * 32)
    permute_bwd_kernel(const uint4* __restrict__ dxp, const int32_t* __restrict__ row_map,
                       const float4* __restrict__ dxr, const uint4* __restrict__ dxs, int T,
                       int nvec, int k, uint4* __restrict__ dx) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) rows[j] = j < k ? __ldg(row_map + t * k + j) : -1;
  for (int v = lane; v < nvec; v += 32) {
    uint4 q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (rows[j] >= 0) q[j] = __ldg(dxp + static_cast<int64_t>(rows[j]) * nvec + v);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (rows[j] < 0) continue;
      float f[8];
      unpack8(q[j], f);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += f[c];
    }
    if (dxr != nullptr) {
      const float4 a = __ldg(dxr + (t * nvec + v) * 2);
      const float4 b = __ldg(dxr + (t * nvec + v) * 2 + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    if constexpr (SHARED) {  // the shared expert's input gradient, added last
      float f[8];
      unpack8(__ldg(dxs + t * nvec + v), f);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += f[c];
    }
    dx[t * nvec + v] = pack8(acc);
  }
}

}  // namespace

cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int align,
                               int32_t* sub_counts, int32_t* counts, int32_t* offsets,
                               DeviceCtl* ctl, cudaStream_t st) {
  const int64_t n_sub = n_subchunks(T, k);
  const unsigned grid = static_cast<unsigned>(ceil_div64(n_sub, kWarps));
  (void)launch_pdl(route_count_kernel, grid, kWarps * 32, kWarps * E * sizeof(int), st, idx,
                   static_cast<int64_t>(T) * k, k, E, n_sub, align, sub_counts, counts, offsets, ctl);
  return cudaGetLastError();
}

cudaError_t launch_route_rank_scatter(const int32_t* idx, const __nv_bfloat16* x, int T, int k,
                                      int E, const int32_t* sub_base, const int32_t* offsets,
                                      const int32_t* counts, int d, int32_t* row_map,
                                      __nv_bfloat16* x_perm, cudaStream_t st) {
  const int64_t n_sub = n_subchunks(T, k);
  const size_t smem = (static_cast<size_t>(E) + static_cast<size_t>(kChunkTokens) * k) * sizeof(int);
  if (x_perm != nullptr) {
    const unsigned grid = static_cast<unsigned>(n_sub + ceil_div64(E, kRsWarps));
    (void)launch_pdl(route_rank_scatter_kernel<true>, grid, kRsWarps * 32, smem, st, idx,
                     reinterpret_cast<const uint4*>(x), T, k, E, n_sub, sub_base, offsets, counts,
                     d / 8, row_map, reinterpret_cast<uint4*>(x_perm));
  } else {
    (void)launch_pdl(route_rank_scatter_kernel<false>, static_cast<unsigned>(n_sub), kRsWarps * 32,
                     smem, st, idx, static_cast<const uint4*>(nullptr), T, k, E, n_sub, sub_base,
                     offsets, counts, d / 8, row_map, static_cast<uint4*>(nullptr));
  }
  return cudaGetLastError();
}

cudaError_t launch_route_src(const int32_t* row_map, const int32_t* offsets, const int32_t* counts,
                             int T, int k, int E, int64_t m_cap, int32_t* row_src,
                             cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(T) * k + m_cap;
  (void)launch_pdl(route_src_kernel, static_cast<unsigned>(ceil_div64(n, 256)), 256, 0, st,
      row_map, offsets, counts, T, k, E, m_cap, T, row_src);
  return cudaGetLastError();
}

cudaError_t launch_combine(const __nv_bfloat16* o_perm, const int32_t* row_map, const float* w,
                           const __nv_bfloat16* shared, int T, int d, int k, __nv_bfloat16* y,
                           cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(T, kWarps));
  auto kern = shared != nullptr ? combine_kernel<true> : combine_kernel<false>;
  (void)launch_pdl(kern, grid, kWarps * 32, 0, st, reinterpret_cast<const uint4*>(o_perm), row_map, w,
                                     reinterpret_cast<const uint4*>(shared), T, d / 8, k,
                                     reinterpret_cast<uint4*>(y));
  return cudaGetLastError();
}

cudaError_t launch_combine_bwd(const __nv_bfloat16* dy, const __nv_bfloat16* o_perm,
                               const int32_t* row_map, const float* w, const int32_t* offsets,
                               const int32_t* counts, int T, int d, int k, int E,
                               __nv_bfloat16* do_perm, float* dw, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(static_cast<int64_t>(T) + E, kWarps));
  (void)launch_pdl(combine_bwd_kernel, grid, kWarps * 32, 0, st,
      reinterpret_cast<const uint4*>(dy), reinterpret_cast<const uint4*>(o_perm), row_map, w,
      offsets, counts, T, d / 8, k, E, reinterpret_cast<uint4*>(do_perm), dw);
  return cudaGetLastError();
}

cudaError_t launch_permute_bwd(const __nv_bfloat16* dx_perm, const int32_t* row_map,
                               const float* dx_router, const __nv_bfloat16* dx_shared, int T, int d,
                               int k, __nv_bfloat16* dx, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div64(T, kWarps));
  auto kern = dx_shared != nullptr ? permute_bwd_kernel<true> : permute_bwd_kernel<false>;
  (void)launch_pdl(kern, grid, kWarps * 32, 0, st,
      reinterpret_cast<const uint4*>(dx_perm), row_map, reinterpret_cast<const float4*>(dx_router),
      reinterpret_cast<const uint4*>(dx_shared), T, d / 8, k, reinterpret_cast<uint4*>(dx));
  return cudaGetLastError();
}

}  // namespace moe
