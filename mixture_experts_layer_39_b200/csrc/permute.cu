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
// The entries are counted in chunks of kCountTokens tokens (k entries each),
// eight chunks to a block, and ranked and copied in blocks of kChunkTokens
// tokens.
//   count        : a warp per chunk counts its experts; each block writes,
//                  per expert, the prefix of its chunks inside the block and
//                  the block's total; the last block to finish (a ticket in
//                  the handle's control block, no waiting) scans the block
//                  totals per expert and then the padded segment offsets;
//   rank+scatter : a block of 4 warps per 16 tokens: its first warp adds up
//                  the bases (segment start + block base + chunk prefix + the
//                  entries of the chunk before these 16 tokens), walks its
//                  entries 32 at a time (the rank of an entry among equal
//                  experts in a batch comes from __match_any_sync, and the
//                  per-expert running base advances by the batch's count),
//                  then the 4 warps copy the tokens to their rows; blocks
//                  past the tokens zero each segment's pad rows.  Small blocks
//                  keep about 7 resident per SM, so the blocks fill the SMs in
//                  one balanced wave.
#include <climits>

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

// Block b of kWarps warps; warp w counts chunk c = b * kWarps + w.  Scratch:
// pre[e * n_sub + c] = the entries of expert e in the block's chunks before c;
// blk[e * n_blk + b] = the block's total for e, turned by the last block into
// the exclusive scan over blocks (the block's base).  The last block also
// writes counts and the segments' offsets (starts rounded up to `align`
// rows) and resets the ticket for the next launch.
__global__ void __launch_bounds__(kWarps * 32)
    route_count_kernel(const int32_t* __restrict__ idx, int64_t n_entries, int k, int E,
                       int64_t n_sub, int64_t n_blk, int align, int32_t* __restrict__ pre,
                       int32_t* __restrict__ blk, int32_t* __restrict__ counts,
                       int32_t* __restrict__ offsets, DeviceCtl* ctl) {
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
    const int64_t per = static_cast<int64_t>(kCountTokens) * k;
    const int64_t beg = c * per;
    const int64_t end = beg + per < n_entries ? beg + per : n_entries;
    // eight ids per lane in flight at once (a chunk holds at most 64 * 8)
    for (int64_t i0 = beg; i0 < end; i0 += 32 * 8) {
      int ids[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + 32 * u + lane;
        ids[u] = i < end ? __ldg(idx + i) : INT_MIN;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = ids[u];
        if (e == INT_MIN) continue;
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else report(ctl, MOE_ERR_DEVICE_CHECK, 200);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kWarps * 32) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int64_t cw = static_cast<int64_t>(blockIdx.x) * kWarps + w;
      if (cw < n_sub) pre[static_cast<int64_t>(e) * n_sub + cw] = run;
      run += s_cnt[w * E + e];
    }
    blk[static_cast<int64_t>(e) * n_blk + blockIdx.x] = run;
  }
  // publish this block's results, then take a ticket; the last one scans
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_ticket = atomicAdd(&ctl->ticket, 1u);
  __syncthreads();
  if (s_ticket != gridDim.x - 1) return;
  __threadfence();
  // per expert, exclusive scan of the block totals: warp w takes experts
  // w + kWarps * (4g + q), four at a time, each lane a run of 4 blocks of a
  // 128-block segment, so that a segment's loads are all in flight at once
  int* s_tot = s_cnt;  // E totals
  for (int e0 = warp; e0 < E; e0 += 4 * kWarps) {
    int carry[4] = {0, 0, 0, 0};
    for (int64_t s0 = 0; s0 < n_blk; s0 += 128) {
      int v[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * kWarps;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t b = s0 + lane * 4 + u;
          v[q][u] = (e < E && b < n_blk) ? __ldcg(blk + static_cast<int64_t>(e) * n_blk + b) : 0;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * kWarps;
        const int local = v[q][0] + v[q][1] + v[q][2] + v[q][3];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        int run = carry[q] + incl - local;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t b = s0 + lane * 4 + u;
          if (e < E && b < n_blk) blk[static_cast<int64_t>(e) * n_blk + b] = run;
          run += v[q][u];
        }
        carry[q] += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + q * kWarps;
      if (e < E && lane == 0) {
        counts[e] = carry[q];
        s_tot[e] = carry[q];
      }
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

// Blocks [0, n_rs): tokens [16 b, 16 b + 16) -- warp 0 ranks their entries
// into row_map (and shared memory; with row_src non-null it also records the
// token of every row it assigns); then, with SCATTER, the block's warps
// copy each token's row of x to its k rows, two tokens per warp at a time.
// Blocks past n_rs (SCATTER only): warp w of block n_rs + b zero-fills the
// pad rows of expert b * kRsWarps + w (and marks them in row_src with T, when
// given).  An entry with an id outside [0, E)
// gets row -1 (the count kernel recorded MOE_ERR_DEVICE_CHECK) and is not
// copied.
template <bool SCATTER>
__global__ void __launch_bounds__(kRsWarps * 32)
    route_rank_scatter_kernel(const int32_t* __restrict__ idx, const uint4* __restrict__ x,
                              int T, int k, int E, int64_t n_rs, int64_t n_sub, int64_t n_blk,
                              const int32_t* __restrict__ pre, const int32_t* __restrict__ blk,
                              const int32_t* __restrict__ offsets,
                              const int32_t* __restrict__ counts, int nvec,
                              int32_t* __restrict__ row_map, uint4* __restrict__ x_perm,
                              int32_t* __restrict__ row_src) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_base[];  // E running bases, then the block's rows
  int* s_rows = s_base + E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  if (c < n_rs) {
    constexpr int kPerCount = kCountTokens / kChunkTokens;  // rank blocks per count chunk
    const int64_t n_entries = static_cast<int64_t>(T) * k;
    const int64_t per = static_cast<int64_t>(kChunkTokens) * k;
    const int64_t beg = c * per;
    const int64_t end = beg + per < n_entries ? beg + per : n_entries;
    if (warp == 0) {
      const int64_t cc = c / kPerCount, cb = cc / kWarps;  // count chunk, count block
      for (int e = lane; e < E; e += 32)
        s_base[e] = __ldg(offsets + e) + blk[static_cast<int64_t>(e) * n_blk + cb] +
                    pre[static_cast<int64_t>(e) * n_sub + cc];
      __syncwarp();
      // entries of the count chunk that come before this block's tokens (at
      // most 48 tokens: 12 ids per lane, all in flight at once)
      {
        const int64_t i0 = cc * kCountTokens * static_cast<int64_t>(k);
        int ids[12];
#pragma unroll
        for (int u = 0; u < 12; ++u) {
          const int64_t i = i0 + 32 * u + lane;
          ids[u] = i < beg ? __ldg(idx + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < 12; ++u)
          if (ids[u] >= 0 && ids[u] < E) atomicAdd(&s_base[ids[u]], 1);
        for (int64_t i = i0 + 32 * 12 + lane; i < beg; i += 32) {  // k > 8 only
          const int e = __ldg(idx + i);
          if (e >= 0 && e < E) atomicAdd(&s_base[e], 1);
        }
      }
      __syncwarp();
      // the block's ids (16 tokens x k <= 8: at most 128), all loaded before
      // the serial walk
      int ids[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = beg + 32 * u + lane;
        ids[u] = i < end ? __ldg(idx + i) : -1;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i0 = beg + 32 * u;
        if (i0 >= end) break;
        const int64_t i = i0 + lane;
        const bool valid = i < end;
        const int e = valid ? ids[u] : -1;
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
          if (row_src != nullptr && row >= 0) row_src[row] = static_cast<int32_t>(i / k);
        }
      }
    }
    if constexpr (SCATTER) {
      const int64_t t0 = c * kChunkTokens;
      // tokens tt and tt + kRsWarps of the chunk (each may be past T), 128
      // vectors of both at a time: loads first, then the k stores of each
      auto live_of = [&](int tt) { return tt < kChunkTokens && t0 + tt < T; };
      auto load_pair = [&](int tt, int v0, uint4 (&val)[2][4]) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (live_of(tt + h * kRsWarps) && v0 + 32 * u < nvec)
              val[h][u] = __ldg(x + (t0 + tt + h * kRsWarps) * nvec + v0 + 32 * u);
      };
      auto store_pair = [&](int tt, int v0, const uint4 (&val)[2][4]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!live_of(tt + h * kRsWarps)) continue;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j >= k) break;
            const int row = s_rows[(tt + h * kRsWarps) * k + j];
            if (row < 0) continue;
            uint4* dst = x_perm + static_cast<int64_t>(row) * nvec;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[h][u];
          }
        }
      };
      {
        // the first pair's first 128 vectors are loaded before waiting for the
        // ranks, so their latency overlaps warp 0's walk
        uint4 val[2][4];
        load_pair(warp, lane, val);
        __syncthreads();
        store_pair(warp, lane, val);
      }
      for (int v0 = lane + 32 * 4; v0 < nvec; v0 += 32 * 4) {
        uint4 val[2][4];
        load_pair(warp, v0, val);
        store_pair(warp, v0, val);
      }
      for (int tt = warp + 2 * kRsWarps; tt < kChunkTokens; tt += 2 * kRsWarps) {
        for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
          uint4 val[2][4];
          load_pair(tt, v0, val);
          store_pair(tt, v0, val);
        }
      }
    }
  } else if constexpr (SCATTER) {
    const int e = static_cast<int>((c - n_rs) * kRsWarps + warp);
    if (e >= E) return;
    const int64_t r0 = static_cast<int64_t>(__ldg(offsets + e)) + __ldg(counts + e);
    const int64_t r1 = __ldg(offsets + e + 1);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t r = r0; r < r1; ++r)
      for (int v = lane; v < nvec; v += 32) x_perm[r * nvec + v] = z;
    if (row_src != nullptr)  // pad rows hold no token
      for (int64_t r = r0 + lane; r < r1; r += 32) row_src[r] = T;
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
                               int32_t* scratch, int32_t* counts, int32_t* offsets,
                               DeviceCtl* ctl, cudaStream_t st) {
  const int64_t n_sub = count_chunks(T), n_blk = count_blocks(T);
  (void)launch_pdl(route_count_kernel, static_cast<unsigned>(n_blk), kWarps * 32,
                   kWarps * E * sizeof(int), st, idx, static_cast<int64_t>(T) * k, k, E, n_sub,
                   n_blk, align, scratch, scratch + static_cast<int64_t>(E) * n_sub, counts,
                   offsets, ctl);
  return cudaGetLastError();
}

cudaError_t launch_route_rank_scatter(const int32_t* idx, const __nv_bfloat16* x, int T, int k,
                                      int E, const int32_t* scratch, const int32_t* offsets,
                                      const int32_t* counts, int d, int32_t* row_map,
                                      __nv_bfloat16* x_perm, int32_t* row_src, cudaStream_t st) {
  const int64_t n_sub = count_chunks(T), n_blk = count_blocks(T);
  const int64_t n_rs = ceil_div64(T, kChunkTokens);
  const int32_t* pre = scratch;
  const int32_t* blk = scratch + static_cast<int64_t>(E) * n_sub;
  const size_t smem = (static_cast<size_t>(E) + static_cast<size_t>(kChunkTokens) * k) * sizeof(int);
  if (x_perm != nullptr) {
    const unsigned grid = static_cast<unsigned>(n_rs + ceil_div64(E, kRsWarps));
    (void)launch_pdl(route_rank_scatter_kernel<true>, grid, kRsWarps * 32, smem, st, idx,
                     reinterpret_cast<const uint4*>(x), T, k, E, n_rs, n_sub, n_blk, pre, blk,
                     offsets, counts, d / 8, row_map, reinterpret_cast<uint4*>(x_perm), row_src);
  } else {
    (void)launch_pdl(route_rank_scatter_kernel<false>, static_cast<unsigned>(n_rs), kRsWarps * 32,
                     smem, st, idx, static_cast<const uint4*>(nullptr), T, k, E, n_rs, n_sub,
                     n_blk, pre, blk, offsets, counts, d / 8, row_map,
                     static_cast<uint4*>(nullptr), static_cast<int32_t*>(nullptr));
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
