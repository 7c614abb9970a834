// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, for sm_100a.
//
// "Grouped GEMM: merge the many small expert GEMMs into one launch so the
// GPU stays busy" and "device-scheduled grouped GEMM" -- Olmo-core 3
// introduction page, section 2 (three routing optimisations).  Here the
// schedule is decoded on the device from the expert offsets, so routing
// never forces a device-to-host copy.
//
// One CTA per SM, 6 warps:
//   warp 0      TMA producer (one lane): A/B tiles into a STAGES-deep ring
//   warp 1      MMA issuer (one lane): tcgen05.mma 128 x BN x 16, fp32 in TMEM;
//               also owns the TMEM allocation
//   warps 2..5  epilogue: tcgen05.ld from TMEM -> registers -> global
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap
// the main loop of tile i+1.
//
// Two grouping modes:
//   M-grouped (KGROUP=false): rows of A are split in groups (experts); group
//     g owns rows [off(g), off(g+1)) and multiplies B[g].  Tiles are 128-row
//     slices of a group; rows past off(g+1) are masked at the store.
//   K-grouped (KGROUP=true, weight gradients): group g owns the contraction
//     range [off(g), off(g+1)) and writes its own output matrix g.  A group
//     with an empty range writes zeros.
//
// Operand layouts in shared memory are the canonical 128-byte-swizzled
// UMMA layouts: K-major = rows of 64 bf16 along K (TMA box {64, rows});
// MN-major = 64-element chunks along M/N, one 128-byte row per K index (TMA
// box {64, 64}), chunks 8 KB apart.
//
// Every mbarrier wait is bounded (globaltimer).  The waits of the main loops
// give up after GemmArgs::wait_ns (the handle's limit, 2 s unless changed);
// the CTA then records MOE_ERR_TIMEOUT, drains its own TMA copies and MMAs
// (those drain waits always allow kWaitLimitNs), frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;  // bf16 elements per smem row: 128 bytes = one swizzle row
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// EPI_BF16_COMBINE: the down projection with the unpermute-combine fused into
// its epilogue (see the epilogue below).
enum Epi : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_SWIGLU_FWD = 2, EPI_SWIGLU_BWD = 3,
                 EPI_BF16_COMBINE = 4 };

struct GemmArgs {
  int n_tiles_n;     // tiles along N per (group, m-tile)
  int n_cols;        // columns of the output (N); the last N tile may run past it
  int m_rows;        // K-grouped: rows of each group's output (M); the last M tile
                     // may run past it (operand rows past it read as TMA zero fill)
  int k_blocks;      // M-grouped: contraction length / BK
  int n_groups;
  const int* offsets;  // [n_groups + 1] on the device, or nullptr: uniform groups
  int uniform_len;     // group length when offsets == nullptr
  int total_len;       // clamp of all group boundaries (rows of the grouped operand)
  int m_tiles_fixed;   // K-grouped: M / BM
  // K-grouped: with tile_end > 0 the launch takes tiles [tile_begin, tile_end)
  // of the full tile list only (a weight gradient's last wave as its own launch)
  int tile_begin, tile_end;
  int64_t m_cap;       // M-grouped: rows of the output buffer (store bound)
  void* out;
  int64_t ldo;
  int64_t out_gstride;  // K-grouped: elements between group outputs
  void* out2;           // SwiGLU forward: H
  int64_t ldo2;
  const __nv_bfloat16* aux;  // SwiGLU backward: saved [A | U]
  int64_t ld_aux;
  int f;  // SwiGLU: width of one half ([A | U] column offset of U)
  DeviceCtl* ctl;
  uint64_t wait_ns;  // limit of the main loops' waits; 0: give up unless already complete
  // GATHER: the operand that holds routed rows is read from the unpermuted
  // matrix (x), routed row r being its row row_src[r]; rows past m_cap and
  // pad rows use src_oob, a row past the matrix that reads as zeros
  const int32_t* row_src;
  int src_oob;
  // EPI_BF16_COMBINE: row_src[r] = the token of routed row r (T on pad rows);
  // y [T, n_cols] = bf16(sum_j topk_w[t, j] out[row_map[t, j]] (+ shared[t]));
  // arrivals [T, n_tiles_n] int32, zero on entry and on return
  const int32_t* row_map;
  const float* topk_w;
  const __nv_bfloat16* shared;
  __nv_bfloat16* y;
  int32_t* arrivals;
  int n_tok, top_k;
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase completed; false when another role
// aborted or `limit_ns` passed (then the abort flag is raised).  A limit of
// 0 gives up at once unless the first test finds the phase complete.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity);

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns, bool honour_abort = true,
                                          bool cluster_scope = false) {
  auto poll = [&]() {
    return cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (poll()) return true;
  if (limit_ns == 0) {
    *abort_flag = 1;
    return false;
  }
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (poll()) return true;
    if (honour_abort && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// ---- CTA-pair (cta_group::2) helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrival on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// Bounded wait with cluster-scope acquire (barriers that receive arrivals from the peer CTA).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Tile loads of a CTA pair: the completion bytes go to the mbarrier `bar`,
// which may live in either CTA of the pair (plain loads, one destination).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// One 512-byte scale atom (box {128, 4, 1, 1, 1} of a 5-D map over the
// atom-ordered scales: coordinates (0, 0, K block, MN block, group)); the
// completion bytes go to `bar`, which may live in either CTA of the pair.
__device__ __forceinline__ void tma_load_atom_pair(uint32_t dst, const CUtensorMap* map,
                                                   uint32_t bar, int kb, int rb, int g) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(kb), "r"(rb), "r"(g), "r"(bar)
      : "memory");
}

// Four rows (r0..r3, any order) x one box of columns from c0, into 4
// consecutive 128-byte rows at dst (the tensor map's box is one row high).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_gather4_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::"
      "complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives (once the pair's prior MMAs completed) on the barrier at this
// shared-memory offset in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(static_cast<uint16_t>(3))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout code 2),
// descriptor version 1 at bits 46-47; addresses and offsets in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 inputs and fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                       // D format fp32
         | (1u << 7)                     // A format bf16
         | (1u << 10)                    // B format bf16
         | ((a_mn ? 1u : 0u) << 15)      // A major
         | ((b_mn ? 1u : 0u) << 16)      // B major
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem),
      "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::mxf8f6f4 (block-scaled): E4M3 A and B, E8M0
// scales (bit 23), K = 32 per MMA.  The scale-factor ids (bits 4-5 for B,
// 29-30 for A) select the byte of each 32-bit scale word and are or-ed in
// per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, bool a_mn, bool b_mn) {
  return ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         (1u << 23) | ((uint32_t)(M >> 4) << 24);
}

// One 512-byte scale atom (32 rows x 16 bytes, no swizzle: 8-row groups 128 B
// apart) from shared memory into 4 TMEM columns, copied to all four lane
// quarters; issued by the pair's leader, each CTA's atom (same shared-memory
// offset) lands in that CTA's TMEM.
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(512u >> 4) << 16;   // leading byte offset (unused at 16 B width)
  d |= static_cast<uint64_t>(128u >> 4) << 32;   // stride byte offset: 8 rows x 16 B
  d |= static_cast<uint64_t>(1) << 46;           // descriptor version
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns of TMEM.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive fp32 columns of TMEM.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Logistic function for the SwiGLU epilogues: sigma(z) = 1/2 + tanh(z/2)/2,
// with the hardware tanh approximation (PTX tanh.approx.f32, relative error
// about 2^-11: below the bf16 rounding the outputs take anyway).  One MUFU
// operation instead of an exponential plus an IEEE division.
__device__ __forceinline__ float sigmoid_fast(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return fmaf(0.5f, t, 0.5f);
}

// ---------------------------------------------------------------- scheduling
struct Tile {
  int m64;      // M-grouped tail tile with at most 64 rows: issued as M = 64 MMAs
  int group;
  int row0;     // M-grouped: first row of the tile; K-grouped: first row of M
  int row_end;  // M-grouped: end of the group's rows (store mask)
  int n_tile;
  int k_lo;     // K-grouped: first contraction row
  int k_blocks;
  int last_k16;  // MMAs of K=16 in the last k-block (1..4)
};

__device__ __forceinline__ int group_off(const GemmArgs& a, int g) {
  int v;
  if (a.offsets != nullptr) {
    v = __ldg(a.offsets + g);
  } else {
    long long u = static_cast<long long>(g) * a.uniform_len;
    v = static_cast<int>(u < a.total_len ? u : a.total_len);
  }
  v = v < 0 ? 0 : v;
  return v > a.total_len ? a.total_len : v;
}

template <bool KGROUP, int BKE = BK, int KMMA = 16, int MT = BM>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, const int* s_tile_start, int t) {
  Tile tl;
  if constexpr (!KGROUP) {
    const int mt = t / a.n_tiles_n;
    tl.n_tile = t - mt * a.n_tiles_n;
    int lo = 0, hi = a.n_groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tile_start[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    tl.group = lo;
    const int g0 = group_off(a, lo), g1 = group_off(a, lo + 1);
    tl.row0 = g0 + (mt - s_tile_start[lo]) * MT;
    tl.row_end = g1 > g0 ? g1 : g0;
    tl.m64 = (tl.row_end - tl.row0) <= 64 ? 1 : 0;
    tl.k_lo = 0;
    tl.k_blocks = a.k_blocks;
    tl.last_k16 = 4;
  } else {
    const int per = a.m_tiles_fixed * a.n_tiles_n;
    tl.group = t / per;
    const int r = t - tl.group * per;
    const int mt = r / a.n_tiles_n;
    tl.n_tile = r - mt * a.n_tiles_n;
    tl.row0 = mt * MT;
    tl.row_end = 0;
    tl.m64 = 0;
    const int g0 = group_off(a, tl.group), g1 = group_off(a, tl.group + 1);
    const int len = g1 > g0 ? g1 - g0 : 0;
    tl.k_lo = g0;
    tl.k_blocks = (len + BKE - 1) / BKE;
    const int rem = len - (tl.k_blocks - 1) * BKE;
    tl.last_k16 = tl.k_blocks > 0 ? (rem + KMMA - 1) / KMMA : 0;
  }
  return tl;
}

// ---------------------------------------------------------------- epilogue helpers
// Each epilogue warp owns 32 consecutive tile rows (its TMEM lane quarter)
// and a 4 KB staging buffer: 32 rows x 128 bytes, 16-byte slots swizzled by
// row (slot q of row r at q ^ (r & 7)) so that both access patterns below
// are free of bank conflicts.
//   row side       : lane r reads/writes the 8 slots of row r;
//   coalesced side : lane i touches row 4j + i/8, slot i%8, so one warp
//                    instruction moves four full 128-byte row segments.
constexpr int kStageRowBytes = 128;
constexpr int kEpiBufBytes = 32 * kStageRowBytes;

__device__ __forceinline__ uint4* stage_slot(uint8_t* buf, int row, int q) {
  return reinterpret_cast<uint4*>(buf + row * kStageRowBytes + ((q ^ (row & 7)) << 4));
}

__device__ __forceinline__ void stage_write_row(uint8_t* buf, int lane, const uint4 (&v)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) *stage_slot(buf, lane, q) = v[q];
}

__device__ __forceinline__ void stage_read_row(uint8_t* buf, int lane, uint4 (&v)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = *stage_slot(buf, lane, q);
}

__device__ __forceinline__ void stage_to_global(uint8_t* buf, uint8_t* g, int64_t ld_bytes,
                                                int valid_rows, int lane) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int row = 4 * j + (lane >> 3);
    const uint4 v = *stage_slot(buf, row, lane & 7);
    if (row < valid_rows)
      *reinterpret_cast<uint4*>(g + row * ld_bytes + ((lane & 7) << 4)) = v;
  }
}

// Writes this lane's 128-byte row `v` through the staging buffer to global.
__device__ __forceinline__ void store_rows(uint8_t* buf, int lane, const uint4 (&v)[8], uint8_t* g,
                                           int64_t ld_bytes, int valid_rows) {
  stage_write_row(buf, lane, v);
  __syncwarp();
  stage_to_global(buf, g, ld_bytes, valid_rows, lane);
  __syncwarp();
}

// 64 fp32 -> 64 bf16 (128 bytes)
__device__ __forceinline__ void pack64(const float* f, uint4 (&v)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    v[q] = make_uint4(pack_bf16x2(f[8 * q + 0], f[8 * q + 1]), pack_bf16x2(f[8 * q + 2], f[8 * q + 3]),
                      pack_bf16x2(f[8 * q + 4], f[8 * q + 5]), pack_bf16x2(f[8 * q + 6], f[8 * q + 7]));
}

// SwiGLU backward: 32 columns of the saved A (slots 0-3 of each staging row)
// and the same 32 columns of U (slots 4-7) for the warp's 32 rows, copied
// asynchronously; rows past valid_rows are zero-filled.
__device__ __forceinline__ void cp_async_au(uint8_t* buf, const uint8_t* ga, const uint8_t* gu,
                                            int64_t ld_bytes, int valid_rows, int lane,
                                            const void* safe) {
  const int q = lane & 7;
  const uint8_t* g = q < 4 ? ga + (q << 4) : gu + ((q - 4) << 4);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int row = 4 * j + (lane >> 3);
    const bool ok = row < valid_rows;
    const uint8_t* src = ok ? g + row * ld_bytes : static_cast<const uint8_t*>(safe);
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(stage_slot(buf, row, q)));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(ok ? 16 : 0)
                 : "memory");
  }
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------- the kernel
template <int BN, int STAGES, int EPI, bool FP8 = false, bool PAIR = false>
struct SmemPlan {
  // one stage holds 128-byte rows: 64 bf16 or 128 fp8 contraction elements;
  // in a CTA pair each CTA holds half of B's BN rows
  static constexpr int kABytes = BM * 128;
  static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // MXFP8 (CTA pairs): per stage and CTA one 512-byte scale atom for its own
  // 128 rows of A and one per 128 of the pair's BN rows of B
  static constexpr int kSfStageBytes = FP8 ? 512 * (1 + BN / 128) : 0;
  static constexpr int kSfOff = STAGES * kStageBytes;
  static constexpr int kBarOff = kSfOff + STAGES * kSfStageBytes;      // 1024-aligned stages
  static constexpr int kBarBytes = (2 * STAGES + 5) * 8;               // full, empty, tfull x2, tempty x2, drain
  static constexpr int kMiscOff = kBarOff + kBarBytes;                 // tmem base, abort flag
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) / 128 * 128;    // 4 epilogue warps' buffers
  // per warp: the 4 KB staging buffer, plus (SwiGLU backward) a 4 KB landing
  // buffer that cp.async fills with the next 32 columns of the saved A and U
  static constexpr int kWarpEpiBytes = kEpiBufBytes + (EPI == EPI_SWIGLU_BWD ? kEpiBufBytes : 0);
  static constexpr int kTileOff = kEpiOff + 4 * kWarpEpiBytes;         // group tile starts
  static constexpr int bytes(int n_groups) { return 1024 + kTileOff + 4 * (n_groups + 1); }
};

// PAIR: a cluster of two CTAs computes a 256 x BN tile with tcgen05.mma
// cta_group::2 (M = 256).  Each CTA loads its own 128 rows of A and half of
// B's BN rows; the even CTA (leader) waits for both CTAs' bytes on its full
// barrier, issues the MMAs and commits to both CTAs' barriers; each CTA's
// TMEM holds its own 128 accumulator rows, so the epilogue is unchanged, and
// the odd CTA's epilogue warps release the accumulator on the leader's
// barrier.
//
// MXFP8 (FP8 = true) always runs on CTA pairs with 256 x 256 tiles and 128
// contraction elements per stage.  The E8M0 scales come from arrays in the
// tensor cores' 512-byte atom order (tmSA, tmSB: 5-D maps, one atom per
// (128 MN indices, 128 contraction elements)): each CTA loads the atom of
// its own 128 A rows and both atoms of the pair's 256 B rows with pair TMA
// loads that complete on the leader's full barrier; the leader copies them
// to TMEM (tcgen05.cp.cta_group::2, each CTA's atoms into its own TMEM) and
// issues block-scaled pair MMAs.  TMEM then holds one 256-column accumulator
// and two alternating scale buffers.
template <int BN, bool A_MN, bool B_MN, int EPI, bool KGROUP, int STAGES, bool FP8 = false,
          bool PAIR = false, bool GATHER = false>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmSA,
                        const __grid_constant__ CUtensorMap tmSB, const GemmArgs args) {
  static_assert(BN == 128 || BN == 256 || (BN == 512 && PAIR), "BN");
  static_assert(!(EPI == EPI_SWIGLU_FWD && B_MN), "SwiGLU forward takes K-major weights");
  static_assert(!FP8 || (PAIR && BN == 256), "MXFP8 runs 256 x 256 CTA-pair tiles");
  static_assert(!PAIR || BN >= 256, "CTA pairs run 256 x 256 or 256 x 512 tiles");
  // GATHER reads routed rows from x: the K-major A of an M-grouped GEMM, or
  // the MN-major B (rows = routed rows) of a K-grouped one
  static_assert(!GATHER || (!FP8 && (KGROUP ? B_MN : !A_MN)), "gathered operand");
  // K-grouped GATHER runs on CTA pairs: one 4-row gather per lane per stage
  static_assert(!GATHER || !KGROUP || (PAIR && (BN / 2 / (FP8 ? 128 : 64)) * (BK / 4) == 32),
                "K-grouped gather layout");
  using Plan = SmemPlan<BN, STAGES, EPI, FP8, PAIR>;
  constexpr int MT = PAIR ? 2 * BM : BM;  // tile rows (of the pair)
  constexpr int BNC = PAIR ? BN / 2 : BN;  // B rows held by one CTA
  // contraction elements per stage, per MMA, per 128-byte MN chunk of an MN-major operand
  constexpr int BKE = FP8 ? 128 : BK;
  constexpr int KMMA = FP8 ? 32 : 16;
  constexpr int CH = FP8 ? 128 : 64;
  constexpr uint32_t kChunkBytes = BKE * 128;      // one MN chunk of an MN-major stage
  constexpr uint32_t kSfCols = 4 + 4 * (BN / 128); // TMEM columns of one scale buffer
  constexpr uint32_t kSfTmaBytes = FP8 ? 512 * (1 + BN / 128) : 0;  // scale atoms per stage, per CTA
  // Wide pairs (BN = 512): two N = 256 MMAs per K step, each reading 128 of
  // every CTA's 256 B rows, into one accumulator that fills TMEM (the
  // epilogue of a tile then does not overlap the next tile's MMAs).  MXFP8
  // pairs also keep one accumulator: the scale buffers need TMEM too.
  constexpr int NMMA = BN > 256 ? 256 : BN;  // N of one MMA instruction
  constexpr int NACC = (BN > 256 || FP8) ? 1 : 2;  // TMEM accumulators
  constexpr uint32_t kBHalfBytes = (BNC / 2) * 128;  // B rows of one wide-pair MMA, per CTA
  constexpr uint32_t kTmemCols = FP8 ? 512 : NACC * BN;
  constexpr uint32_t kIdesc = FP8 ? idesc_mxf8(MT, BN, A_MN, B_MN) : idesc_bf16(MT, NMMA, A_MN, B_MN);
  // M-grouped bf16 tail tiles of <= 64 rows run M = 64 MMAs: rows 16q..16q+15
  // of the accumulator then sit in TMEM lanes 32q..32q+15
  constexpr bool kTail64 = !FP8 && !KGROUP && !A_MN && !PAIR;
  constexpr uint32_t kIdesc64 = idesc_bf16(64, BN, A_MN, B_MN);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Plan::kMiscOff + 4);
  int* s_tile_start = reinterpret_cast<int*>(smem + Plan::kTileOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // CTA within the pair
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };
  auto tfull_bar = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
  auto tempty_bar = [&](int b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * STAGES + 4]);

  // ---- set-up: barriers, TMEM, group tile starts
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PAIR ? 8 : 4);  // epilogue warps of one or both CTAs
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if constexpr (FP8) {
      prefetch_tmap(&tmSA);
      prefetch_tmap(&tmSB);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(s_tmem)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(s_tmem)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  // everything above touched only shared memory, TMEM and kernel parameters;
  // the previous kernel's outputs (offsets, operands) are read from here on
  pdl_wait();
  pdl_trigger();
  int total_tiles;
  if constexpr (!KGROUP) {
    // tiles per group, then an exclusive scan by warp 2
    for (int g = threadIdx.x; g < args.n_groups; g += kThreads) {
      const int len = group_off(args, g + 1) - group_off(args, g);
      s_tile_start[g + 1] = len > 0 ? (len + MT - 1) / MT : 0;
    }
    __syncthreads();
    if (warp == 2) {
      int carry = 0;
      for (int base = 0; base < args.n_groups; base += 32) {
        const int g = base + lane;
        int v = g < args.n_groups ? s_tile_start[g + 1] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (g < args.n_groups) s_tile_start[g + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) s_tile_start[0] = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer's barriers are initialised before any use
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if constexpr (!KGROUP) {
    total_tiles = s_tile_start[args.n_groups] * args.n_tiles_n;
  } else {
    total_tiles = args.n_groups * args.m_tiles_fixed * args.n_tiles_n;
  }
  int t_begin = 0;
  if constexpr (KGROUP) {
    if (args.tile_end > 0) {
      t_begin = args.tile_begin;
      total_tiles = args.tile_end < total_tiles ? args.tile_end : total_tiles;
    }
  }

  if (warp == 0) {
    // ================================================================ producer
    // lane 0 issues the TMA tile loads (and, MXFP8, the stage's scale atoms)
    // GATHER: every lane issues one 4-row gather per 4 routed rows it owns
    auto src_row = [&](int64_t r) -> int {
      return r < args.m_cap ? __ldg(args.row_src + r) : args.src_oob;
    };
    if (GATHER || lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage: a load is in flight / its phase
      bool ok = true;
      for (int t = t_begin + unit; t < total_tiles && ok; t += n_units) {
        const Tile tl = decode_tile<KGROUP, BKE, KMMA, MT>(args, s_tile_start, t);
        // GATHER: x rows of this lane's 4 rows of the stage (M-grouped: the same
        // rows for the whole tile; K-grouped: loaded one K-block ahead)
        int gsrc[4] = {0, 0, 0, 0};
        if constexpr (GATHER && !KGROUP) {
          const int64_t r = static_cast<int64_t>(tl.row0) + BM * static_cast<int>(rank) + 4 * lane;
#pragma unroll
          for (int i = 0; i < 4; ++i) gsrc[i] = src_row(r + i);
        }
        constexpr int kGq = BKE / 4;  // 4-row pieces per 64-row K-block chunk
        if constexpr (GATHER && KGROUP) {
          const int64_t r = static_cast<int64_t>(tl.k_lo) + 4 * (lane % kGq);
#pragma unroll
          for (int i = 0; i < 4; ++i) gsrc[i] = src_row(r + i);
        }
        for (int kb = 0; kb < tl.k_blocks; ++kb) {
          bool got = mbar_wait(empty_bar(stage), phase ^ 1u, s_abort, args.wait_ns, true, PAIR);
          if constexpr (GATHER) got = __all_sync(0xffffffffu, got);
          if (!got) { ok = false; break; }
          const uint32_t sa = smem_base + stage * Plan::kStageBytes;
          const uint32_t sb = sa + Plan::kABytes;
          const uint32_t fb = full_bar(stage);
          if constexpr (PAIR) {
            // both CTAs' bytes complete on the leader's full barrier
            const uint32_t fbl = mapa_shared(fb, 0);
            if (rank == 0 && lane == 0) {
              mbar_arrive_expect_tx(fb, 2 * (Plan::kStageBytes + kSfTmaBytes));
              armed |= 1u << stage;
              armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            }
            if constexpr (GATHER) __syncwarp();
            if constexpr (!KGROUP) {
              const int k0 = kb * BKE;
              if constexpr (GATHER) {
                tma_gather4_pair(sa + lane * 512, &tmA, fbl, k0, gsrc[0], gsrc[1], gsrc[2],
                                 gsrc[3]);
              } else {
                tma_load_2d_pair(sa, &tmA, fbl, k0, tl.row0 + BM * static_cast<int>(rank));
              }
              if (lane != 0) {
              } else if constexpr (EPI == EPI_SWIGLU_FWD) {
                // the pair's B tile is [gate rows | up rows]: CTA 0 loads gate, CTA 1 up
                const int nh = tl.n_tile * (BN / 2);
                tma_load_3d_pair(sb, &tmB, fbl, k0, (rank ? args.f : 0) + nh, tl.group);
              } else if constexpr (!B_MN) {
                tma_load_3d_pair(sb, &tmB, fbl, k0, tl.n_tile * BN + BNC * static_cast<int>(rank),
                                 tl.group);
              } else {
#pragma unroll
                for (int j = 0; j < BNC / CH; ++j)
                  tma_load_3d_pair(sb + j * kChunkBytes, &tmB, fbl,
                                   tl.n_tile * BN + BNC * static_cast<int>(rank) + CH * j, k0, tl.group);
              }
            } else {
              const int kr = tl.k_lo + kb * BKE;
              if (lane == 0) {
#pragma unroll
                for (int j = 0; j < BM / CH; ++j)
                  tma_load_2d_pair(sa + j * kChunkBytes, &tmA, fbl,
                                   tl.row0 + BM * static_cast<int>(rank) + CH * j, kr);
              }
              if constexpr (GATHER) {
                // B rows are routed rows kr.. of x: lane -> chunk j, rows 4q..4q+3
                const int j = lane / kGq, q = lane % kGq;
                tma_gather4_pair(sb + j * kChunkBytes + q * 512, &tmB, fbl,
                                 tl.n_tile * BN + BNC * static_cast<int>(rank) + CH * j, gsrc[0],
                                 gsrc[1], gsrc[2], gsrc[3]);
                if (kb + 1 < tl.k_blocks) {  // the next K-block's rows, in flight during the wait
                  const int64_t r = static_cast<int64_t>(kr) + BKE + 4 * q;
#pragma unroll
                  for (int i = 0; i < 4; ++i) gsrc[i] = src_row(r + i);
                }
              } else if (lane == 0) {
#pragma unroll
                for (int j = 0; j < BNC / CH; ++j)
                  tma_load_3d_pair(sb + j * kChunkBytes, &tmB, fbl,
                                   tl.n_tile * BN + BNC * static_cast<int>(rank) + CH * j, kr, 0);
              }
            }
          } else if (GATHER || lane == 0) {
            if (lane == 0) {
              mbar_arrive_expect_tx(fb, Plan::kStageBytes);
              armed |= 1u << stage;
              armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            }
            if constexpr (GATHER) __syncwarp();
            if constexpr (!KGROUP) {
              const int k0 = kb * BKE;
              // A: K-major rows of the group's slice
              if constexpr (GATHER) {
                tma_gather4(sa + lane * 512, &tmA, fb, k0, gsrc[0], gsrc[1], gsrc[2], gsrc[3]);
              } else {
                tma_load_2d(sa, &tmA, fb, k0, tl.row0);
              }
              if (lane != 0) {
              } else if constexpr (EPI == EPI_SWIGLU_FWD) {
                const int nh = tl.n_tile * (BN / 2);
                tma_load_3d(sb, &tmB, fb, k0, nh, tl.group);
                tma_load_3d(sb + (BN / 2) * 128, &tmB, fb, k0, args.f + nh, tl.group);
              } else if constexpr (!B_MN) {
                tma_load_3d(sb, &tmB, fb, k0, tl.n_tile * BN, tl.group);
              } else {
#pragma unroll
                for (int j = 0; j < BN / CH; ++j)
                  tma_load_3d(sb + j * kChunkBytes, &tmB, fb, tl.n_tile * BN + CH * j, k0, tl.group);
              }
            } else {
              const int kr = tl.k_lo + kb * BKE;
              if (lane == 0) {
#pragma unroll
                for (int j = 0; j < BM / CH; ++j)
                  tma_load_2d(sa + j * kChunkBytes, &tmA, fb, tl.row0 + CH * j, kr);
              }
              if (lane == 0) {
#pragma unroll
                for (int j = 0; j < BN / CH; ++j)
                  tma_load_3d(sb + j * kChunkBytes, &tmB, fb, tl.n_tile * BN + CH * j, kr, 0);
              }
            }
          }
          if constexpr (FP8) {
            // scale atoms (512 bytes each): the one of this CTA's 128 A rows, then
            // both of the pair's 256 B rows (identical in the two CTAs); their
            // bytes complete on the leader's full barrier like the tiles
            if (lane == 0) {
              const uint32_t fbl = mapa_shared(fb, 0);
              const uint32_t sfa_s = smem_base + Plan::kSfOff + stage * Plan::kSfStageBytes;
              const int kbs = KGROUP ? (tl.k_lo >> 7) + kb : kb;  // 128-element K block
              tma_load_atom_pair(sfa_s, &tmSA, fbl, kbs, (tl.row0 >> 7) + static_cast<int>(rank), 0);
#pragma unroll
              for (int j = 0; j < BN / 128; ++j) {
                int rb;
                if constexpr (EPI == EPI_SWIGLU_FWD) {
                  rb = j == 0 ? tl.n_tile : (args.f >> 7) + tl.n_tile;  // gate rows, then up rows
                } else {
                  rb = tl.n_tile * (BN / 128) + j;
                }
                tma_load_atom_pair(sfa_s + 512 + 512 * j, &tmSB, fbl, kbs, rb, KGROUP ? 0 : tl.group);
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        if (lane == 0) report(args.ctl, MOE_ERR_TIMEOUT, 1);
        // let every copy this warp started land before the CTA exits
        if (lane == 0)
          for (int s = 0; s < STAGES; ++s)
            if (armed & (1u << s))
              mbar_wait(full_bar(s), (armed_parity >> s) & 1u, s_abort, kWaitLimitNs, false);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (PAIR && lane == 0 && rank != 0) {
      // the leader issues the pair's MMAs; wait for them before TMEM is freed
      mbar_wait(drain_bar, 0, s_abort, kWaitLimitNs, false, true);
    } else if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t sf_buf = 0;
      bool ok = true;
      for (int t = t_begin + unit; t < total_tiles && ok; t += n_units) {
        const Tile tl = decode_tile<KGROUP, BKE, KMMA, MT>(args, s_tile_start, t);
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, s_abort, args.wait_ns, true, PAIR)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);  // acc = 0 when NACC = 1
        for (int kb = 0; kb < tl.k_blocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, s_abort, args.wait_ns, true, PAIR)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * Plan::kStageBytes;
          const uint32_t sb = sa + Plan::kABytes;
          const int n16 = (kb == tl.k_blocks - 1) ? tl.last_k16 : 4;
          uint32_t sf_col = 0;
          if constexpr (FP8) {
            // the stage's scale atoms (landed by TMA with the tiles) into TMEM,
            // alternating buffers after the accumulator; each CTA's own atoms go
            // to its own TMEM
            sf_col = tmem_base + NACC * BN + sf_buf * kSfCols;
            sf_buf ^= 1u;
            const uint32_t sfa_s = smem_base + Plan::kSfOff + stage * Plan::kSfStageBytes;
            tmem_cp_sf_pair(sf_col, sfa_s);
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tmem_cp_sf_pair(sf_col + 4 + 4 * j, sfa_s + 512 + 512 * j);
          }
          for (int kk = 0; kk < n16; ++kk) {
            // K-major: the next MMA starts 32 bytes further along each 128-byte row;
            // MN-major: KMMA rows of 128 bytes further
            const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * KMMA * 128, kChunkBytes, 1024)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * KMMA * 128, kChunkBytes, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            if constexpr (FP8) {
              const uint32_t sid = static_cast<uint32_t>(kk);
              mma_mxf8_pair(d_tmem, ad, bd, kIdesc | (sid << 4) | (sid << 29), sf_col | (sid << 30),
                            (sf_col + 4) | (sid << 30), (kb > 0 || kk > 0) ? 1u : 0u);
            } else if constexpr (PAIR && BN > 256) {
              // B rows [0,128) and [128,256) of each CTA: 16 KB apart in both layouts
              const uint64_t bd1 = B_MN ? smem_desc_sw128(sb + kBHalfBytes + kk * KMMA * 128, kChunkBytes, 1024)
                                        : smem_desc_sw128(sb + kBHalfBytes + kk * 32, 16, 1024);
              mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
              mma_bf16_pair(d_tmem + NMMA, ad, bd1, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
            } else if constexpr (PAIR) {
              mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
            } else {
              const uint32_t idesc = (kTail64 && tl.m64) ? kIdesc64 : kIdesc;
              mma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if constexpr (PAIR) mma_commit_pair(empty_bar(stage)); else mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) mma_commit_pair(tfull_bar(acc)); else mma_commit(tfull_bar(acc));
        if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) report(args.ctl, MOE_ERR_TIMEOUT, 2);
      // all MMAs issued by this thread have finished once the drain barrier flips
      if constexpr (PAIR) mma_commit_pair(drain_bar); else mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, s_abort, kWaitLimitNs, false, PAIR);
    }
  } else {
    // ================================================================ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    // TMEM column of tile column c (in B-row order).  Wide pairs: CTA p holds
    // B rows [256p, 256p+256) and MMA h reads rows [128h, 128h+128) of each
    // CTA, writing TMEM columns [256h, 256h+256) = (CTA 0's, CTA 1's).
    auto tcol = [](int c) -> uint32_t {
      if constexpr (BN > 256) {
        return static_cast<uint32_t>(((c >> 7) & 1) * 256 + (c >> 8) * 128 + (c & 127));
      } else {
        return static_cast<uint32_t>(c);
      }
    };
    uint8_t* ebuf = smem + Plan::kEpiOff + (warp - 2) * Plan::kWarpEpiBytes;
    uint8_t* lbuf = ebuf + kEpiBufBytes;  // SwiGLU backward: landing buffer for [A | U]
    int acc = 0;
    uint32_t acc_phase = 0;
    // rows of this warp's quarter in the tile, and the row prefetch of a tile's
    // saved [A | U] slice (SwiGLU backward) into L2
    // tile rows owned by this warp: 32 (16 in an M = 64 tail tile) starting at
    // quarter_first; quarter_rows = how many of them are real rows
    auto rows_per_warp = [&](const Tile& tl) -> int { return (kTail64 && tl.m64) ? 16 : 32; };
    auto quarter_first = [&](const Tile& tl) -> int64_t {
      return static_cast<int64_t>(tl.row0) + BM * static_cast<int>(rank) + quarter * rows_per_warp(tl);
    };
    auto quarter_rows = [&](const Tile& tl) -> int {
      if constexpr (KGROUP) {
        const int64_t n = args.m_rows - quarter_first(tl);
        return n <= 0 ? 0 : (n >= 32 ? 32 : static_cast<int>(n));
      } else {
        const int rpw = rows_per_warp(tl);
        int64_t lim = tl.row_end < args.m_cap ? tl.row_end : args.m_cap;
        const int64_t n = lim - quarter_first(tl);
        return n <= 0 ? 0 : (n >= rpw ? rpw : static_cast<int>(n));
      }
    };
    for (int t = t_begin + unit; t < total_tiles; t += n_units) {
      const Tile tl = decode_tile<KGROUP, BKE, KMMA, MT>(args, s_tile_start, t);
      const int vrows = quarter_rows(tl);
      const int64_t row_first = quarter_first(tl);  // warp's first row
      // SwiGLU backward: the saved A and U of the first 32 columns are
      // requested before waiting for the accumulator, so their latency
      // overlaps the main loop; each later 32 columns are requested while the
      // previous ones are computed.
      const __nv_bfloat16* aux = nullptr;
      if constexpr (EPI == EPI_SWIGLU_BWD) {
        aux = args.aux + row_first * args.ld_aux + static_cast<int64_t>(tl.n_tile) * BN;
        cp_async_au(lbuf, reinterpret_cast<const uint8_t*>(aux),
                    reinterpret_cast<const uint8_t*>(aux + args.f), args.ld_aux * 2, vrows, lane,
                    args.aux);
        cp_async_commit();
      }
      const bool ok = __all_sync(
          0xffffffffu, mbar_wait(tfull_bar(acc), acc_phase, s_abort, args.wait_ns, true, PAIR));
      if (!ok) {
        if constexpr (EPI == EPI_SWIGLU_BWD) cp_async_wait_all();  // own copies land first
        if (lane == 0) report(args.ctl, MOE_ERR_TIMEOUT, 3);
        break;
      }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const bool zero_acc = KGROUP && tl.k_blocks == 0;
      // output columns of this tile that exist (a multiple of 64; the SwiGLU
      // forward tile always lies inside [A | U])
      const int n_left = args.n_cols - tl.n_tile * BN;
      const int ncols = n_left < BN ? n_left : BN;
      const int64_t gofs = KGROUP ? static_cast<int64_t>(tl.group) * args.out_gstride : 0;
      // the warp's part of the accumulator goes back to the MMA issuer
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && rank != 0) mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
          else mbar_arrive(tempty_bar(acc));
        }
      };
      // MXFP8 keeps one accumulator (TMEM also holds the scales), so a tile's
      // epilogue would hold up the next tile's MMAs.  A plain bf16 output
      // row of 256 columns fits in 128 registers as bf16 pairs, the SwiGLU
      // forward's A, U and H of 128 columns in 192: they are formed straight
      // out of TMEM, the accumulator is released, and the stores follow.
      constexpr bool kEarlyRelease = FP8 && (EPI == EPI_BF16 || EPI == EPI_SWIGLU_FWD) && BN == 256;
      if constexpr (kEarlyRelease && EPI == EPI_BF16) {
        auto* base = static_cast<__nv_bfloat16*>(args.out) + gofs + row_first * args.ldo +
                     static_cast<int64_t>(tl.n_tile) * BN;
        uint32_t pk[BN / 2];  // bf16 pairs of this lane's row
#pragma unroll
        for (int c = 0; c < BN; c += 64) {
          if (c < ncols) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tbase + tcol(c), r0);
            tmem_ld32(tbase + tcol(c + 32), r1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              pk[c / 2 + i] = zero_acc ? 0u
                                       : pack_bf16x2(__uint_as_float(r0[2 * i]),
                                                     __uint_as_float(r0[2 * i + 1]));
              pk[c / 2 + 16 + i] = zero_acc ? 0u
                                            : pack_bf16x2(__uint_as_float(r1[2 * i]),
                                                          __uint_as_float(r1[2 * i + 1]));
            }
          }
        }
        release_acc();
#pragma unroll
        for (int c = 0; c < BN; c += 64) {
          if (c < ncols) {
            uint4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              v[q] = make_uint4(pk[c / 2 + 4 * q], pk[c / 2 + 4 * q + 1], pk[c / 2 + 4 * q + 2],
                                pk[c / 2 + 4 * q + 3]);
            store_rows(ebuf, lane, v, reinterpret_cast<uint8_t*>(base + c), args.ldo * 2, vrows);
          }
        }
      } else if constexpr (EPI == EPI_BF16 || EPI == EPI_BF16_COMBINE) {
        auto* base = static_cast<__nv_bfloat16*>(args.out) + gofs + row_first * args.ldo +
                     static_cast<int64_t>(tl.n_tile) * BN;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 64) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + tcol(c), r0);
          tmem_ld32(tbase + tcol(c + 32), r1);
          tmem_ld_wait();
          float f[64];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            f[i] = zero_acc ? 0.f : __uint_as_float(r0[i]);
            f[32 + i] = zero_acc ? 0.f : __uint_as_float(r1[i]);
          }
          uint4 v[8];
          pack64(f, v);
          store_rows(ebuf, lane, v, reinterpret_cast<uint8_t*>(base + c), args.ldo * 2, vrows);
        }
      } else if constexpr (EPI == EPI_F32) {
        auto* base = static_cast<float*>(args.out) + gofs + row_first * args.ldo +
                     static_cast<int64_t>(tl.n_tile) * BN;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + tcol(c), r);
          tmem_ld_wait();
          uint4 v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            v[q] = zero_acc ? make_uint4(0, 0, 0, 0)
                            : make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
          store_rows(ebuf, lane, v, reinterpret_cast<uint8_t*>(base + c), args.ldo * 4, vrows);
        }
      } else if constexpr (EPI == EPI_SWIGLU_FWD && FP8) {
        // as above: A, U and H of the warp's rows (3 x 64 registers of bf16
        // pairs) are formed straight out of TMEM, 16 columns at a time; the
        // accumulator is released, then the rows are stored
        constexpr int BNH = BN / 2;
        const int64_t col0 = static_cast<int64_t>(tl.n_tile) * BNH;
        auto* au = args.out != nullptr
                       ? static_cast<__nv_bfloat16*>(args.out) + row_first * args.ldo + col0
                       : nullptr;
        auto* hh = static_cast<__nv_bfloat16*>(args.out2) + row_first * args.ldo2 + col0;
        uint32_t pa[BNH / 2], pu[BNH / 2], ph[BNH / 2];
#pragma unroll
        for (int c = 0; c < BNH; c += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(tbase + tcol(c), g);
          tmem_ld16(tbase + tcol(BNH + c), u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a0 = __uint_as_float(g[2 * i]), a1 = __uint_as_float(g[2 * i + 1]);
            const float b0 = __uint_as_float(u[2 * i]), b1 = __uint_as_float(u[2 * i + 1]);
            pa[c / 2 + i] = pack_bf16x2(a0, a1);
            pu[c / 2 + i] = pack_bf16x2(b0, b1);
            ph[c / 2 + i] = pack_bf16x2(a0 * sigmoid_fast(a0) * b0, a1 * sigmoid_fast(a1) * b1);
          }
        }
        release_acc();
        auto put = [&](const uint32_t (&p)[BNH / 2], int c, __nv_bfloat16* dst, int64_t ld) {
          uint4 v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            v[q] = make_uint4(p[c / 2 + 4 * q], p[c / 2 + 4 * q + 1], p[c / 2 + 4 * q + 2],
                              p[c / 2 + 4 * q + 3]);
          store_rows(ebuf, lane, v, reinterpret_cast<uint8_t*>(dst + c), ld * 2, vrows);
        };
#pragma unroll
        for (int c = 0; c < BNH; c += 64) {
          if (au != nullptr) {  // [A | U] is not kept when the backward recomputes it
            put(pa, c, au, args.ldo);
            put(pu, c, au + args.f, args.ldo);
          }
          put(ph, c, hh, args.ldo2);
        }
      } else if constexpr (EPI == EPI_SWIGLU_FWD) {
        constexpr int BNH = BN / 2;
        const int64_t col0 = static_cast<int64_t>(tl.n_tile) * BNH;
        auto* au = args.out != nullptr
                       ? static_cast<__nv_bfloat16*>(args.out) + row_first * args.ldo + col0
                       : nullptr;
        auto* hh = static_cast<__nv_bfloat16*>(args.out2) + row_first * args.ldo2 + col0;
#pragma unroll 1
        for (int c = 0; c < BNH; c += 64) {
          uint4 vg[8], vu[8], vh[8];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t g[32], u[32];
            tmem_ld32(tbase + tcol(c + 32 * half), g);
            tmem_ld32(tbase + tcol(BNH + c + 32 * half), u);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float a[8], b[8], h[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                a[i] = __uint_as_float(g[8 * q + i]);
                b[i] = __uint_as_float(u[8 * q + i]);
                h[i] = a[i] * sigmoid_fast(a[i]) * b[i];
              }
              vg[4 * half + q] = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                            pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
              vu[4 * half + q] = make_uint4(pack_bf16x2(b[0], b[1]), pack_bf16x2(b[2], b[3]),
                                            pack_bf16x2(b[4], b[5]), pack_bf16x2(b[6], b[7]));
              vh[4 * half + q] = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]),
                                            pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
            }
          }
          if (args.out != nullptr) {  // [A | U] is not kept when the backward recomputes it
            store_rows(ebuf, lane, vg, reinterpret_cast<uint8_t*>(au + c), args.ldo * 2, vrows);
            store_rows(ebuf, lane, vu, reinterpret_cast<uint8_t*>(au + args.f + c), args.ldo * 2,
                       vrows);
          }
          store_rows(ebuf, lane, vh, reinterpret_cast<uint8_t*>(hh + c), args.ldo2 * 2, vrows);
        }
      } else {  // EPI_SWIGLU_BWD
        auto* dau = static_cast<__nv_bfloat16*>(args.out) + row_first * args.ldo +
                    static_cast<int64_t>(tl.n_tile) * BN;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 64) {
          uint4 ou[8];  // dU in registers; dA goes straight to the staging buffer
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int cc = c + 32 * half;
            uint4 vau[8];  // this lane's row: A in slots 0-3, U in slots 4-7
            cp_async_wait_all();
            __syncwarp();
            stage_read_row(lbuf, lane, vau);
            __syncwarp();
            if (cc + 32 < ncols) {  // the next 32 columns land while these are computed
              cp_async_au(lbuf, reinterpret_cast<const uint8_t*>(aux + cc + 32),
                          reinterpret_cast<const uint8_t*>(aux + args.f + cc + 32),
                          args.ld_aux * 2, vrows, lane, args.aux);
              cp_async_commit();
            }
            uint32_t r[32];
            tmem_ld32(tbase + tcol(cc), r);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 qa = vau[q], qu = vau[4 + q];
              const float a[8] = {bf16_lo(qa.x), bf16_hi(qa.x), bf16_lo(qa.y), bf16_hi(qa.y),
                                  bf16_lo(qa.z), bf16_hi(qa.z), bf16_lo(qa.w), bf16_hi(qa.w)};
              const float u[8] = {bf16_lo(qu.x), bf16_hi(qu.x), bf16_lo(qu.y), bf16_hi(qu.y),
                                  bf16_lo(qu.z), bf16_hi(qu.z), bf16_lo(qu.w), bf16_hi(qu.w)};
              float da[8], du[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float dh = __uint_as_float(r[8 * q + i]);
                const float sg = sigmoid_fast(a[i]);
                da[i] = dh * u[i] * sg * (1.0f + a[i] * (1.0f - sg));
                du[i] = dh * a[i] * sg;
              }
              *stage_slot(ebuf, lane, 4 * half + q) =
                  make_uint4(pack_bf16x2(da[0], da[1]), pack_bf16x2(da[2], da[3]),
                             pack_bf16x2(da[4], da[5]), pack_bf16x2(da[6], da[7]));
              ou[4 * half + q] = make_uint4(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]),
                                            pack_bf16x2(du[4], du[5]), pack_bf16x2(du[6], du[7]));
            }
          }
          __syncwarp();
          stage_to_global(ebuf, reinterpret_cast<uint8_t*>(dau + c), args.ldo * 2, vrows, lane);
          __syncwarp();
          store_rows(ebuf, lane, ou, reinterpret_cast<uint8_t*>(dau + args.f + c), args.ldo * 2, vrows);
        }
      }
      if constexpr (!kEarlyRelease) release_acc();
      if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
      if constexpr (EPI == EPI_BF16_COMBINE) {
        // The warp's rows of this column tile are stored and the accumulator
        // is released, so what follows overlaps the next tile's main loop.
        // Publish the rows, then count one arrival per (token, column tile);
        // the arrival that completes a token's valid rows forms y[t] over the
        // tile's columns from the stored bf16 rows, in slot order with the
        // combine kernel's arithmetic (same bits), and clears the count.
        __threadfence();
        __syncwarp();
        int t = -1;
        int32_t* cnt = nullptr;
        bool last = false;
        if (lane < vrows) {
          const int src = __ldg(args.row_src + row_first + lane);
          if (src >= 0 && src < args.n_tok) t = src;
        }
        if (t >= 0) {
          int need = 0;
          for (int j = 0; j < args.top_k; ++j)
            need += __ldg(args.row_map + static_cast<int64_t>(t) * args.top_k + j) >= 0 ? 1 : 0;
          cnt = args.arrivals + static_cast<int64_t>(t) * args.n_tiles_n + tl.n_tile;
          last = atomicAdd(cnt, 1) == need - 1;
        }
        uint32_t done = __ballot_sync(0xffffffffu, last);
        if (done != 0u) __threadfence();
        const auto* obase = static_cast<const __nv_bfloat16*>(args.out);
        const int64_t col0 = static_cast<int64_t>(tl.n_tile) * BN;
        const int n_left = args.n_cols - tl.n_tile * BN;
        const int ncols = n_left < BN ? n_left : BN;
        while (done != 0u) {
          // two completed tokens at a time: all their loads in flight together
          int64_t tt[2];
          int srcl[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            srcl[h] = done != 0u ? __ffs(done) - 1 : -1;
            if (done != 0u) done &= done - 1u;
            tt[h] = srcl[h] >= 0 ? __shfl_sync(0xffffffffu, t, srcl[h]) : -1;
          }
          int rows[2][8];
          float wt[2][8];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const bool ok = tt[h] >= 0 && j < args.top_k;
              rows[h][j] = ok ? __ldg(args.row_map + tt[h] * args.top_k + j) : -1;
              wt[h][j] = ok ? __ldg(args.topk_w + tt[h] * args.top_k + j) : 0.f;
            }
          for (int c = lane * 8; c < ncols; c += 256) {
            uint4 q[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (rows[h][j] >= 0)
                  q[h][j] = __ldcg(reinterpret_cast<const uint4*>(obase + rows[h][j] * args.ldo + col0 + c));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (tt[h] < 0) continue;
              float acc[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                if (rows[h][j] < 0) continue;
                float fv[8];
                unpack8(q[h][j], fv);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(wt[h][j], fv[i], acc[i]);
              }
              if (args.shared != nullptr) {  // the shared expert's output, added last
                float fv[8];
                unpack8(__ldg(reinterpret_cast<const uint4*>(args.shared + tt[h] * args.ldo + col0 + c)),
                        fv);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += fv[i];
              }
              *reinterpret_cast<uint4*>(args.y + tt[h] * args.ldo + col0 + c) = pack8(acc);
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (lane == srcl[h]) *cnt = 0;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer is done with this CTA's TMEM and barriers
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(kTmemCols)
                   : "memory");
    } else {
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(kTmemCols)
                   : "memory");
    }
  }
}

}  // namespace tc
}  // namespace moe
