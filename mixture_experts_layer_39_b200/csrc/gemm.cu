// Host side of the tcgen05 grouped GEMMs: TMA descriptors and launches for
// every contraction of the layer.
//
//   forward   gate/up : [M, d] x W_gu[e]^T  -> SwiGLU epilogue -> AU, H
//             down    : [M, f] x W_d[e]^T   -> O
//   backward  dgrad-down : dO x W_d[e]      -> SwiGLU-backward epilogue -> dAU
//             dgrad-gu   : dAU x W_gu[e]    -> dX_perm
//             wgrad-down : dO_e^T H_e       -> dW_d[e]   (contraction over e's rows)
//             wgrad-gu   : dAU_e^T X_e      -> dW_gu[e]
//   router    logits  : x W_r^T (E > 64), dX_router = dL W_r,
//             dW_r partials = dL^T x over token chunks
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm.cuh"
#include "host_ctx.cuh"
#include "tc_gemm.cuh"

namespace moe {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a row-major [outer, inner] matrix (bf16, or E4M3 codes as uint8).
bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
             uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool u8 = false) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over [groups, outer, inner].
bool tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t groups,
             uint64_t row_bytes, uint64_t group_bytes, uint32_t box_inner, uint32_t box_outer,
             bool u8 = false) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {inner, outer, groups};
  cuuint64_t strides[2] = {row_bytes, group_bytes};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D map over MXFP8 scales in the tensor cores' atom order: 512-byte atoms
// (128 MN indices x 128 contraction elements) indexed (K block, MN block,
// group); one box is one atom.  Atoms past an operand's MN extent read as
// zeros (their rows of the operand tile are zero fill too).
bool tmap_sf(CUtensorMap* m, const void* base, uint64_t n_kb, uint64_t n_rb, uint64_t groups) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[5] = {128, 4, n_kb, n_rb, groups};
  cuuint64_t strides[4] = {128, 512, 512 * n_kb, 512 * n_kb * n_rb};
  cuuint32_t box[5] = {128, 4, 1, 1, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kMaxDynSmem = 227 * 1024;  // per block on sm_100

template <int BN, bool A_MN, bool B_MN, int EPI, bool KGROUP, int STAGES, bool FP8, bool PAIR,
          bool GATHER>
moe_status_t launch_stages(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& sa,
                           const CUtensorMap& sb, const tc::GemmArgs& args, int grid,
                           cudaStream_t st) {
  auto kern = tc::grouped_gemm_kernel<BN, A_MN, B_MN, EPI, KGROUP, STAGES, FP8, PAIR, GATHER>;
  const size_t smem = tc::SmemPlan<BN, STAGES, EPI, FP8, PAIR>::bytes(args.n_groups);
  if (!set_max_dyn_smem(reinterpret_cast<const void*>(kern), smem)) return MOE_ERR_CUDA;
  if (grid <= 0) return MOE_OK;
  if constexpr (PAIR) {
    grid &= ~1;  // whole pairs
    if (grid <= 0) return MOE_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a, b, sa, sb, args) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  } else {
    return launch_pdl(kern, dim3(grid), dim3(tc::kThreads), smem, st, a, b, sa, sb, args) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  }
}

// Ring depth: as many stages as fit beside the epilogue buffers.  A stage is
// 48 KB for single-CTA 128 x 256 tiles and for wide pairs, 32 KB for 256 x 256
// pairs (bf16 or MXFP8; MXFP8 adds 1.5 KB of scale atoms).  The SwiGLU
// backward's landing buffers take 16 KB more; with more than ~440 experts the
// tile table no longer fits beside a sixth pair stage, and the launch falls
// back to one stage fewer.  sa, sb: the MXFP8 scale maps (unused otherwise).
template <int BN, bool A_MN, bool B_MN, int EPI, bool KGROUP, bool FP8 = false, bool PAIR = false,
          bool GATHER = false>
moe_status_t launch(const CUtensorMap& a, const CUtensorMap& b, const tc::GemmArgs& args, int grid,
                    cudaStream_t st, const CUtensorMap* sa = nullptr,
                    const CUtensorMap* sb = nullptr) {
  const CUtensorMap& sfa = sa != nullptr ? *sa : a;
  const CUtensorMap& sfb = sb != nullptr ? *sb : b;
  constexpr bool BWD = EPI == tc::EPI_SWIGLU_BWD;
  constexpr int STAGES = FP8    ? (BWD ? 5 : 6)
                         : PAIR ? (BN == 512 ? (BWD ? 3 : 4) : 6)
                                : (BN == 256 ? 4 : 6);
  if constexpr (BWD || FP8) {
    const size_t need = tc::SmemPlan<BN, STAGES, EPI, FP8, PAIR>::bytes(args.n_groups);
    if (need > kMaxDynSmem)
      return launch_stages<BN, A_MN, B_MN, EPI, KGROUP, STAGES - 1, FP8, PAIR, GATHER>(
          a, b, sfa, sfb, args, grid, st);
  }
  return launch_stages<BN, A_MN, B_MN, EPI, KGROUP, STAGES, FP8, PAIR, GATHER>(a, b, sfa, sfb, args,
                                                                              grid, st);
}

// The last wave of wide weight-gradient tiles keeps every busy pair for a
// whole wide tile while the others idle.  When that wave holds at most half
// as many tiles as there are pairs, its tiles run instead as a second launch
// of 256 x 256 tiles (two per wide tile, one per pair), which ends in about
// 0.6 of a wide tile's time.  Returns the number of wide tiles moved there.
int64_t wide_tail(int num_sms, int64_t wide_tiles) {
  const int64_t units = num_sms / 2 > 0 ? num_sms / 2 : 1;
  const int64_t rem = wide_tiles % units;
  return (rem > 0 && 2 * rem <= units) ? rem : 0;
}

// Weight gradients run 256 x 512 pair tiles ("wide") when the experts'
// contraction ranges are long (at least 4096 routed rows on average: the
// single accumulator's epilogue, which no longer overlaps the next tile, is
// then a few percent of a tile) and the waves come out shorter than with
// 256 x 256 tiles.  In units of a wide tile's time: a narrow tile takes about
// 0.575 (half the work at 0.87 of the wide rate: it reads 25% more operand
// bytes per FLOP) and a tail moved to a narrow launch about 0.6; tiles =
// E x M tiles x N tiles, units = CTA pairs.
bool wide_wgrad(int num_sms, int64_t E, int64_t M, int64_t N, int64_t rows) {
  if (rows < 4096 * E) return false;
  const int64_t units = num_sms / 2 > 0 ? num_sms / 2 : 1;
  const int64_t mt = ceil_div64(M, 256);
  const int64_t tiles_n = E * mt * ceil_div64(N, 256);
  const int64_t tiles_w = E * mt * ceil_div64(N, 512);
  const int64_t tail = tiles_w % units == 0 ? 0 : (wide_tail(num_sms, tiles_w) > 0 ? 600 : 1000);
  return 1000 * (tiles_w / units) + tail <= 575 * ceil_div64(tiles_n, units);
}

tc::GemmArgs base_args(const GemmCtx& c) {
  tc::GemmArgs a{};
  a.ctl = c.ctl;
  a.wait_ns = c.wait_ns;
  return a;
}

// N output columns in tiles of bn (the last tile may be partly past N)
void set_n(tc::GemmArgs& a, int64_t N, int bn) {
  a.n_cols = static_cast<int>(N);
  a.n_tiles_n = static_cast<int>(ceil_div64(N, bn));
}

// K-grouped: M output rows per group in tiles of mt rows
void set_m(tc::GemmArgs& a, int64_t M, int mt) {
  a.m_rows = static_cast<int>(M);
  a.m_tiles_fixed = static_cast<int>(ceil_div64(M, mt));
}

// A K-grouped weight gradient on wide tiles, its last wave (wide_tail) as a
// second launch of 256 x 256 tiles over the same groups and M tiles: wide
// tile w covers narrow tiles 2w and 2w + 1, so the tail is one contiguous
// range of the narrow launch's tile list.
moe_status_t launch_wgrad_wide(const GemmCtx& c, const CUtensorMap& ta, const CUtensorMap& tb,
                               tc::GemmArgs a, int64_t N, cudaStream_t st) {
  set_n(a, N, 512);
  const int64_t tiles = static_cast<int64_t>(a.n_groups) * a.m_tiles_fixed * a.n_tiles_n;
  const int64_t tail = wide_tail(c.num_sms, tiles);
  const int64_t head = tiles - tail;
  if (head > 0) {
    tc::GemmArgs w = a;
    if (tail > 0) {
      w.tile_begin = 0;
      w.tile_end = static_cast<int>(head);
    }
    const int grid = static_cast<int>(2 * head < c.num_sms ? 2 * head : c.num_sms);
    const moe_status_t r = launch<512, true, true, tc::EPI_BF16, true, false, true>(ta, tb, w, grid, st);
    if (r != MOE_OK) return r;
  }
  if (tail == 0) return MOE_OK;
  tc::GemmArgs n = a;
  // two 256-column tiles per wide tile, also where N ends in the first half
  // of the last wide tile (that tile's second half then writes nothing)
  n.n_cols = static_cast<int>(N);
  n.n_tiles_n = 2 * a.n_tiles_n;
  n.tile_begin = static_cast<int>(2 * head);
  n.tile_end = static_cast<int>(2 * tiles);
  if (c.extra_launches != nullptr) ++*c.extra_launches;
  const int grid = static_cast<int>(4 * tail < c.num_sms ? 4 * tail : c.num_sms);
  return launch<256, true, true, tc::EPI_BF16, true, false, true>(ta, tb, n, grid, st);
}


}  // namespace

moe_status_t gemm_fwd_gate_up(const GemmCtx& c, const void* x_perm, const int32_t* offsets,
                              const void* w_gu, void* au, void* h, int E, int d, int f,
                              int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, x_perm, d, m_cap, 2ull * d, 64, 128)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_gu, d, 2ull * f, E, 2ull * d, 4ull * f * d, 64, 128)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, 2ll * f, 256);  // 128 columns of A and of U per tile
  a.k_blocks = d / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.m_cap = m_cap;
  a.out = au;
  a.ldo = 2ll * f;
  a.out2 = h;
  a.ldo2 = f;
  a.f = f;
  if (c.pair_m) return launch<256, false, false, tc::EPI_SWIGLU_FWD, false, false, true>(ta, tb, a, c.num_sms, st);
  return launch<256, false, false, tc::EPI_SWIGLU_FWD, false>(ta, tb, a, c.num_sms, st);
}

moe_status_t gemm_fwd_down(const GemmCtx& c, const void* h, const int32_t* offsets,
                           const void* w_d, void* o_perm, int E, int d, int f, int64_t m_cap,
                           cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, h, f, m_cap, 2ull * f, 64, 128)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_d, f, d, E, 2ull * f, 2ull * d * f, 64, c.pair_m ? 128 : 256))
    return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  a.k_blocks = f / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.m_cap = m_cap;
  a.out = o_perm;
  a.ldo = d;
  if (c.pair_m) return launch<256, false, false, tc::EPI_BF16, false, false, true>(ta, tb, a, c.num_sms, st);
  return launch<256, false, false, tc::EPI_BF16, false>(ta, tb, a, c.num_sms, st);
}

moe_status_t gemm_fwd_down_combine(const GemmCtx& c, const void* h, const int32_t* offsets,
                                   const void* w_d, void* o_perm, int E, int d, int f,
                                   int64_t m_cap, const CombineArgs& cb, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, h, f, m_cap, 2ull * f, 64, 128)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_d, f, d, E, 2ull * f, 2ull * d * f, 64, c.pair_m ? 128 : 256))
    return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  a.k_blocks = f / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);
  a.m_cap = m_cap;
  a.out = o_perm;
  a.ldo = d;
  a.row_src = cb.row_src;
  a.row_map = cb.row_map;
  a.topk_w = cb.topk_w;
  a.shared = static_cast<const __nv_bfloat16*>(cb.shared);
  a.y = static_cast<__nv_bfloat16*>(cb.y);
  a.arrivals = cb.arrivals;
  a.n_tok = cb.T;
  a.top_k = cb.k;
  if (c.pair_m)
    return launch<256, false, false, tc::EPI_BF16_COMBINE, false, false, true>(ta, tb, a, c.num_sms, st);
  return launch<256, false, false, tc::EPI_BF16_COMBINE, false>(ta, tb, a, c.num_sms, st);
}

moe_status_t gemm_dgrad_down_swiglu(const GemmCtx& c, const void* do_perm, const int32_t* offsets,
                                    const void* w_d, const void* au, void* dau, int E, int d,
                                    int f, int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, do_perm, d, m_cap, 2ull * d, 64, 128)) return MOE_ERR_CUDA;
  // W_d[e] is [d (contraction), f (output)]: N-major operand
  if (!tmap_3d(&tb, w_d, f, d, E, 2ull * f, 2ull * d * f, 64, 64)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, f, 256);
  a.k_blocks = d / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.m_cap = m_cap;
  a.out = dau;
  a.ldo = 2ll * f;
  a.aux = static_cast<const __nv_bfloat16*>(au);
  a.ld_aux = 2ll * f;
  a.f = f;
  if (c.pair_m) return launch<256, false, true, tc::EPI_SWIGLU_BWD, false, false, true>(ta, tb, a, c.num_sms, st);
  return launch<256, false, true, tc::EPI_SWIGLU_BWD, false>(ta, tb, a, c.num_sms, st);
}

moe_status_t gemm_dgrad_gate_up(const GemmCtx& c, const void* dau, const int32_t* offsets,
                                const void* w_gu, void* dx_perm, int E, int d, int f,
                                int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, dau, 2ull * f, m_cap, 4ull * f, 64, 128)) return MOE_ERR_CUDA;
  // W_gu[e] is [2f (contraction), d (output)]: N-major operand
  if (!tmap_3d(&tb, w_gu, d, 2ull * f, E, 2ull * d, 4ull * f * d, 64, 64)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  a.k_blocks = 2 * f / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.m_cap = m_cap;
  a.out = dx_perm;
  a.ldo = d;
  if (c.pair_m) return launch<256, false, true, tc::EPI_BF16, false, false, true>(ta, tb, a, c.num_sms, st);
  return launch<256, false, true, tc::EPI_BF16, false>(ta, tb, a, c.num_sms, st);
}

moe_status_t gemm_wgrad_down(const GemmCtx& c, const void* do_perm, const void* h,
                             const int32_t* offsets, void* dw_d, int E, int d, int f,
                             int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  // A = dO^T (M = d along the rows' contiguous axis), B = H (N = f)
  if (!tmap_2d(&ta, do_perm, d, m_cap, 2ull * d, 64, 64)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, h, f, m_cap, 1, 2ull * f, 2ull * f * m_cap, 64, 64)) return MOE_ERR_CUDA;
  const bool wide = wide_wgrad(c.num_sms, E, d, f, m_cap);
  tc::GemmArgs a = base_args(c);
  set_n(a, f, wide ? 512 : 256);
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.out = dw_d;
  a.ldo = f;
  a.out_gstride = static_cast<int64_t>(d) * f;
  set_m(a, d, 2 * tc::BM);  // CTA pairs: 256-row tiles
  if (wide) return launch_wgrad_wide(c, ta, tb, a, f, st);
  const int64_t tiles = static_cast<int64_t>(E) * a.m_tiles_fixed * a.n_tiles_n;
  const int grid = static_cast<int>(2 * tiles < c.num_sms ? 2 * tiles : c.num_sms);
  return launch<256, true, true, tc::EPI_BF16, true, false, true>(ta, tb, a, grid, st);
}

moe_status_t gemm_wgrad_gate_up(const GemmCtx& c, const void* dau, const void* x_perm,
                                const int32_t* offsets, void* dw_gu, int E, int d, int f,
                                int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, dau, 2ull * f, m_cap, 4ull * f, 64, 64)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, x_perm, d, m_cap, 1, 2ull * d, 2ull * d * m_cap, 64, 64)) return MOE_ERR_CUDA;
  const bool wide = wide_wgrad(c.num_sms, E, 2ll * f, d, m_cap);
  tc::GemmArgs a = base_args(c);
  set_n(a, d, wide ? 512 : 256);
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.out = dw_gu;
  a.ldo = d;
  a.out_gstride = 2ll * f * d;
  set_m(a, 2ll * f, 2 * tc::BM);  // CTA pairs: 256-row tiles
  if (wide) return launch_wgrad_wide(c, ta, tb, a, d, st);
  const int64_t tiles = static_cast<int64_t>(E) * a.m_tiles_fixed * a.n_tiles_n;
  const int grid = static_cast<int>(2 * tiles < c.num_sms ? 2 * tiles : c.num_sms);
  return launch<256, true, true, tc::EPI_BF16, true, false, true>(ta, tb, a, grid, st);
}

// Gather forms: the routed rows are read from x (T rows) through row_src
// (tile::gather4 loads; the tensor map's box is one row of 64 columns).
moe_status_t gemm_fwd_gate_up_gather(const GemmCtx& c, const void* x, int T,
                                     const int32_t* row_src, const int32_t* offsets,
                                     const void* w_gu, void* au, void* h, int E, int d, int f,
                                     int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, x, d, T, 2ull * d, 64, 1)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_gu, d, 2ull * f, E, 2ull * d, 4ull * f * d, 64, 128)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, 2ll * f, 256);  // 128 columns of A and of U per tile
  a.k_blocks = d / tc::BK;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);
  a.m_cap = m_cap;
  a.out = au;
  a.ldo = 2ll * f;
  a.out2 = h;
  a.ldo2 = f;
  a.f = f;
  a.row_src = row_src;
  a.src_oob = T;
  if (c.pair_m)
    return launch<256, false, false, tc::EPI_SWIGLU_FWD, false, false, true, true>(ta, tb, a,
                                                                                   c.num_sms, st);
  return launch<256, false, false, tc::EPI_SWIGLU_FWD, false, false, false, true>(ta, tb, a,
                                                                                  c.num_sms, st);
}

moe_status_t gemm_wgrad_gate_up_gather(const GemmCtx& c, const void* dau, const void* x, int T,
                                       const int32_t* row_src, const int32_t* offsets,
                                       void* dw_gu, int E, int d, int f, int64_t m_cap,
                                       cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, dau, 2ull * f, m_cap, 4ull * f, 64, 64)) return MOE_ERR_CUDA;
  if (!tmap_2d(&tb, x, d, T, 2ull * d, 64, 1)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);
  a.m_cap = m_cap;
  a.out = dw_gu;
  a.ldo = d;
  a.out_gstride = 2ll * f * d;
  set_m(a, 2ll * f, 2 * tc::BM);  // CTA pairs: 256-row tiles
  a.row_src = row_src;
  a.src_oob = T;
  const int64_t tiles = static_cast<int64_t>(E) * a.m_tiles_fixed * a.n_tiles_n;
  const int grid = static_cast<int>(2 * tiles < c.num_sms ? 2 * tiles : c.num_sms);
  return launch<256, true, true, tc::EPI_BF16, true, false, true, true>(ta, tb, a, grid, st);
}

moe_status_t gemm_router_logits(const GemmCtx& c, const void* x, const void* w_r, float* logits,
                                int T, int d, int E, int ld, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, x, d, T, 2ull * d, 64, 128)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_r, d, E, 1, 2ull * d, 2ull * d * E, 64, 128)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  // ld = E rounded up to whole 128-column tiles; the columns past E come out
  // zero (W_r rows past E read as TMA zero fill)
  set_n(a, ld, 128);
  a.k_blocks = d / tc::BK;
  a.n_groups = 1;
  a.offsets = nullptr;
  a.uniform_len = T;
  a.total_len = T;
  a.m_cap = T;
  a.out = logits;
  a.ldo = ld;
  const int64_t tiles = ceil_div64(T, tc::BM) * a.n_tiles_n;
  const int grid = static_cast<int>(tiles < c.num_sms ? tiles : c.num_sms);
  return launch<128, false, false, tc::EPI_F32, false>(ta, tb, a, grid, st);
}

moe_status_t gemm_router_dx(const GemmCtx& c, const void* dl_bf16, int ld, const void* w_r,
                            float* dx_router, int T, int d, int E, cudaStream_t st) {
  CUtensorMap ta, tb;
  // contraction over E, zero-filled past E in both operands
  if (!tmap_2d(&ta, dl_bf16, E, T, 2ull * ld, 64, 128)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_r, d, E, 1, 2ull * d, 2ull * d * E, 64, 64)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  a.k_blocks = static_cast<int>(ceil_div64(E, tc::BK));
  a.n_groups = 1;
  a.offsets = nullptr;
  a.uniform_len = T;
  a.total_len = T;
  a.m_cap = T;
  a.out = dx_router;
  a.ldo = d;
  const int64_t tiles = ceil_div64(T, tc::BM) * a.n_tiles_n;
  const int grid = static_cast<int>(tiles < c.num_sms ? tiles : c.num_sms);
  return launch<256, false, true, tc::EPI_F32, false>(ta, tb, a, grid, st);
}

int router_dw_groups(int num_sms, int T, int d, int E, int* group_len) {
  const int tiles_per_group = static_cast<int>(ceil_div64(E, tc::BM) * ceil_div64(d, 256));
  int g = num_sms / (tiles_per_group > 0 ? tiles_per_group : 1);
  if (g < 1) g = 1;
  int64_t len = ceil_div64(ceil_div64(T, g), 64) * 64;
  g = static_cast<int>(ceil_div64(T, len));
  *group_len = static_cast<int>(len);
  return g;
}

moe_status_t gemm_router_dw_partial(const GemmCtx& c, const void* dl_bf16, int ld, const void* x,
                                    float* partial, int T, int d, int E, int n_groups,
                                    int group_len, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_2d(&ta, dl_bf16, E, T, 2ull * ld, 64, 64)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, x, d, T, 1, 2ull * d, 2ull * d * T, 64, 64)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, d, 256);
  set_m(a, E, tc::BM);
  a.n_groups = n_groups;
  a.offsets = nullptr;
  a.uniform_len = group_len;
  a.total_len = T;
  a.out = partial;
  a.ldo = d;
  a.out_gstride = static_cast<int64_t>(E) * d;
  const int64_t tiles = static_cast<int64_t>(n_groups) * a.m_tiles_fixed * a.n_tiles_n;
  const int grid = static_cast<int>(tiles < c.num_sms ? tiles : c.num_sms);
  return launch<256, true, true, tc::EPI_F32, true>(ta, tb, a, grid, st);
}

// ------------------------------------------------------------------ MXFP8
// Operands are E4M3 codes with E8M0 scales in atom order (see tmap_sf); the
// GEMMs run 256 x 256 CTA-pair tiles with 128 contraction elements (128
// bytes) per stage.

namespace {

tc::GemmArgs mx_m_grouped(const GemmCtx& c, const int32_t* offsets, int E, int64_t N, int K,
                          int64_t m_cap) {
  tc::GemmArgs a = base_args(c);
  set_n(a, N, 256);
  a.k_blocks = K / 128;
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.m_cap = m_cap;
  return a;
}

}  // namespace

moe_status_t gemm_mx_fwd_gate_up(const GemmCtx& c, const MxOperand& x, const int32_t* offsets,
                                 const MxOperand& w_gu, void* au, void* h, int E, int d, int f,
                                 int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_2d(&ta, x.q, d, m_cap, d, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_gu.q, d, 2ull * f, E, d, 2ull * f * d, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsa, x.s, d / 128, m_cap / 128, 1)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsb, w_gu.s, d / 128, 2ull * f / 128, E)) return MOE_ERR_CUDA;
  tc::GemmArgs a = mx_m_grouped(c, offsets, E, 2ll * f, d, m_cap);  // 128 of A and of U per tile
  a.out = au;
  a.ldo = 2ll * f;
  a.out2 = h;
  a.ldo2 = f;
  a.f = f;
  return launch<256, false, false, tc::EPI_SWIGLU_FWD, false, true, true>(ta, tb, a, c.num_sms, st,
                                                                        &tsa, &tsb);
}

moe_status_t gemm_mx_fwd_down(const GemmCtx& c, const MxOperand& h, const int32_t* offsets,
                              const MxOperand& w_d, void* o_perm, int E, int d, int f,
                              int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_2d(&ta, h.q, f, m_cap, f, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, w_d.q, f, d, E, f, 1ull * d * f, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsa, h.s, f / 128, m_cap / 128, 1)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsb, w_d.s, f / 128, d / 128, E)) return MOE_ERR_CUDA;
  tc::GemmArgs a = mx_m_grouped(c, offsets, E, d, f, m_cap);
  a.out = o_perm;
  a.ldo = d;
  return launch<256, false, false, tc::EPI_BF16, false, true, true>(ta, tb, a, c.num_sms, st, &tsa,
                                                                  &tsb);
}

moe_status_t gemm_mx_dgrad_down_swiglu(const GemmCtx& c, const MxOperand& dO, const int32_t* offsets,
                                       const MxOperand& w_d_col, const void* au, void* dau, int E,
                                       int d, int f, int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_2d(&ta, dO.q, d, m_cap, d, 128, 128, true)) return MOE_ERR_CUDA;
  // W_d[e] is [d (contraction), f (output)]: N-major, quantised along d
  if (!tmap_3d(&tb, w_d_col.q, f, d, E, f, 1ull * d * f, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsa, dO.s, d / 128, m_cap / 128, 1)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsb, w_d_col.s, d / 128, f / 128, E)) return MOE_ERR_CUDA;
  tc::GemmArgs a = mx_m_grouped(c, offsets, E, f, d, m_cap);
  a.out = dau;
  a.ldo = 2ll * f;
  a.aux = static_cast<const __nv_bfloat16*>(au);
  a.ld_aux = 2ll * f;
  a.f = f;
  return launch<256, false, true, tc::EPI_SWIGLU_BWD, false, true, true>(ta, tb, a, c.num_sms, st,
                                                                       &tsa, &tsb);
}

moe_status_t gemm_mx_dgrad_gate_up(const GemmCtx& c, const MxOperand& dau, const int32_t* offsets,
                                   const MxOperand& w_gu_col, void* dx_perm, int E, int d, int f,
                                   int64_t m_cap, cudaStream_t st) {
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_2d(&ta, dau.q, 2ull * f, m_cap, 2ull * f, 128, 128, true)) return MOE_ERR_CUDA;
  // W_gu[e] is [2f (contraction), d (output)]: N-major, quantised along 2f
  if (!tmap_3d(&tb, w_gu_col.q, d, 2ull * f, E, d, 2ull * f * d, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsa, dau.s, 2ull * f / 128, m_cap / 128, 1)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsb, w_gu_col.s, 2ull * f / 128, d / 128, E)) return MOE_ERR_CUDA;
  tc::GemmArgs a = mx_m_grouped(c, offsets, E, d, 2 * f, m_cap);
  a.out = dx_perm;
  a.ldo = d;
  return launch<256, false, true, tc::EPI_BF16, false, true, true>(ta, tb, a, c.num_sms, st, &tsa,
                                                                 &tsb);
}

moe_status_t gemm_mx_wgrad(const GemmCtx& c, const MxOperand& a_col, int M, const MxOperand& b_col,
                           int N, const int32_t* offsets, void* dw, int E, int64_t m_cap,
                           cudaStream_t st) {
  // dW[e] (M x N) = A_e^T B_e over e's token rows; both operands are token-major
  // (MN-major) and quantised along tokens (scale atoms over 128 tokens)
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_2d(&ta, a_col.q, M, m_cap, M, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_3d(&tb, b_col.q, N, m_cap, 1, N, 1ull * N * m_cap, 128, 128, true)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsa, a_col.s, m_cap / 128, M / 128, 1)) return MOE_ERR_CUDA;
  if (!tmap_sf(&tsb, b_col.s, m_cap / 128, N / 128, 1)) return MOE_ERR_CUDA;
  tc::GemmArgs a = base_args(c);
  set_n(a, N, 256);
  set_m(a, M, 2 * tc::BM);  // CTA pairs: 256-row tiles
  a.n_groups = E;
  a.offsets = offsets;
  a.total_len = static_cast<int>(m_cap);
  a.uniform_len = static_cast<int>(m_cap);  // one group of m_cap rows when offsets is null
  a.out = dw;
  a.ldo = N;
  a.out_gstride = static_cast<int64_t>(M) * N;
  const int64_t tiles = static_cast<int64_t>(E) * a.m_tiles_fixed * a.n_tiles_n;
  const int grid = static_cast<int>(2 * tiles < c.num_sms ? 2 * tiles : c.num_sms);
  return launch<256, true, true, tc::EPI_BF16, true, true, true>(ta, tb, a, grid, st, &tsa, &tsb);
}

}  // namespace moe
