// extern "C" entry points of libmoe.so (declared and documented in
// include/moe.h): argument checks, workspace carving, launch order.
#include <cstdio>
#include <new>

#include "context.cuh"
#include "gemm.cuh"
#include "kernels.cuh"

namespace {

using moe::ceil_div64;

using moe::aligned;
using moe::check_shape;
using moe::DeviceGuard;

using moe::max_rows;

bool router_on_tensor_cores(int E) { return E > 64; }

// Row stride of the tensor-core router's logits and bf16 dL buffers: E
// rounded up to whole 128-column tiles.
int router_ld(int E) { return (E + 127) / 128 * 128; }

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// 256-row CTA-pair tiles for the M-grouped expert GEMMs when the average
// expert segment spans at least four of them; shorter segments (about 512
// rows at E = 128 and T k = 65536) keep 128-row tiles, whose tail rows waste
// half as much.  The routing is not known on the host, so a skewed routing
// with this average (a few long segments) also gets pairs, which suit it.
bool pair_tiles(const moe_shape_t* s) {
  return static_cast<int64_t>(s->T) * s->top_k >= 1024ll * s->n_experts;
}

moe::GemmCtx gemm_ctx(moe_context* h, bool pair_m) {
  moe::GemmCtx c;
  c.extra_launches = &h->launches;
  c.num_sms = h->num_sms;
  c.ctl = h->ctl;
  c.pair_m = pair_m;
  c.wait_ns = h->wait_ns;
  return c;
}

// Router backward workspace layout.
struct RouterBwdWs {
  size_t dl, db_part, part, total;
  int nblocks, n_part, group_len;
};

RouterBwdWs router_bwd_layout(const moe_context* h, const moe_shape_t* s) {
  RouterBwdWs w{};
  const int T = s->T, d = s->d_model, E = s->n_experts;
  w.nblocks = moe::router_bwd_blocks(h->num_sms);
  size_t off = 0;
  w.dl = off;
  off += align256(router_on_tensor_cores(E) ? static_cast<size_t>(T) * router_ld(E) * 2
                                            : static_cast<size_t>(T) * E * 4);
  w.db_part = off;
  off += align256(static_cast<size_t>(w.nblocks) * E * 4);
  w.part = off;
  if (router_on_tensor_cores(E)) {
    w.n_part = moe::router_dw_groups(h->num_sms, T, d, E, &w.group_len);
  } else {
    w.n_part = moe::router_dw_chunks(h->num_sms, T, d, E, &w.group_len);
  }
  off += align256(static_cast<size_t>(w.n_part) * E * d * 4);
  w.total = off;
  return w;
}

// MXFP8 expert GEMMs: quantised operand copies (E4M3 codes + E8M0 scales in
// the GEMMs' atom order) carved from the workspace.  The forward quantises
// each of its operands once into both orientations: the row-wise copy it
// uses itself goes to the transient region (shared with the backward's own
// copies and with the other calls' scratch), the column-wise copy the
// backward needs (W_gu and W_d along their output axis, x_perm and H along
// tokens) goes to the persistent region that follows, which no other call
// touches.  The backward quantises dO and dAU into both orientations.
struct MxWs {
  // transient, forward
  size_t xq, xs, wguq, wgus, hq, hs, wdq, wds, fwd_total;
  // transient, backward
  size_t doq, dos, dauq, daus, doq_c, dos_c, dauq_c, daus_c, bwd_total;
  // persistent (offsets from the start of the persistent region)
  size_t wdq_c, wds_c, wguq_c, wgus_c, xq_c, xs_c, hq_c, hs_c, keep_total;
};

MxWs mx_layout(const moe_shape_t* s) {
  const size_t M = static_cast<size_t>(max_rows(s)), d = s->d_model, f = s->d_ff,
               E = s->n_experts;
  MxWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  w.xq = take(M * d);           w.xs = take(M * d / 32);
  w.wguq = take(E * 2 * f * d); w.wgus = take(E * 2 * f * d / 32);
  w.hq = take(M * f);           w.hs = take(M * f / 32);
  w.wdq = take(E * d * f);      w.wds = take(E * d * f / 32);
  w.fwd_total = off;
  off = 0;
  w.doq = take(M * d);              w.dos = take(M * d / 32);
  w.dauq = take(M * 2 * f);         w.daus = take(M * 2 * f / 32);
  w.doq_c = take(M * d);            w.dos_c = take(d * M / 32);
  w.dauq_c = take(M * 2 * f);       w.daus_c = take(2 * f * M / 32);
  w.bwd_total = off;
  off = 0;
  w.wdq_c = take(E * d * f);        w.wds_c = take(E * f * d / 32);
  w.wguq_c = take(E * 2 * f * d);   w.wgus_c = take(E * d * 2 * f / 32);
  w.xq_c = take(M * d);             w.xs_c = take(d * M / 32);
  w.hq_c = take(M * f);             w.hs_c = take(f * M / 32);
  w.keep_total = off;
  return w;
}

// Bytes of the workspace's leading scratch region, which every call may
// overwrite (in MXFP8 mode the persistent region follows it).
size_t scratch_bytes(const moe_context* h, const moe_shape_t* s) {
  const int64_t T = s->T, E = s->n_experts;
  size_t need = 0;
  auto upd = [&](size_t v) { need = v > need ? v : need; };
  if (s->dtype == MOE_DTYPE_MXFP8) {
    const MxWs w = mx_layout(s);
    upd(w.fwd_total);
    upd(w.bwd_total);
  }
  upd(align256(static_cast<size_t>(T) * router_ld(static_cast<int>(E)) * 4));       // router logits
  upd(align256(static_cast<size_t>(moe::route_scratch_ints(s->T, s->n_experts)) * 4));  // permute
  upd(router_bwd_layout(h, s).total);                                              // router bwd
  return need;
}

size_t workspace_bytes(const moe_context* h, const moe_shape_t* s) {
  const size_t scratch = scratch_bytes(h, s);
  return s->dtype == MOE_DTYPE_MXFP8 ? scratch + mx_layout(s).keep_total : scratch;
}

moe_status_t check_ws(const moe_context* h, const moe_shape_t* s, void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < workspace_bytes(h, s)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                          \
  do {                                         \
    const moe_status_t _st = (expr);           \
    if (_st != MOE_OK) return _st;             \
  } while (0)

#define MOE_CHECK_HANDLE(h, s)                                  \
  do {                                                          \
    if ((h) == nullptr) return MOE_ERR_INVALID_ARG;             \
    MOE_TRY(check_shape(s));                                    \
  } while (0)

#define MOE_GUARD(h)                         \
  DeviceGuard _guard((h)->device);           \
  if (!_guard.ok) return MOE_ERR_CUDA

template <typename... P>
bool all_nonnull(P... p) { return ((p != nullptr) && ...); }

}  // namespace

extern "C" {

moe_status_t moe_create(moe_handle_t* out, int device) {
  MOE_TRACE();
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(device);
  if (!g.ok) return MOE_ERR_CUDA;
  auto* h = new (std::nothrow) moe_context();
  if (h == nullptr) return MOE_ERR_CUDA;
  h->device = device;
  if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  if (cudaMalloc(&h->ctl, 256) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  if (cudaMemset(h->ctl, 0, 256) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->ctl);
    delete h;
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

moe_status_t moe_destroy(moe_handle_t h) {
  MOE_TRACE();
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  {
    DeviceGuard g(h->device);
    cudaFree(h->ctl);
  }
  delete h;
  return MOE_OK;
}

moe_status_t moe_workspace_size(moe_handle_t h, const moe_shape_t* s, size_t* bytes) {
  MOE_CHECK_HANDLE(h, s);
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *bytes = workspace_bytes(h, s);
  return MOE_OK;
}

moe_status_t moe_max_rows(const moe_shape_t* s, int64_t* rows) {
  MOE_TRY(check_shape(s));
  if (rows == nullptr) return MOE_ERR_INVALID_ARG;
  *rows = max_rows(s);
  return MOE_OK;
}

moe_status_t moe_router_topk(moe_handle_t h, const moe_shape_t* s, const void* x,
                             const void* w_router, const float* bias, const int32_t* route_in,
                             int32_t* topk_idx, float* topk_w, float* probs, float* logits,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(x, w_router, topk_idx, topk_w, probs)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_router, 16)) return MOE_ERR_INVALID_ARG;
  const int T = s->T, d = s->d_model, E = s->n_experts, k = s->top_k;
  const bool renorm = (s->flags & MOE_FLAG_RENORM) != 0;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  if (!router_on_tensor_cores(E)) {
    h->launches += 1;
    return cuda_status(moe::launch_router_fused(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w_router), bias,
        route_in, T, d, E, k, renorm, topk_idx, topk_w, probs, logits, h->ctl, h->num_sms, st));
  }
  // the GEMM writes whole 128-column tiles: straight into `logits` when E
  // fills them, else into the workspace, from which the softmax copies
  // the first E columns of each row to `logits`
  const int ld = router_ld(E);
  float* lg = logits;
  if (lg == nullptr || ld != E) {
    MOE_TRY(check_ws(h, s, ws, ws_bytes));
    lg = static_cast<float*>(ws);
  } else if (!aligned(lg, 16)) {
    return MOE_ERR_INVALID_ARG;
  }
  const moe::GemmCtx c = gemm_ctx(h, false);
  h->launches += 2;
  MOE_TRY(moe::gemm_router_logits(c, x, w_router, lg, T, d, E, ld, st));
  return cuda_status(moe::launch_softmax_topk(lg, ld, bias, route_in, T, E, k, renorm, topk_idx,
                                              topk_w, probs, logits, h->ctl, st));
}

moe_status_t moe_permute(moe_handle_t h, const moe_shape_t* s, const void* x,
                         const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                         int32_t* row_map, void* x_perm, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(x, topk_idx, counts, offsets, row_map, x_perm)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(h, s, ws, ws_bytes));
  const int T = s->T, d = s->d_model, E = s->n_experts, k = s->top_k;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  auto* sub = static_cast<int32_t*>(ws);
  h->launches += 2;
  MOE_TRY(cuda_status(moe::launch_route_count(topk_idx, T, k, E, moe::seg_align(s), sub, counts,
                                              offsets, h->ctl, st)));
  return cuda_status(moe::launch_route_rank_scatter(
      topk_idx, static_cast<const __nv_bfloat16*>(x), T, k, E, sub, offsets, counts, d, row_map,
      static_cast<__nv_bfloat16*>(x_perm), nullptr, st));
}

moe_status_t moe_permute_src(moe_handle_t h, const moe_shape_t* s, const void* x,
                             const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                             int32_t* row_map, int32_t* row_src, void* x_perm, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(x, topk_idx, counts, offsets, row_map, row_src, x_perm))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(h, s, ws, ws_bytes));
  const int T = s->T, d = s->d_model, E = s->n_experts, k = s->top_k;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  auto* sub = static_cast<int32_t*>(ws);
  h->launches += 2;
  MOE_TRY(cuda_status(moe::launch_route_count(topk_idx, T, k, E, moe::seg_align(s), sub, counts,
                                              offsets, h->ctl, st)));
  return cuda_status(moe::launch_route_rank_scatter(
      topk_idx, static_cast<const __nv_bfloat16*>(x), T, k, E, sub, offsets, counts, d, row_map,
      static_cast<__nv_bfloat16*>(x_perm), row_src, st));
}

moe_status_t moe_grouped_swiglu_fwd_combine(moe_handle_t h, const moe_shape_t* s,
                                            const void* x_perm, const int32_t* offsets,
                                            const int32_t* row_map, const int32_t* row_src,
                                            const float* topk_w, const void* w_gu,
                                            const void* w_down, void* au, void* hbuf,
                                            void* o_perm, const void* shared_out, void* y,
                                            int32_t* arrivals, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(x_perm, offsets, row_map, row_src, topk_w, w_gu, w_down, hbuf, o_perm, y,
                   arrivals))
    return MOE_ERR_INVALID_ARG;
  for (const void* p : {x_perm, w_gu, w_down, static_cast<const void*>(au),
                        static_cast<const void*>(hbuf), static_cast<const void*>(o_perm),
                        shared_out, static_cast<const void*>(y)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  const moe::CombineArgs cb{row_src, row_map, topk_w, shared_out, y, arrivals, s->T, s->top_k};
  h->launches += 2;
  MOE_TRY(moe::gemm_fwd_gate_up(c, x_perm, offsets, w_gu, au, hbuf, E, d, f, m_cap, st));
  return moe::gemm_fwd_down_combine(c, hbuf, offsets, w_down, o_perm, E, d, f, m_cap, cb, st);
}

// ---- gather forms (no materialised x_perm; bf16)
moe_status_t moe_route(moe_handle_t h, const moe_shape_t* s, const int32_t* topk_idx,
                       int32_t* counts, int32_t* offsets, int32_t* row_map, int32_t* row_src,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(topk_idx, counts, offsets, row_map, row_src)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(h, s, ws, ws_bytes));
  const int T = s->T, E = s->n_experts, k = s->top_k;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  auto* sub = static_cast<int32_t*>(ws);
  h->launches += 3;
  MOE_TRY(cuda_status(moe::launch_route_count(topk_idx, T, k, E, moe::seg_align(s), sub, counts,
                                              offsets, h->ctl, st)));
  MOE_TRY(cuda_status(moe::launch_route_rank_scatter(topk_idx, nullptr, T, k, E, sub, offsets,
                                                     counts, s->d_model, row_map, nullptr, nullptr,
                                                     st)));
  return cuda_status(
      moe::launch_route_src(row_map, offsets, counts, T, k, E, max_rows(s), row_src, st));
}

moe_status_t moe_grouped_swiglu_fwd_gather(moe_handle_t h, const moe_shape_t* s, const void* x,
                                           const int32_t* row_src, const int32_t* offsets,
                                           const void* w_gu, const void* w_down, void* au,
                                           void* hbuf, void* o_perm, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(x, row_src, offsets, w_gu, w_down, hbuf, o_perm)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x, w_gu, w_down, static_cast<const void*>(au),
                        static_cast<const void*>(hbuf), static_cast<const void*>(o_perm)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  h->launches += 2;
  MOE_TRY(moe::gemm_fwd_gate_up_gather(c, x, s->T, row_src, offsets, w_gu, au, hbuf, E, d, f,
                                       m_cap, st));
  return moe::gemm_fwd_down(c, hbuf, offsets, w_down, o_perm, E, d, f, m_cap, st);
}

moe_status_t moe_grouped_swiglu_recompute_gather(moe_handle_t h, const moe_shape_t* s,
                                                 const void* x, const int32_t* row_src,
                                                 const int32_t* offsets, const void* w_gu,
                                                 void* au, void* hbuf, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(x, row_src, offsets, w_gu, au, hbuf)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x, w_gu, static_cast<const void*>(au), static_cast<const void*>(hbuf)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  h->launches += 1;
  return moe::gemm_fwd_gate_up_gather(c, x, s->T, row_src, offsets, w_gu, au, hbuf, s->n_experts,
                                      s->d_model, s->d_ff, max_rows(s), st);
}

moe_status_t moe_grouped_swiglu_bwd_gather(moe_handle_t h, const moe_shape_t* s,
                                           const void* do_perm, const void* x,
                                           const int32_t* row_src, const void* au,
                                           const void* hbuf, const int32_t* offsets,
                                           const void* w_gu, const void* w_down, void* dau,
                                           void* dx_perm, void* dw_gu, void* dw_down,
                                           moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(do_perm, x, row_src, au, hbuf, offsets, w_gu, w_down, dau, dx_perm, dw_gu,
                   dw_down))
    return MOE_ERR_INVALID_ARG;
  for (const void* p : {do_perm, x, au, hbuf, w_gu, w_down, static_cast<const void*>(dau),
                        static_cast<const void*>(dx_perm), static_cast<const void*>(dw_gu),
                        static_cast<const void*>(dw_down)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  h->launches += 4;
  MOE_TRY(moe::gemm_dgrad_down_swiglu(c, do_perm, offsets, w_down, au, dau, E, d, f, m_cap, st));
  MOE_TRY(moe::gemm_wgrad_down(c, do_perm, hbuf, offsets, dw_down, E, d, f, m_cap, st));
  MOE_TRY(moe::gemm_dgrad_gate_up(c, dau, offsets, w_gu, dx_perm, E, d, f, m_cap, st));
  return moe::gemm_wgrad_gate_up_gather(c, dau, x, s->T, row_src, offsets, dw_gu, E, d, f, m_cap,
                                        st);
}

moe_status_t moe_grouped_swiglu_fwd(moe_handle_t h, const moe_shape_t* s, const void* x_perm,
                                    const int32_t* offsets, const void* w_gu, const void* w_down,
                                    void* au, void* hbuf, void* o_perm, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(x_perm, offsets, w_gu, w_down, hbuf, o_perm)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x_perm, w_gu, w_down, static_cast<const void*>(au),
                        static_cast<const void*>(hbuf), static_cast<const void*>(o_perm)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  if (s->dtype == MOE_DTYPE_MXFP8) {
    MOE_TRY(check_ws(h, s, ws, ws_bytes));
    const MxWs L = mx_layout(s);
    auto* b = static_cast<uint8_t*>(ws);
    auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
    auto* keep = b + scratch_bytes(h, s);  // read by moe_grouped_swiglu_bwd
    // row-wise copy for this call, column-wise copy kept for the backward
    auto both = [&](const void* in, int64_t r, int64_t cols, int64_t group, size_t q, size_t sc,
                    size_t qc, size_t scc) {
      return cuda_status(moe::launch_mxfp8_quantize_both(bf(in), r, cols, group, b + q, b + sc,
                                                         keep + qc, keep + scc, h->num_sms, st));
    };
    h->launches += 6;
    MOE_TRY(both(x_perm, m_cap, d, m_cap, L.xq, L.xs, L.xq_c, L.xs_c));
    MOE_TRY(both(w_gu, 2ll * E * f, d, 2ll * f, L.wguq, L.wgus, L.wguq_c, L.wgus_c));
    MOE_TRY(moe::gemm_mx_fwd_gate_up(c, {b + L.xq, b + L.xs}, offsets, {b + L.wguq, b + L.wgus}, au,
                                     hbuf, E, d, f, m_cap, st));
    MOE_TRY(both(hbuf, m_cap, f, m_cap, L.hq, L.hs, L.hq_c, L.hs_c));
    MOE_TRY(both(w_down, static_cast<int64_t>(E) * d, f, d, L.wdq, L.wds, L.wdq_c, L.wds_c));
    return moe::gemm_mx_fwd_down(c, {b + L.hq, b + L.hs}, offsets, {b + L.wdq, b + L.wds}, o_perm,
                                 E, d, f, m_cap, st);
  }
  h->launches += 2;
  MOE_TRY(moe::gemm_fwd_gate_up(c, x_perm, offsets, w_gu, au, hbuf, E, d, f, m_cap, st));
  return moe::gemm_fwd_down(c, hbuf, offsets, w_down, o_perm, E, d, f, m_cap, st);
}

moe_status_t moe_grouped_swiglu_recompute(moe_handle_t h, const moe_shape_t* s, const void* x_perm,
                                          const int32_t* offsets, const void* w_gu, void* au,
                                          void* hbuf, void* ws, size_t ws_bytes,
                                          moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(x_perm, offsets, w_gu, au, hbuf)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x_perm, w_gu, static_cast<const void*>(au), static_cast<const void*>(hbuf)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  if (s->dtype == MOE_DTYPE_MXFP8) {
    // the forward's operand quantisation and gate/up GEMM, again
    MOE_TRY(check_ws(h, s, ws, ws_bytes));
    const MxWs L = mx_layout(s);
    auto* b = static_cast<uint8_t*>(ws);
    auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
    h->launches += 3;
    MOE_TRY(cuda_status(moe::launch_mxfp8_quantize_atoms(bf(x_perm), m_cap, d, b + L.xq, b + L.xs, st)));
    MOE_TRY(cuda_status(
        moe::launch_mxfp8_quantize_atoms(bf(w_gu), 2ll * E * f, d, b + L.wguq, b + L.wgus, st)));
    return moe::gemm_mx_fwd_gate_up(c, {b + L.xq, b + L.xs}, offsets, {b + L.wguq, b + L.wgus}, au,
                                    hbuf, E, d, f, m_cap, st);
  }
  h->launches += 1;
  return moe::gemm_fwd_gate_up(c, x_perm, offsets, w_gu, au, hbuf, E, d, f, m_cap, st);
}

moe_status_t moe_unpermute_combine(moe_handle_t h, const moe_shape_t* s, const void* o_perm,
                                   const int32_t* row_map, const float* topk_w,
                                   const void* shared_out, void* y, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(o_perm, row_map, topk_w, y)) return MOE_ERR_INVALID_ARG;
  if (!aligned(o_perm, 16) || !aligned(y, 16) || !aligned(shared_out, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_combine(static_cast<const __nv_bfloat16*>(o_perm), row_map, topk_w,
                                         static_cast<const __nv_bfloat16*>(shared_out), s->T,
                                         s->d_model, s->top_k,
                                         static_cast<__nv_bfloat16*>(y),
                                         static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_unpermute_combine_bwd(moe_handle_t h, const moe_shape_t* s, const void* dy,
                                       const void* o_perm, const int32_t* row_map,
                                       const float* topk_w, const int32_t* offsets,
                                       const int32_t* counts, void* do_perm, float* d_topk_w,
                                       moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(dy, o_perm, row_map, topk_w, offsets, counts, do_perm, d_topk_w))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(dy, 16) || !aligned(o_perm, 16) || !aligned(do_perm, 16)) return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_combine_bwd(
      static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(o_perm), row_map,
      topk_w, offsets, counts, s->T, s->d_model, s->top_k, s->n_experts,
      static_cast<__nv_bfloat16*>(do_perm), d_topk_w, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_swiglu_bwd(moe_handle_t h, const moe_shape_t* s, const void* do_perm,
                                    const void* x_perm, const void* au, const void* hbuf,
                                    const int32_t* offsets, const void* w_gu, const void* w_down,
                                    void* dau, void* dx_perm, void* dw_gu, void* dw_down, void* ws,
                                    size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(do_perm, x_perm, au, hbuf, offsets, w_gu, w_down, dau, dx_perm, dw_gu, dw_down))
    return MOE_ERR_INVALID_ARG;
  for (const void* p : {do_perm, x_perm, au, hbuf, w_gu, w_down, static_cast<const void*>(dau),
                        static_cast<const void*>(dx_perm), static_cast<const void*>(dw_gu),
                        static_cast<const void*>(dw_down)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const int d = s->d_model, f = s->d_ff, E = s->n_experts;
  const int64_t m_cap = max_rows(s);
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(s));
  if (s->dtype == MOE_DTYPE_MXFP8) {
    MOE_TRY(check_ws(h, s, ws, ws_bytes));
    const MxWs L = mx_layout(s);
    auto* b = static_cast<uint8_t*>(ws);
    auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
    auto both = [&](const void* in, int64_t r, int64_t cols, size_t q, size_t sc, size_t qc,
                    size_t scc) {
      return cuda_status(moe::launch_mxfp8_quantize_both(bf(in), r, cols, r, b + q, b + sc, b + qc,
                                                         b + scc, h->num_sms, st));
    };
    // the forward's column-wise copies of W_d, W_gu, H and x_perm
    const uint8_t* keep = b + scratch_bytes(h, s);
    h->launches += 6;
    // dgrad of the down projection (+ SwiGLU backward): dO along d, W_d along d
    MOE_TRY(both(do_perm, m_cap, d, L.doq, L.dos, L.doq_c, L.dos_c));
    MOE_TRY(moe::gemm_mx_dgrad_down_swiglu(c, {b + L.doq, b + L.dos}, offsets,
                                           {keep + L.wdq_c, keep + L.wds_c}, au, dau, E, d, f,
                                           m_cap, st));
    // dgrad of gate/up: dAU along 2f, W_gu along 2f
    MOE_TRY(both(dau, m_cap, 2ll * f, L.dauq, L.daus, L.dauq_c, L.daus_c));
    MOE_TRY(moe::gemm_mx_dgrad_gate_up(c, {b + L.dauq, b + L.daus}, offsets,
                                       {keep + L.wguq_c, keep + L.wgus_c}, dx_perm, E, d, f, m_cap,
                                       st));
    // weight gradients: every operand along tokens
    MOE_TRY(moe::gemm_mx_wgrad(c, {b + L.doq_c, b + L.dos_c}, d, {keep + L.hq_c, keep + L.hs_c}, f,
                               offsets, dw_down, E, m_cap, st));
    return moe::gemm_mx_wgrad(c, {b + L.dauq_c, b + L.daus_c}, 2 * f,
                              {keep + L.xq_c, keep + L.xs_c}, d, offsets, dw_gu, E, m_cap, st);
  }
  h->launches += 4;
  MOE_TRY(moe::gemm_dgrad_down_swiglu(c, do_perm, offsets, w_down, au, dau, E, d, f, m_cap, st));
  MOE_TRY(moe::gemm_wgrad_down(c, do_perm, hbuf, offsets, dw_down, E, d, f, m_cap, st));
  MOE_TRY(moe::gemm_dgrad_gate_up(c, dau, offsets, w_gu, dx_perm, E, d, f, m_cap, st));
  return moe::gemm_wgrad_gate_up(c, dau, x_perm, offsets, dw_gu, E, d, f, m_cap, st);
}

// Shared expert: the routed experts' GEMMs over one group of all T tokens,
// read in place from x / dY (no permute); tensor maps are exactly T rows
// tall, so a ragged last tile reads zeros.
moe_status_t moe_shared_expert_fwd(moe_handle_t h, const moe_shape_t* s, const void* x,
                                   const void* w_gu_s, const void* w_d_s, void* au_s, void* h_s,
                                   void* o_s, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(x, w_gu_s, w_d_s, au_s, h_s, o_s)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x, w_gu_s, w_d_s, static_cast<const void*>(au_s),
                        static_cast<const void*>(h_s), static_cast<const void*>(o_s)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const moe_shape_t one{s->T, s->d_model, s->d_ff, 1, 1, MOE_DTYPE_BF16, 0};
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(&one));
  h->launches += 2;
  MOE_TRY(moe::gemm_fwd_gate_up(c, x, nullptr, w_gu_s, au_s, h_s, 1, s->d_model, s->d_ff, s->T, st));
  return moe::gemm_fwd_down(c, h_s, nullptr, w_d_s, o_s, 1, s->d_model, s->d_ff, s->T, st);
}

moe_status_t moe_shared_expert_bwd(moe_handle_t h, const moe_shape_t* s, const void* dy,
                                   const void* x, const void* au_s, const void* h_s,
                                   const void* w_gu_s, const void* w_d_s, void* dau_s, void* dx_s,
                                   void* dw_gu_s, void* dw_d_s, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(dy, x, au_s, h_s, w_gu_s, w_d_s, dau_s, dx_s, dw_gu_s, dw_d_s))
    return MOE_ERR_INVALID_ARG;
  for (const void* p : {dy, x, au_s, h_s, w_gu_s, w_d_s, static_cast<const void*>(dau_s),
                        static_cast<const void*>(dx_s), static_cast<const void*>(dw_gu_s),
                        static_cast<const void*>(dw_d_s)})
    if (!aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  const moe_shape_t one{s->T, s->d_model, s->d_ff, 1, 1, MOE_DTYPE_BF16, 0};
  const int d = s->d_model, f = s->d_ff, T = s->T;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const moe::GemmCtx c = gemm_ctx(h, pair_tiles(&one));
  h->launches += 4;
  MOE_TRY(moe::gemm_dgrad_down_swiglu(c, dy, nullptr, w_d_s, au_s, dau_s, 1, d, f, T, st));
  MOE_TRY(moe::gemm_wgrad_down(c, dy, h_s, nullptr, dw_d_s, 1, d, f, T, st));
  MOE_TRY(moe::gemm_dgrad_gate_up(c, dau_s, nullptr, w_gu_s, dx_s, 1, d, f, T, st));
  return moe::gemm_wgrad_gate_up(c, dau_s, x, nullptr, dw_gu_s, 1, d, f, T, st);
}

moe_status_t moe_permute_bwd(moe_handle_t h, const moe_shape_t* s, const void* dx_perm,
                             const int32_t* row_map, const float* dx_router, const void* dx_shared,
                             void* dx, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(dx_perm, row_map, dx)) return MOE_ERR_INVALID_ARG;
  if (!aligned(dx_perm, 16) || !aligned(dx, 16) || !aligned(dx_router, 16) ||
      !aligned(dx_shared, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_permute_bwd(static_cast<const __nv_bfloat16*>(dx_perm), row_map,
                                             dx_router,
                                             static_cast<const __nv_bfloat16*>(dx_shared), s->T,
                                             s->d_model, s->top_k,
                                             static_cast<__nv_bfloat16*>(dx),
                                             static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute_router_bwd(moe_handle_t h, const moe_shape_t* s, const void* dx_perm,
                                    const int32_t* row_map, const float* d_topk_w,
                                    const float* probs, const int32_t* topk_idx,
                                    const float* d_probs_aux, const void* w_router,
                                    const void* dx_shared, void* dx, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (s->n_experts > 64) return MOE_ERR_UNSUPPORTED;
  if (!all_nonnull(dx_perm, row_map, d_topk_w, probs, topk_idx, w_router, dx))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(dx_perm, 16) || !aligned(dx, 16) || !aligned(w_router, 16) ||
      !aligned(dx_shared, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_permute_router_bwd(
      static_cast<const __nv_bfloat16*>(dx_perm), row_map, d_topk_w, probs, topk_idx, d_probs_aux,
      static_cast<const __nv_bfloat16*>(w_router), static_cast<const __nv_bfloat16*>(dx_shared),
      s->T, s->d_model, s->n_experts, s->top_k,
      (s->flags & MOE_FLAG_RENORM) != 0, static_cast<__nv_bfloat16*>(dx),
      static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_router_topk_bwd(moe_handle_t h, const moe_shape_t* s, const float* d_topk_w,
                                 const float* probs, const int32_t* topk_idx,
                                 const float* d_probs_aux, const void* x,
                                 const void* w_router, float* dx_router, void* dw_router,
                                 float* dbias, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(d_topk_w, probs, topk_idx, x, w_router, dw_router)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(dx_router, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(h, s, ws, ws_bytes));
  const int T = s->T, d = s->d_model, E = s->n_experts, k = s->top_k;
  const bool renorm = (s->flags & MOE_FLAG_RENORM) != 0;
  auto st = static_cast<cudaStream_t>(stream);
  MOE_GUARD(h);
  const RouterBwdWs L = router_bwd_layout(h, s);
  auto* base = static_cast<uint8_t*>(ws);
  auto* db_part = reinterpret_cast<float*>(base + L.db_part);
  auto* part = reinterpret_cast<float*>(base + L.part);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wb = static_cast<const __nv_bfloat16*>(w_router);
  const bool want_dx = dx_router != nullptr;
  if (!router_on_tensor_cores(E)) {
    // dL and its per-block db sums (and dX_router when asked), then dW_r
    // partial rows in one pass over x, then one reduction for dW_r and db
    h->launches += 3;
    auto* dl = reinterpret_cast<float*>(base + L.dl);
    MOE_TRY(cuda_status(moe::launch_router_bwd_dl(d_topk_w, probs, topk_idx, d_probs_aux, wb, T, d,
                                                  E, k, renorm, want_dx, dl, nullptr, 0, dx_router,
                                                  db_part,
                                                  L.nblocks, h->ctl, st)));
    MOE_TRY(cuda_status(
        moe::launch_router_dw(dl, xb, T, d, E, L.n_part, L.group_len, part, h->ctl, st)));
    return cuda_status(moe::launch_reduce_dw(part, L.n_part, static_cast<int64_t>(E) * d, db_part,
                                             L.nblocks, E, static_cast<__nv_bfloat16*>(dw_router),
                                             dbias, st));
  }
  // E above 64: dL in bf16 (row stride router_ld(E)), both products on the
  // tensor cores
  h->launches += want_dx ? 4 : 3;
  auto* dl = reinterpret_cast<__nv_bfloat16*>(base + L.dl);
  const int ld = router_ld(E);
  MOE_TRY(cuda_status(moe::launch_router_bwd_dl(d_topk_w, probs, topk_idx, d_probs_aux, wb, T, d, E,
                                                k, renorm, false, nullptr, dl, ld, nullptr, db_part,
                                                L.nblocks, h->ctl, st)));
  const moe::GemmCtx c = gemm_ctx(h, false);
  if (want_dx) MOE_TRY(moe::gemm_router_dx(c, dl, ld, w_router, dx_router, T, d, E, st));
  MOE_TRY(moe::gemm_router_dw_partial(c, dl, ld, x, part, T, d, E, L.n_part, L.group_len, st));
  return cuda_status(moe::launch_reduce_dw(part, L.n_part, static_cast<int64_t>(E) * d, db_part,
                                           L.nblocks, E, static_cast<__nv_bfloat16*>(dw_router),
                                           dbias, st));
}

moe_status_t moe_router_load_stats(moe_handle_t h, const moe_shape_t* s, const float* probs,
                                   const int32_t* counts, int accumulate, float* stats, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (!all_nonnull(probs, counts, stats)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(h, s, ws, ws_bytes));
  const int nb = moe::router_stats_blocks(h->num_sms, s->T);
  if (static_cast<size_t>(nb) * s->n_experts * 4 > ws_bytes) return MOE_ERR_WORKSPACE;
  MOE_GUARD(h);
  h->launches += 2;
  return cuda_status(moe::launch_router_load_stats(probs, counts, s->T, s->n_experts, nb,
                                                   accumulate != 0, static_cast<float*>(ws), stats,
                                                   static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_router_aux_loss(moe_handle_t h, const moe_shape_t* s, const float* stats,
                                 int64_t n_tokens, float alpha, float* loss, float* d_probs_aux,
                                 moe_stream_t stream) {
  MOE_TRACE();
  MOE_CHECK_HANDLE(h, s);
  if (stats == nullptr || (loss == nullptr && d_probs_aux == nullptr)) return MOE_ERR_INVALID_ARG;
  if (n_tokens < 1 || !(alpha >= 0.f)) return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_router_aux_loss(stats, s->n_experts, s->top_k,
                                                 static_cast<float>(n_tokens), alpha, loss,
                                                 d_probs_aux, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_mxfp8_quantize(moe_handle_t h, const void* in, int64_t rows, int64_t cols,
                                int axis, uint8_t* q, uint8_t* scales, moe_stream_t stream) {
  MOE_TRACE();
  if (h == nullptr || !all_nonnull(in, q, scales)) return MOE_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || (axis != 0 && axis != 1)) return MOE_ERR_INVALID_ARG;
  if (axis == 1 && (cols % 32 != 0 || !aligned(in, 16) || !aligned(q, 16)))
    return MOE_ERR_INVALID_ARG;
  if (axis == 0 && (rows % 32 != 0 || cols % 2 != 0 || !aligned(in, 4) || !aligned(q, 2) ||
                    !aligned(scales, 2)))
    return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_mxfp8_quantize(static_cast<const __nv_bfloat16*>(in), rows, cols,
                                                axis, q, scales, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_mxfp8_quantize_gemm(moe_handle_t h, const void* in, int64_t rows, int64_t cols,
                                     int64_t rows_per_group, uint8_t* q_row, uint8_t* s_row,
                                     uint8_t* q_col, uint8_t* s_col, moe_stream_t stream) {
  MOE_TRACE();
  if (h == nullptr || !all_nonnull(in, q_row, s_row) || !all_nonnull(q_col, s_col))
    return MOE_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || rows_per_group < 1 || cols % 128 != 0 || rows_per_group % 128 != 0 ||
      rows % rows_per_group != 0)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(q_row, 16) || !aligned(q_col, 16)) return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  h->launches += 1;
  return cuda_status(moe::launch_mxfp8_quantize_both(static_cast<const __nv_bfloat16*>(in), rows,
                                                     cols, rows_per_group, q_row, s_row, q_col,
                                                     s_col, h->num_sms,
                                                     static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_status(moe_handle_t h, int* device_status) {
  MOE_TRACE();
  if (h == nullptr || device_status == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_GUARD(h);
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  moe::DeviceCtl c{};
  if (cudaMemcpy(&c, h->ctl, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(h->ctl, 0, sizeof(c)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = c.status;
  return MOE_OK;
}

moe_status_t moe_set_wait_limit(moe_handle_t h, uint64_t ns) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  h->wait_ns = ns;
  return MOE_OK;
}

moe_status_t moe_get_launch_count(moe_handle_t h, uint64_t* launches) {
  if (h == nullptr || launches == nullptr) return MOE_ERR_INVALID_ARG;
  *launches = h->launches;
  return MOE_OK;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_DEVICE_CHECK: return "device-side index check failed";
    case MOE_ERR_TIMEOUT: return "device-side bounded wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
