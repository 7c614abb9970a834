// Declarations of the memory-bound kernels' host launchers (router,
// routing metadata, permute, combine and their backwards, MXFP8 quantise).
#pragma once

#include "common.cuh"

namespace moe {

// Routing metadata: a warp counts kCountTokens tokens (k flat (token, slot)
// entries each), eight such chunks to a block; a block ranks and copies
// kChunkTokens tokens.
constexpr int kCountTokens = 64;
constexpr int kChunkTokens = 16;

inline int64_t count_chunks(int T) { return ceil_div64(T, kCountTokens); }
inline int64_t count_blocks(int T) { return ceil_div64(count_chunks(T), 8); }
// int32 scratch of the two routing-metadata launches
inline int64_t route_scratch_ints(int T, int E) {
  return static_cast<int64_t>(E) * (count_chunks(T) + count_blocks(T));
}

// ---- router forward
cudaError_t launch_router_fused(const __nv_bfloat16* x, const __nv_bfloat16* w_r, const float* bias,
                                const int32_t* route_in, int T, int d, int E, int k, bool renorm,
                                int32_t* idx, float* w, float* probs, float* logits,
                                DeviceCtl* ctl, int num_sms, cudaStream_t st);
// logits_in has row stride ld_in; logits_out (dense [T, E]) may alias it when ld_in = E
cudaError_t launch_softmax_topk(const float* logits_in, int ld_in, const float* bias,
                                const int32_t* route_in, int T, int E, int k, bool renorm,
                                int32_t* idx, float* w, float* probs, float* logits_out,
                                DeviceCtl* ctl, cudaStream_t st);

// ---- router load statistics and load-balancing loss
int router_stats_blocks(int num_sms, int T);
// partial: router_stats_blocks() x E floats of scratch
cudaError_t launch_router_load_stats(const float* probs, const int32_t* counts, int T, int E,
                                     int n_blocks, bool accumulate, float* partial, float* stats,
                                     cudaStream_t st);
cudaError_t launch_router_aux_loss(const float* stats, int E, int k, float n_tokens, float alpha,
                                   float* loss, float* dprob, cudaStream_t st);

// ---- routing metadata + permute
// counts, padded offsets and, in scratch (route_scratch_ints), the chunk and
// block bases (one launch; its last block scans; `ctl->ticket` must be 0).
cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int align,
                               int32_t* scratch, int32_t* counts, int32_t* offsets,
                               DeviceCtl* ctl, cudaStream_t st);
// row_map, and with x_perm non-null the permuted copy (pad rows zeroed) and,
// with row_src also non-null, the token of every row in a segment (T on the
// segments' pad rows; rows past the last segment are not written).
cudaError_t launch_route_rank_scatter(const int32_t* idx, const __nv_bfloat16* x, int T, int k,
                                      int E, const int32_t* scratch, const int32_t* offsets,
                                      const int32_t* counts, int d, int32_t* row_map,
                                      __nv_bfloat16* x_perm, int32_t* row_src, cudaStream_t st);
// row_src [m_cap]: source token of every routed row, T for pad rows and rows
// past the last segment.
cudaError_t launch_route_src(const int32_t* row_map, const int32_t* offsets, const int32_t* counts,
                             int T, int k, int E, int64_t m_cap, int32_t* row_src,
                             cudaStream_t st);

// ---- combine and backwards
cudaError_t launch_combine(const __nv_bfloat16* o_perm, const int32_t* row_map, const float* w,
                           const __nv_bfloat16* shared, int T, int d, int k, __nv_bfloat16* y,
                           cudaStream_t st);
cudaError_t launch_combine_bwd(const __nv_bfloat16* dy, const __nv_bfloat16* o_perm,
                               const int32_t* row_map, const float* w, const int32_t* offsets,
                               const int32_t* counts, int T, int d, int k, int E,
                               __nv_bfloat16* do_perm, float* dw, cudaStream_t st);
cudaError_t launch_permute_bwd(const __nv_bfloat16* dx_perm, const int32_t* row_map,
                               const float* dx_router, const __nv_bfloat16* dx_shared, int T, int d,
                               int k, __nv_bfloat16* dx, cudaStream_t st);

// ---- router backward
// dX = bf16(unpermute-reduce of dX_perm + dL W_r) in one pass, E <= 64.
cudaError_t launch_permute_router_bwd(const __nv_bfloat16* dx_perm, const int32_t* row_map,
                                      const float* dw, const float* probs, const int32_t* idx,
                                      const float* dprob_aux, const __nv_bfloat16* w_r,
                                      const __nv_bfloat16* dx_shared, int T, int d, int E, int k,
                                      bool renorm, __nv_bfloat16* dx, cudaStream_t st);
int router_bwd_blocks(int num_sms);
cudaError_t launch_router_bwd_dl(const float* dw, const float* probs, const int32_t* idx,
                                 const float* dprob_aux, const __nv_bfloat16* w_r, int T, int d,
                                 int E, int k, bool renorm,
                                 bool fuse_dx, float* dl_f32, __nv_bfloat16* dl_bf16,
                                 int ld_bf16, float* dx_router, float* db_partial, int nblocks,
                                 DeviceCtl* ctl, cudaStream_t st);
// dW_r partial rows [n_chunks][E*d] over token chunks (E <= 64; E <= 16 streamed
// with bulk copies, the dL buffer padded to a multiple of 256 bytes);
// router_dw_chunks picks the chunking.
int router_dw_chunks(int num_sms, int T, int d, int E, int* group_len);
cudaError_t launch_router_dw(const float* dl, const __nv_bfloat16* x, int T, int d, int E,
                             int n_chunks, int group_len, float* partial, DeviceCtl* ctl,
                             cudaStream_t st);
// dw_out = bf16(sum of the n_part partial rows of n_w floats); when db_out
// is given also db_out = sum of the n_db rows of E floats in db_part.
cudaError_t launch_reduce_dw(const float* partial, int n_part, int64_t n_w, const float* db_part,
                             int n_db, int E, __nv_bfloat16* dw_out, float* db_out,
                             cudaStream_t st);


// ---- MXFP8
cudaError_t launch_mxfp8_quantize(const __nv_bfloat16* in, int64_t rows, int64_t cols, int axis,
                                  uint8_t* q, uint8_t* scales, cudaStream_t st);
// GEMM operands (scales in the tensor cores' 512-byte atom order; see
// mxfp8.cu).  Row-wise: [rows, cols] along cols, rows and cols multiples of
// 128.  Column-wise: 32-row blocks along the rows of each group of
// rows_per_group rows, the column being the MN index; cols and
// rows_per_group multiples of 128.
cudaError_t launch_mxfp8_quantize_atoms(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                        uint8_t* q, uint8_t* scales, cudaStream_t st);
// Both at once from one read: row-wise codes/scales (q_row, s_row) and
// column-wise ones per group of rows_per_group rows (q_col, s_col); rows a
// multiple of 32, cols and rows_per_group multiples of 128.
cudaError_t launch_mxfp8_quantize_both(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                       int64_t rows_per_group, uint8_t* q_row, uint8_t* s_row,
                                       uint8_t* q_col, uint8_t* s_col, int num_sms,
                                       cudaStream_t st);

}  // namespace moe
