/*
 * moe.h -- C ABI of libmoe.so, the dropless mixture-of-experts expert layer
 * (one training step, one GPU, NVIDIA B200 / sm_100a).
 *
 * The layer, as the Olmo-core 3 pages describe it in words:
 *   - a router computes a score distribution over the experts for every
 *     token and keeps the k best (discosf.com article on Olmo-core 3,
 *     section 1.1 "sparse computation" and section 2.1 "how a token is sent
 *     to the experts in one forward pass");
 *   - the routing metadata stays on the GPU so the host never waits for a
 *     copy back; routed tokens are written straight into each expert's
 *     contiguous input buffer; all experts' small GEMMs run as one grouped
 *     GEMM whose schedule is read on the device (Olmo-core 3 introduction
 *     page, section 2 "three parallelisms plus three routing
 *     optimisations");
 *   - no token is dropped when an expert is over-subscribed (vibecoding.ru
 *     news item on Olmo-core 3, paragraph on grouped_gemm and dropless MoE);
 *   - expert outputs are put back in the original token order (discosf.com
 *     article, section 2.1);
 *   - MXFP8 is offered for selected operations (Olmo-core 3 introduction
 *     page, section 3 "MXFP8").
 * The pages give no formulas; the readings used are stated per call.
 *
 * Conventions for every call below
 *   - Pointers named as device pointers must point to device memory of the
 *     handle's device; all of them are owned by the caller.  No call
 *     allocates, frees or copies to the host; all scratch comes from `ws`
 *     (size from moe_workspace_size).  The one exception is moe_create,
 *     which allocates a 256-byte control block freed by moe_destroy.
 *   - Every call only enqueues work on `stream` (a cudaStream_t, may be 0)
 *     and returns; nothing synchronises the host except moe_get_status.
 *   - Host-side checks run before any launch: a NULL required pointer, a
 *     bad size or a misaligned pointer returns MOE_ERR_INVALID_ARG, a shape
 *     outside the supported set returns MOE_ERR_UNSUPPORTED, and nothing is
 *     launched.  A failed launch returns MOE_ERR_CUDA.
 *   - Problems only the device can see (an expert id outside [0, E) in a
 *     caller-written topk_idx, a bounded wait that ran out) never trap: the
 *     kernel records a code in the handle's status word, skips the bad
 *     entry, and moe_get_status reports it later.
 *   - Every call that takes a stream, and moe_create, moe_destroy and
 *     moe_get_status, opens one NVTX range named for itself and closes it
 *     before returning (NVTX 3, header-only; a no-op without a tool).
 *   - Layouts are row-major.  bf16 = bfloat16 (round to nearest even).
 *   - Supported shapes: 1 <= k <= min(E, 8), 1 <= E <= 1024, T >= 1,
 *     d_model and d_ff multiples of 128.
 *
 * Routed-row space.  Every expert e owns a segment of rows
 * [offsets[e], offsets[e+1]) in the permuted buffers; segments start at
 * multiples of A rows (A = 32, or 128 when dtype is MOE_DTYPE_MXFP8), hold
 * counts[e] real rows in ascending (token, slot) order followed by zero pad
 * rows.  Buffers in this space have M_cap rows (moe_max_rows): T*k + 31*E,
 * or roundup(T*k + 127*E, 128) in MXFP8 mode; rows at and past offsets[E]
 * are never written.
 *
 * MXFP8 mode (shape dtype MOE_DTYPE_MXFP8): the expert GEMMs of
 * moe_grouped_swiglu_fwd/bwd quantise every operand along its contraction
 * axis (E4M3 elements, one E8M0 scale per 32) into the workspace and run
 * block-scaled tcgen05 MMAs with fp32 accumulation; their outputs stay
 * bf16.  The router, permute and combine are unchanged.  The workspace then
 * has two parts: a leading scratch region that every call may overwrite,
 * and a persistent region after it into which moe_grouped_swiglu_fwd writes
 * the column-wise quantised W_gu, W_down, x_perm and h that
 * moe_grouped_swiglu_bwd reads.  So in MXFP8 mode the backward must get the
 * workspace the forward of the same step used, and nothing else may write
 * past the scratch region in between (no other call of this library does).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_CUDA = 3,
  MOE_ERR_WORKSPACE = 4,
  MOE_ERR_DEVICE_CHECK = 5, /* device saw a bad index / offset */
  MOE_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up */
} moe_status_t;

enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_MXFP8 = 1 };
enum { MOE_FLAG_RENORM = 1 }; /* gate weights divided by their sum over k */

typedef struct moe_shape {
  int T;         /* tokens */
  int d_model;   /* d */
  int d_ff;      /* f, per-expert hidden width */
  int n_experts; /* E */
  int top_k;     /* k */
  int dtype;     /* MOE_DTYPE_BF16 or MOE_DTYPE_MXFP8 (expert GEMM operands) */
  int flags;     /* MOE_FLAG_* */
} moe_shape_t;

typedef struct moe_context* moe_handle_t;

typedef void* moe_stream_t; /* a cudaStream_t */

/* Creates a handle bound to CUDA device `device`: caches the SM count and
 * allocates the device status word.  *h receives the handle.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_create(moe_handle_t* h, int device);

/* Frees the handle's control block.  Pending work must have finished.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_destroy(moe_handle_t h);

/* Bytes of scratch every step call of this shape may use, in one buffer
 * shared by all calls (calls on one stream run in order, so they can share
 * it).  Must be 256-byte aligned.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_workspace_size(moe_handle_t h, const moe_shape_t* s, size_t* bytes);

/* M_cap: rows of every buffer in the routed-row space (see above).
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_max_rows(const moe_shape_t* s, int64_t* rows);

/* Router forward (top-k softmax).  The pages: a router network scores each
 * token over the experts and the k highest are kept (discosf.com article on
 * Olmo-core 3, sections 1.1 and 2.1); the trillion-scale runs route at
 * random (Olmo-core 3 introduction page, key-numbers caveats), which
 * route_in serves.  Softmax before top-k, no renormalisation and the tie
 * rule are readings (the pages give no formula).
 *   L[t,e] = sum_i x[t,i] * w_router[e,i] (+ bias[e]), fp32 accumulate;
 *   probs  = softmax over all E experts, fp32;
 *   topk_idx[t, 0..k-1] = the k largest L[t,:], ties to the lower expert
 *     index, ordered by descending logit;  when route_in != NULL its ids
 *     are used instead (random-routing benchmark mode of the pages);
 *   topk_w[t,j] = probs[t, topk_idx[t,j]] (divided by their sum when
 *     MOE_FLAG_RENORM).
 * In : x [T,d] bf16, w_router [E,d] bf16, bias [E] fp32 or NULL,
 *      route_in [T,k] int32 or NULL (must hold k distinct ids in [0,E)).
 * Out: topk_idx [T,k] int32, topk_w [T,k] fp32, probs [T,E] fp32 (kept for
 *      the backward), logits [T,E] fp32 or NULL (optional copy of L).
 * One warp per token does the softmax and the top-k in registers. */
MOE_API moe_status_t moe_router_topk(moe_handle_t h, const moe_shape_t* s,
                             const void* x, const void* w_router, const float* bias,
                             const int32_t* route_in, int32_t* topk_idx, float* topk_w,
                             float* probs, float* logits, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/* Routing metadata + rowwise permute, all on the device.  The pages: the
 * routing metadata stays on the GPU so the host never waits for a copy back,
 * and routed tokens are written straight into each expert's input buffer
 * (Olmo-core 3 introduction page, section 2, GPU-resident routing and
 * rowwise expert parallelism); the routing result becomes a permutation
 * index that regroups tokens per expert (discosf.com article on Olmo-core 3,
 * section 2.1).  Expert-major stable order and 32-row segment padding are
 * readings.
 *   counts[e]   = number of (t,j) with topk_idx[t,j] == e;
 *   offsets[e]  = sum_{e'<e} roundup(counts[e'], A); offsets[E] = M_pad
 *                 (A = 32, or 128 in MXFP8 mode);
 *   row_map[t,j]= offsets[e] + #{(t',j') before (t,j) in t*k+j order with
 *                 the same expert e};
 *   x_perm[row_map[t,j]] = x[t]; pad rows of every segment are zero.
 * In : x [T,d] bf16, topk_idx [T,k] int32.
 * Out: counts [E] int32, offsets [E+1] int32, row_map [T,k] int32,
 *      x_perm [M_cap,d] bf16.
 * An id outside [0,E) sets MOE_ERR_DEVICE_CHECK and that entry is skipped
 * (its row_map entry is -1). */
MOE_API moe_status_t moe_permute(moe_handle_t h, const moe_shape_t* s, const void* x,
                         const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                         int32_t* row_map, void* x_perm, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* moe_permute without a workspace argument, for callers that cannot provide
 * scratch memory at all (no workspace buffer and no permission to allocate,
 * e.g. a plug-in inside a host program that owns every byte of device memory,
 * or a latency-critical path that must never call cudaMalloc).  The pages
 * describe no such call; it is an addition of this library.
 * Same arguments, outputs and device-side checks as moe_permute.  Its scratch
 * is a fixed 1 MiB array inside the library (one per GPU that loads it, held
 * until the process exits), so the shape must satisfy
 *   (ceil(T / 64) + ceil(T / 512)) * E <= MOE_NOALLOC_SCRATCH_INTS,
 * otherwise MOE_ERR_WORKSPACE is returned before any launch.  The first call
 * on a device looks up the array's device address (a host-side step, done
 * once per device with that device current); make that first call before
 * any stream capture.  The address is kept per CUDA context: after a device
 * reset the next call looks it up again, so make that call before any
 * capture too.  All calls share the array: calls whose work can
 * overlap on the GPU (unordered streams, several host threads) race on it.
 * Nothing is allocated or freed by this call. */
#define MOE_NOALLOC_SCRATCH_INTS (1 << 18)
MOE_API moe_status_t moe_permute_noalloc(moe_handle_t h, const moe_shape_t* s, const void* x,
                                         const int32_t* topk_idx, int32_t* counts,
                                         int32_t* offsets, int32_t* row_map, void* x_perm,
                                         moe_stream_t stream);

/* Grouped SwiGLU expert FFN, forward.  The pages: all experts' small GEMMs
 * run as one grouped GEMM whose schedule is read on the device (Olmo-core 3
 * introduction page, section 2, grouped GEMM and device-scheduled grouped
 * GEMM), and no token is dropped when an expert is over-subscribed
 * (vibecoding.ru news item on Olmo-core 3, paragraph on grouped_gemm and
 * dropless MoE).  The SwiGLU form without biases is a reading.
 * For the rows of expert e:
 *   A = X W_gu[e][0:f]^T, U = X W_gu[e][f:2f]^T   (fp32 accumulate)
 *   au[:, 0:f] = bf16(A), au[:, f:2f] = bf16(U)   (saved for the backward)
 *   h = bf16(silu(A) * U), silu(z) = z / (1 + exp(-z))
 *   o_perm = bf16(h W_down[e]^T)
 * In : x_perm [M_cap,d] bf16, offsets [E+1] int32 (from moe_permute),
 *      w_gu [E,2f,d] bf16, w_down [E,d,f] bf16.
 * Out: au [M_cap,2f] bf16 (or NULL: not kept, for activation recompute),
 *      h [M_cap,f] bf16, o_perm [M_cap,d] bf16.
 * Persistent tcgen05/TMEM kernels fed by TMA; the tile schedule is decoded
 * from `offsets` on the device. */
MOE_API moe_status_t moe_grouped_swiglu_fwd(moe_handle_t h, const moe_shape_t* s, const void* x_perm,
                                    const int32_t* offsets, const void* w_gu,
                                    const void* w_down, void* au, void* hbuf, void* o_perm,
                                    void* ws, size_t ws_bytes, moe_stream_t stream);

/* Activation recompute (the pages: recomputing activations in the backward
 * cuts about two thirds of activation memory for about a fifth of
 * throughput -- Olmo-core 3 introduction page, section 4).  Recomputes the
 * forward's gate/up GEMM and SwiGLU for the backward: the same au and h, bit
 * for bit, as moe_grouped_swiglu_fwd on the same inputs (MXFP8 mode
 * re-quantises x_perm and w_gu in the workspace first).  With it the
 * forward can run with au = NULL and h as a transient buffer, and only
 * x_perm and o_perm need to live from the forward to the backward.
 * In : x_perm [M_cap,d] bf16, offsets [E+1], w_gu [E,2f,d] bf16.
 * Out: au [M_cap,2f] bf16, h [M_cap,f] bf16. */
MOE_API moe_status_t moe_grouped_swiglu_recompute(moe_handle_t h, const moe_shape_t* s,
                                                  const void* x_perm, const int32_t* offsets,
                                                  const void* w_gu, void* au, void* hbuf, void* ws,
                                                  size_t ws_bytes, moe_stream_t stream);

/* moe_permute that also writes row_src [M_cap] int32: the token whose copy
 * each routed row holds, T on the segments' pad rows (rows past offsets[E]
 * are not written).  Same passages as moe_permute (Olmo-core 3 introduction
 * page, section 2; discosf.com article on Olmo-core 3, section 2.1); it
 * feeds moe_grouped_swiglu_fwd_combine.  Same workspace and checks. */
MOE_API moe_status_t moe_permute_src(moe_handle_t h, const moe_shape_t* s, const void* x,
                                     const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                                     int32_t* row_map, int32_t* row_src, void* x_perm, void* ws,
                                     size_t ws_bytes, moe_stream_t stream);

/* moe_grouped_swiglu_fwd with the weighted unpermute-combine fused into the
 * down projection's epilogue ("restore" step: discosf.com article on
 * Olmo-core 3, section 2.1; the grouped GEMM: Olmo-core 3 introduction page,
 * section 2).  Besides au, h and o_perm it writes
 *   y[t] = bf16( sum_j topk_w[t,j] * o_perm[row_map[t,j]] + shared_out[t] ),
 * the same bits as moe_unpermute_combine on the same inputs: every stored
 * routed row counts one arrival for its token and column tile of 256, and
 * the epilogue that completes a token's valid rows sums them in slot order
 * from the stored bf16 rows (no floating-point atomics) and clears the
 * count.  bf16 only (MOE_ERR_UNSUPPORTED for MXFP8).
 * In : as moe_grouped_swiglu_fwd, plus row_map [T,k], row_src [M_cap] (from
 *      moe_permute_src), topk_w [T,k] fp32, shared_out [T,d] bf16 or NULL
 *      (a shared expert's output, computed before this call).
 * Out: au (or NULL), h, o_perm as moe_grouped_swiglu_fwd; y [T,d] bf16.
 * arrivals [T, ceil(d/256)] int32: caller-owned, all zero before the first
 *      call; every completed call leaves it zero again.  A call stopped by an
 *      error (MOE_ERR_TIMEOUT, or ids outside [0,E) in the permute) may leave
 *      counts behind: clear it before the next call. */
MOE_API moe_status_t moe_grouped_swiglu_fwd_combine(moe_handle_t h, const moe_shape_t* s,
                                                    const void* x_perm, const int32_t* offsets,
                                                    const int32_t* row_map, const int32_t* row_src,
                                                    const float* topk_w, const void* w_gu,
                                                    const void* w_down, void* au, void* hbuf,
                                                    void* o_perm, const void* shared_out, void* y,
                                                    int32_t* arrivals, moe_stream_t stream);

/* ---- Gather forms: the routed copies of x are never written.  Instead of
 * a materialised x_perm, the two expert GEMMs that read routed rows of x
 * (gate/up forward and its recompute; gate/up weight gradient) gather them
 * from x with TMA tile::gather4 loads through row_src.  The pages describe
 * routing data straight into each expert's input buffer (Olmo-core 3
 * introduction page, section 2, rowwise expert parallelism); this goes one
 * step further on one GPU and skips that buffer.  bf16 only
 * (MOE_ERR_UNSUPPORTED for MXFP8); results equal the x_perm forms bit for
 * bit.
 *
 * moe_route: moe_permute without x_perm.
 * Out: counts, offsets, row_map as moe_permute; row_src [M_cap] int32 =
 *      the token whose copy routed row r holds, T for pad rows and rows past
 *      offsets[E]. */
MOE_API moe_status_t moe_route(moe_handle_t h, const moe_shape_t* s, const int32_t* topk_idx,
                               int32_t* counts, int32_t* offsets, int32_t* row_map,
                               int32_t* row_src, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_grouped_swiglu_fwd with x [T,d] and row_src in place of x_perm (au may
 * be NULL as there).  No workspace.  Same passages as moe_grouped_swiglu_fwd
 * and moe_route (Olmo-core 3 introduction page, section 2). */
MOE_API moe_status_t moe_grouped_swiglu_fwd_gather(moe_handle_t h, const moe_shape_t* s,
                                                   const void* x, const int32_t* row_src,
                                                   const int32_t* offsets, const void* w_gu,
                                                   const void* w_down, void* au, void* hbuf,
                                                   void* o_perm, moe_stream_t stream);

/* moe_grouped_swiglu_recompute with x [T,d] and row_src in place of x_perm.
 * Same passages as moe_grouped_swiglu_recompute (Olmo-core 3 introduction
 * page, section 4) and moe_route (same page, section 2). */
MOE_API moe_status_t moe_grouped_swiglu_recompute_gather(moe_handle_t h, const moe_shape_t* s,
                                                         const void* x, const int32_t* row_src,
                                                         const int32_t* offsets, const void* w_gu,
                                                         void* au, void* hbuf,
                                                         moe_stream_t stream);

/* moe_grouped_swiglu_bwd with x [T,d] and row_src in place of x_perm (only
 * the gate/up weight gradient reads it).  No workspace.  Same passages as
 * moe_grouped_swiglu_bwd and moe_route (Olmo-core 3 introduction page,
 * section 2). */
MOE_API moe_status_t moe_grouped_swiglu_bwd_gather(moe_handle_t h, const moe_shape_t* s,
                                                   const void* do_perm, const void* x,
                                                   const int32_t* row_src, const void* au,
                                                   const void* hbuf, const int32_t* offsets,
                                                   const void* w_gu, const void* w_down, void* dau,
                                                   void* dx_perm, void* dw_gu, void* dw_down,
                                                   moe_stream_t stream);

/* Weighted unpermute-combine ("restore").  The pages: expert outputs are
 * put back in the tokens' original order (discosf.com article on Olmo-core 3,
 * section 2.1); weighting by the gate weights and the slot-order fp32 sum
 * are readings.
 *   y[t] = bf16( sum_j topk_w[t,j] * o_perm[row_map[t,j]] + shared_out[t] ),
 *   fp32 sum in slot order, the shared expert's output (when non-NULL) last.
 * In : o_perm [M_cap,d] bf16, row_map [T,k] int32, topk_w [T,k] fp32,
 *      shared_out [T,d] bf16 or NULL (moe_shared_expert_fwd).
 * Out: y [T,d] bf16. */
MOE_API moe_status_t moe_unpermute_combine(moe_handle_t h, const moe_shape_t* s, const void* o_perm,
                                   const int32_t* row_map, const float* topk_w,
                                   const void* shared_out, void* y, moe_stream_t stream);

/* Backward of the combine: the plain backward of moe_unpermute_combine
 * (restore step: discosf.com article on Olmo-core 3, section 2.1; the
 * pages train the layer but give no backward formula).
 *   do_perm[row_map[t,j]] = bf16(topk_w[t,j] * dy[t]); pad rows = 0;
 *   d_topk_w[t,j] = sum_i dy[t,i] * o_perm[row_map[t,j], i]  (fp32).
 * In : dy [T,d] bf16, o_perm, row_map, topk_w, offsets [E+1], counts [E].
 * Out: do_perm [M_cap,d] bf16, d_topk_w [T,k] fp32. */
MOE_API moe_status_t moe_unpermute_combine_bwd(moe_handle_t h, const moe_shape_t* s, const void* dy,
                                       const void* o_perm, const int32_t* row_map,
                                       const float* topk_w, const int32_t* offsets,
                                       const int32_t* counts, void* do_perm, float* d_topk_w,
                                       moe_stream_t stream);

/* Grouped SwiGLU expert FFN, backward (dgrad and wgrad).  The same grouped,
 * device-scheduled GEMMs as the forward (Olmo-core 3 introduction page,
 * section 2); the formulas are the plain backward of the SwiGLU reading.
 * Per expert e:
 *   dH = do_perm W_down[e]                       (fp32 accumulate)
 *   s = sigmoid(A), A and U read from au
 *   dau[:,0:f] = bf16(dH U s (1 + A (1 - s))),  dau[:,f:2f] = bf16(dH silu(A))
 *   dw_down[e] = bf16(do_perm_e^T h_e)           (sum over e's rows)
 *   dx_perm    = bf16(dau W_gu[e])
 *   dw_gu[e]   = bf16(dau_e^T x_perm_e)
 * Experts with no rows get zero weight gradients.
 * In : do_perm, x_perm, au, hbuf [M_cap,*] bf16, offsets [E+1], w_gu, w_down.
 * Out: dau [M_cap,2f] bf16, dx_perm [M_cap,d] bf16, dw_gu [E,2f,d] bf16,
 *      dw_down [E,d,f] bf16.
 * MXFP8 mode: x_perm, hbuf, w_gu and w_down enter through the column-wise
 * copies the forward left in the workspace (see the MXFP8 note above); the
 * arguments must still be the forward's tensors. */
MOE_API moe_status_t moe_grouped_swiglu_bwd(moe_handle_t h, const moe_shape_t* s, const void* do_perm,
                                    const void* x_perm, const void* au, const void* hbuf,
                                    const int32_t* offsets, const void* w_gu,
                                    const void* w_down, void* dau, void* dx_perm, void* dw_gu,
                                    void* dw_down, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* Backward of the permute: the plain backward of moe_permute's copy
 * (permutation index and restore: discosf.com article on Olmo-core 3,
 * section 2.1), each token's k routed gradients summed back to it.
 *   dx[t] = bf16( sum_j dx_perm[row_map[t,j]] + dx_router[t] + dx_shared[t] ),
 *   fp32 sum, rounded once.  dx_router and dx_shared may be NULL.
 * In : dx_perm [M_cap,d] bf16, row_map [T,k], dx_router [T,d] fp32 or NULL,
 *      dx_shared [T,d] bf16 or NULL (moe_shared_expert_bwd).
 * Out: dx [T,d] bf16. */
MOE_API moe_status_t moe_permute_bwd(moe_handle_t h, const moe_shape_t* s, const void* dx_perm,
                             const int32_t* row_map, const float* dx_router,
                             const void* dx_shared, void* dx, moe_stream_t stream);

/* Backward of the permute with the router's share of the input gradient
 * added in the same pass (the pages name only the steps -- the router:
 * discosf.com article on Olmo-core 3, sections 1.1 and 2.1; the permutation
 * and restore: same article, section 2.1 -- and the formulas are the plain
 * backward of the router and of the permute):
 *   dL[t]  = as in moe_router_topk_bwd, from d_topk_w, probs, topk_idx and
 *            d_probs_aux (nullable)
 *   dx[t]  = bf16( sum_j dx_perm[row_map[t,j]] + dL[t] w_router
 *                  + dx_shared[t] ), fp32, rounded once; dL[t] w_router sums
 *            experts in increasing order; dx_shared may be NULL.
 * Gives the same bits as moe_router_topk_bwd (with dx_router) followed by
 * moe_permute_bwd, but never stores dL w_router.  n_experts <= 64 only
 * (MOE_ERR_UNSUPPORTED otherwise: above 64 experts that product runs on the
 * tensor cores inside moe_router_topk_bwd).
 * In : dx_perm [M_cap,d] bf16, row_map [T,k], d_topk_w [T,k] fp32,
 *      probs [T,E] fp32, topk_idx [T,k], d_probs_aux [E] fp32 or NULL,
 *      w_router [E,d] bf16, dx_shared [T,d] bf16 or NULL.
 * Out: dx [T,d] bf16.  All pointers device, caller-owned; no workspace. */
MOE_API moe_status_t moe_permute_router_bwd(moe_handle_t h, const moe_shape_t* s,
                                            const void* dx_perm, const int32_t* row_map,
                                            const float* d_topk_w, const float* probs,
                                            const int32_t* topk_idx, const float* d_probs_aux,
                                            const void* w_router, const void* dx_shared, void* dx,
                                            moe_stream_t stream);

/* Shared expert (the pages list shared experts among the v2 router's
 * features -- Olmo-core 3 introduction page, section 4 -- without defining
 * them; reading: one more SwiGLU expert every token passes through, its
 * output added to the combine with weight one).  Forward, over all T tokens
 * in place (no permute):
 *   AU_s = bf16([x W_g^T, x W_u^T]),  H_s = bf16(silu(A) U),  O_s = bf16(H_s W_d^T)
 * with W_gu_s [2 f_s, d] (gate rows first) and W_d_s [d, f_s]; s->T and
 * s->d_model as for the layer, s->d_ff = f_s (n_experts, top_k unused).
 * bf16 only.  Feed o_s to moe_unpermute_combine's shared_out.
 * In : x [T,d], w_gu_s [2f_s,d], w_d_s [d,f_s] bf16.
 * Out: au_s [T,2f_s], h_s [T,f_s], o_s [T,d] bf16.  No workspace. */
MOE_API moe_status_t moe_shared_expert_fwd(moe_handle_t h, const moe_shape_t* s, const void* x,
                                           const void* w_gu_s, const void* w_d_s, void* au_s,
                                           void* h_s, void* o_s, moe_stream_t stream);

/* Shared expert backward (shared experts: Olmo-core 3 introduction page,
 * section 4; the plain backward of the reading above), from its output
 * gradient dY (weight one):
 *   dAU_s = SwiGLU backward of dY W_d_s (as moe_grouped_swiglu_bwd),
 *   dW_d_s = bf16(dY^T H_s), dx_s = bf16(dAU_s W_gu_s), dW_gu_s = bf16(dAU_s^T x).
 * Feed dx_s to moe_permute_bwd / moe_permute_router_bwd's dx_shared.
 * In : dy [T,d], x [T,d], au_s, h_s, w_gu_s, w_d_s bf16.
 * Out: dau_s [T,2f_s], dx_s [T,d], dw_gu_s [2f_s,d], dw_d_s [d,f_s] bf16. */
MOE_API moe_status_t moe_shared_expert_bwd(moe_handle_t h, const moe_shape_t* s, const void* dy,
                                           const void* x, const void* au_s, const void* h_s,
                                           const void* w_gu_s, const void* w_d_s, void* dau_s,
                                           void* dx_s, void* dw_gu_s, void* dw_d_s,
                                           moe_stream_t stream);

/* Router backward (through the selected probabilities; top-k itself has no
 * gradient).  The plain backward of the router of moe_router_topk
 * (discosf.com article on Olmo-core 3, sections 1.1 and 2.1):
 *   g = d_topk_w, or with MOE_FLAG_RENORM g_j = (dw_j - sum_i dw_i w_i) / S
 *   dp[t, topk_idx[t,j]] = g[t,j], 0 elsewhere
 *   dp[t, e] += d_probs_aux[e] for every t, when d_probs_aux is non-NULL
 *               (the load-balancing loss: moe_router_aux_loss)
 *   dL = probs * (dp - sum_e probs dp)
 *   dx_router = dL w_router            [T,d] fp32 (fed to moe_permute_bwd),
 *                                      written when non-NULL
 *   dw_router = bf16(dL^T x)           [E,d]
 *   dbias     = sum_t dL               [E] fp32, written when non-NULL
 * With dx_router NULL the call leaves the input gradient to
 * moe_permute_router_bwd (n_experts <= 64), which forms dL w_router on the
 * fly instead of passing [T,d] fp32 through device memory.
 * In : d_topk_w [T,k] fp32, probs [T,E] fp32, topk_idx [T,k],
 *      d_probs_aux [E] fp32 or NULL, x [T,d] bf16, w_router [E,d] bf16. */
MOE_API moe_status_t moe_router_topk_bwd(moe_handle_t h, const moe_shape_t* s, const float* d_topk_w,
                                 const float* probs, const int32_t* topk_idx,
                                 const float* d_probs_aux, const void* x,
                                 const void* w_router, float* dx_router, void* dw_router,
                                 float* dbias, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router load statistics of one batch, for the load-balancing loss.  The
 * pages call for a load-balancing auxiliary loss (discosf.com article on
 * Olmo-core 3, sections 2.2 and 4.3) and for balancing over the global
 * batch (Olmo-core 3 introduction page, section 4); they give no formula,
 * and the reading is the Switch-Transformer loss over the k routed slots.
 *   stats[e]     = counts[e]            routed (token, slot) pairs, as fp32
 *   stats[E + e] = sum_t probs[t, e]    router probability mass
 * accumulate != 0 adds into stats instead of overwriting it, so that the
 * sums of several micro-batches (and, summed over ranks by the caller, of
 * several GPUs) make the global batch's statistics.  Sums in a fixed order.
 * In : probs [T,E] fp32, counts [E] int32 (from moe_permute).
 * Out: stats [2E] fp32.  Uses the workspace. */
MOE_API moe_status_t moe_router_load_stats(moe_handle_t h, const moe_shape_t* s, const float* probs,
                                           const int32_t* counts, int accumulate, float* stats,
                                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Load-balancing loss (discosf.com article on Olmo-core 3, sections 2.2 and
 * 4.3; the Switch-Transformer reading of moe_router_load_stats) of
 * (possibly summed) statistics over n_tokens tokens:
 *   f_e = stats[e] / (n_tokens k),  P_e = stats[E+e] / n_tokens
 *   loss = alpha E sum_e f_e P_e        (alpha at balance, alpha E at collapse)
 *   d_probs_aux[e] = alpha E f_e / n_tokens = d loss / d probs[t, e] for every
 *                    token (f_e is piecewise constant in the logits)
 * Feed d_probs_aux to moe_router_topk_bwd / moe_permute_router_bwd.
 * In : stats [2E] fp32, n_tokens >= 1, alpha >= 0.
 * Out: loss [1] fp32 and d_probs_aux [E] fp32 (either may be NULL, not both). */
MOE_API moe_status_t moe_router_aux_loss(moe_handle_t h, const moe_shape_t* s, const float* stats,
                                         int64_t n_tokens, float alpha, float* loss,
                                         float* d_probs_aux, moe_stream_t stream);

/* MXFP8 quantisation of a bf16 matrix [rows, cols] (OCP MX v1.0 reading of
 * the pages' "MXFP8", offered for selected operations, its gain coming from
 * the FFN and expert data movement: Olmo-core 3 introduction page, section 3
 * "MXFP8"): blocks of 32 consecutive elements, along each row
 * (axis = 1) or down each column (axis = 0); per block the E8M0 scale code
 * is clamp(floor(log2(amax)) - 8, -127, 127) + 127 (code 0 for an all-zero
 * block) and each element is the E4M3 code of round-to-nearest-even
 * (v / 2^(code-127)), saturated to +-448.
 * In : in [rows, cols] bf16; rows (axis 0) or cols (axis 1) multiple of 32.
 * Out: q [rows, cols] uint8 (E4M3 codes), scales uint8 (E8M0 codes),
 *      [rows, cols/32] for axis 1, [rows/32, cols] for axis 0. */
MOE_API moe_status_t moe_mxfp8_quantize(moe_handle_t h, const void* in, int64_t rows, int64_t cols,
                                int axis, uint8_t* q, uint8_t* scales, moe_stream_t stream);

/* Both MXFP8 quantisations of a bf16 matrix from one read, written in the
 * layout the MXFP8 expert GEMMs take: the step the expert calls run on each
 * operand (Olmo-core 3 introduction page, section 3 "MXFP8"; the same OCP
 * MX v1.0 per-block rule as moe_mxfp8_quantize):
 *   row-wise   : blocks of 32 consecutive elements along each row;
 *   column-wise: blocks of 32 consecutive rows down each column, inside each
 *                group of rows_per_group rows (the token-axis blocks of one
 *                expert segment never reach into the next).
 * Scale codes are in the tensor cores' 512-byte scale-atom order: for a
 * matrix with MN index r and 32-element contraction block b (n_b4 = number
 * of contraction blocks / 4), the code sits at byte
 *   ((r / 128) * n_b4 + b / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + b % 4.
 * Row-wise: r = row, b = column / 32, n_b4 = cols / 128.  Column-wise, per
 * group g (its codes start at byte g * cols * rows_per_group / 32): r =
 * column, b = (row within the group) / 32, n_b4 = rows_per_group / 128.
 * In : in [rows, cols] bf16, 16-byte aligned; rows a multiple of
 *      rows_per_group, rows_per_group and cols multiples of 128.
 * Out: q_row, q_col [rows, cols] uint8 E4M3 codes (row-major, 16-byte
 *      aligned); s_row, s_col rows * cols / 32 bytes each (caller-owned).
 * One launch; MOE_ERR_INVALID_ARG for shapes or alignments outside these. */
MOE_API moe_status_t moe_mxfp8_quantize_gemm(moe_handle_t h, const void* in, int64_t rows,
                                             int64_t cols, int64_t rows_per_group, uint8_t* q_row,
                                             uint8_t* s_row, uint8_t* q_col, uint8_t* s_col,
                                             moe_stream_t stream);

/* Waits for the device, then returns the status word recorded by kernels
 * (MOE_OK if none) in *device_status and clears it.  The only call that
 * synchronises; not meant for use inside a step.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_get_status(moe_handle_t h, int* device_status);

/* Number of kernels this handle has launched since it was created (a host
 * counter: it costs nothing on the device and does not synchronise).
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_get_launch_count(moe_handle_t h, uint64_t* launches);

/* Time limit, in nanoseconds, of the bounded waits in the main loops of the
 * grouped-GEMM kernels this handle launches from now on (default 2 s).  A
 * wait that runs out records MOE_ERR_TIMEOUT in the status word; the kernel
 * then waits for its own copies and MMAs in flight (those drain waits keep
 * the 2 s bound), frees its tensor memory and returns, so the context stays
 * usable.  ns = 0 makes every such wait give up unless its first test finds
 * it complete: a test uses that to check the timeout path without faulting
 * the GPU.  Host-only; launches nothing.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API moe_status_t moe_set_wait_limit(moe_handle_t h, uint64_t ns);

/* Static description of a status code.
 * (Library plumbing: the pages have no counterpart.) */
MOE_API const char* moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
