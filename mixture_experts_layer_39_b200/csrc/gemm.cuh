// Host launchers of the tcgen05 grouped GEMMs (implemented in gemm.cu).
#pragma once

#include "common.cuh"

namespace moe {

struct GemmCtx {
  int num_sms;
  DeviceCtl* ctl;
  // M-grouped bf16 GEMMs run 256-row tiles on CTA pairs (worth it when the
  // experts' row segments are long compared with a tile)
  bool pair_m = false;
  // time limit of the GEMMs' main-loop waits (the handle's; 0 = give up
  // unless already complete)
  uint64_t wait_ns = 2000000000ull;
  // launches beyond the fixed count an entry point books (a weight gradient
  // whose last wave runs as a second launch) are added here
  uint64_t* extra_launches = nullptr;
};

// An MXFP8 operand: E4M3 codes and E8M0 scales ([MN index][K/32] bytes).
struct MxOperand {
  const uint8_t* q;
  const uint8_t* s;
};

moe_status_t gemm_fwd_gate_up(const GemmCtx& c, const void* x_perm, const int32_t* offsets,
                              const void* w_gu, void* au, void* h, int E, int d, int f,
                              int64_t m_cap, cudaStream_t st);
moe_status_t gemm_fwd_down(const GemmCtx& c, const void* h, const int32_t* offsets,
                           const void* w_d, void* o_perm, int E, int d, int f, int64_t m_cap,
                           cudaStream_t st);
// The down projection with the unpermute-combine fused into its epilogue:
// also y[t] = bf16(sum_j topk_w[t,j] O[row_map[t,j]] (+ shared[t])).
struct CombineArgs {
  const int32_t* row_src;  // [m_cap] token of each routed row, T on pad rows
  const int32_t* row_map;  // [T, k]
  const float* topk_w;     // [T, k]
  const void* shared;      // [T, d] bf16 or nullptr
  void* y;                 // [T, d] bf16
  int32_t* arrivals;       // [T, ceil(d / 256)], zero on entry and on return
  int T, k;
};
moe_status_t gemm_fwd_down_combine(const GemmCtx& c, const void* h, const int32_t* offsets,
                                   const void* w_d, void* o_perm, int E, int d, int f,
                                   int64_t m_cap, const CombineArgs& cb, cudaStream_t st);
moe_status_t gemm_dgrad_down_swiglu(const GemmCtx& c, const void* do_perm, const int32_t* offsets,
                                    const void* w_d, const void* au, void* dau, int E, int d,
                                    int f, int64_t m_cap, cudaStream_t st);
moe_status_t gemm_dgrad_gate_up(const GemmCtx& c, const void* dau, const int32_t* offsets,
                                const void* w_gu, void* dx_perm, int E, int d, int f,
                                int64_t m_cap, cudaStream_t st);
moe_status_t gemm_wgrad_down(const GemmCtx& c, const void* do_perm, const void* h,
                             const int32_t* offsets, void* dw_d, int E, int d, int f,
                             int64_t m_cap, cudaStream_t st);
moe_status_t gemm_wgrad_gate_up(const GemmCtx& c, const void* dau, const void* x_perm,
                                const int32_t* offsets, void* dw_gu, int E, int d, int f,
                                int64_t m_cap, cudaStream_t st);
// Gather forms of the two GEMMs that read routed copies of x: row r of the
// routed operand is x[row_src[r]] (T rows; row T and beyond read as zeros).
moe_status_t gemm_fwd_gate_up_gather(const GemmCtx& c, const void* x, int T,
                                     const int32_t* row_src, const int32_t* offsets,
                                     const void* w_gu, void* au, void* h, int E, int d, int f,
                                     int64_t m_cap, cudaStream_t st);
moe_status_t gemm_wgrad_gate_up_gather(const GemmCtx& c, const void* dau, const void* x, int T,
                                       const int32_t* row_src, const int32_t* offsets,
                                       void* dw_gu, int E, int d, int f, int64_t m_cap,
                                       cudaStream_t st);
// Router on the tensor cores (any E above 64): the logits buffer and the
// bf16 dL buffer have row stride ld = E rounded up to a multiple of 128.
moe_status_t gemm_router_logits(const GemmCtx& c, const void* x, const void* w_r, float* logits,
                                int T, int d, int E, int ld, cudaStream_t st);
moe_status_t gemm_router_dx(const GemmCtx& c, const void* dl_bf16, int ld, const void* w_r,
                            float* dx_router, int T, int d, int E, cudaStream_t st);
int router_dw_groups(int num_sms, int T, int d, int E, int* group_len);
moe_status_t gemm_router_dw_partial(const GemmCtx& c, const void* dl_bf16, int ld, const void* x,
                                    float* partial, int T, int d, int E, int n_groups,
                                    int group_len, cudaStream_t st);

moe_status_t gemm_mx_fwd_gate_up(const GemmCtx& c, const MxOperand& x, const int32_t* offsets,
                                 const MxOperand& w_gu, void* au, void* h, int E, int d, int f,
                                 int64_t m_cap, cudaStream_t st);
moe_status_t gemm_mx_fwd_down(const GemmCtx& c, const MxOperand& h, const int32_t* offsets,
                              const MxOperand& w_d, void* o_perm, int E, int d, int f,
                              int64_t m_cap, cudaStream_t st);
moe_status_t gemm_mx_dgrad_down_swiglu(const GemmCtx& c, const MxOperand& dO, const int32_t* offsets,
                                       const MxOperand& w_d_col, const void* au, void* dau, int E,
                                       int d, int f, int64_t m_cap, cudaStream_t st);
moe_status_t gemm_mx_dgrad_gate_up(const GemmCtx& c, const MxOperand& dau, const int32_t* offsets,
                                   const MxOperand& w_gu_col, void* dx_perm, int E, int d, int f,
                                   int64_t m_cap, cudaStream_t st);
moe_status_t gemm_mx_wgrad(const GemmCtx& c, const MxOperand& a_col, int M, const MxOperand& b_col,
                           int N, const int32_t* offsets, void* dw, int E, int64_t m_cap,
                           cudaStream_t st);

}  // namespace moe
