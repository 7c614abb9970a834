// The library handle behind moe_handle_t (private to libmoe.so).
#pragma once

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

struct moe_context {
  int device;
  int num_sms;
  moe::DeviceCtl* ctl;    // device status word
  uint64_t launches = 0;  // kernels launched through this handle
  uint64_t wait_ns = 2000000000ull;  // GEMM main-loop wait limit (moe_set_wait_limit)
};

namespace moe {

// One NVTX range per entry point that touches the device, named for the
// entry point, pushed on entry and popped on every return: a timeline tool
// (Nsight Systems, or any NVTX client) then shows each call's host span
// around the kernels it launched.  With no tool attached the header-only
// NVTX 3 calls go to empty functions.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

#define MOE_TRACE() const ::moe::TraceRange _moe_trace(__func__)

// Makes the handle's device current for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    if (prev >= 0) {
      int cur = -1;
      if (cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
  }
};

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int seg_align(const moe_shape_t* s) {
  return s->dtype == MOE_DTYPE_MXFP8 ? kSegAlignMx : kSegAlign;
}

// Rows of every buffer in the routed-row space.
inline int64_t max_rows(const moe_shape_t* s) {
  const int64_t a = seg_align(s);
  const int64_t r = static_cast<int64_t>(s->T) * s->top_k + (a - 1) * s->n_experts;
  return s->dtype == MOE_DTYPE_MXFP8 ? (r + a - 1) / a * a : r;
}

// Shape checks shared by every entry point (see include/moe.h, "Supported shapes").
inline moe_status_t check_shape(const moe_shape_t* s) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->T < 1 || s->d_model < 1 || s->d_ff < 1 || s->n_experts < 1 || s->top_k < 1)
    return MOE_ERR_INVALID_ARG;
  if (s->top_k > s->n_experts) return MOE_ERR_INVALID_ARG;
  if (s->top_k > 8 || s->n_experts > 1024) return MOE_ERR_UNSUPPORTED;
  if (s->d_model % 128 != 0 || s->d_ff % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (s->dtype != MOE_DTYPE_BF16 && s->dtype != MOE_DTYPE_MXFP8) return MOE_ERR_INVALID_ARG;
  if (max_rows(s) >= (1ll << 31) - 256) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace moe
