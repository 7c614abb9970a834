// Host-side state that belongs to a CUDA context rather than to the process:
// the current context's id, and kernel attributes set once per context.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

namespace moe {

// Id of the calling thread's current CUDA context (unique per context
// created in this process), or 0 when there is none or it cannot be read.
inline unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Raises `kern`'s dynamic shared-memory limit to at least `bytes` in the
// current context.  The attribute lives in the context (one per device, and
// a device reset starts a new one), so the limits already set are kept per
// context and kernel; without a readable context id the call is always made.
inline bool set_max_dyn_smem(const void* kern, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<unsigned long long, const void*>, size_t> done;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  size_t* have = ctx != 0 ? &done[{ctx, kern}] : nullptr;
  if (have != nullptr && bytes <= *have) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  if (have != nullptr) *have = bytes;
  return true;
}

}  // namespace moe
