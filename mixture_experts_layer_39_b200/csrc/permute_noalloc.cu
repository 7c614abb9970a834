// moe_permute_noalloc: the routing metadata + permute of moe_permute, for
// callers that cannot hand the library any scratch memory.
//
// moe_permute needs a small scratch buffer (per expert, a count for every
// 64 and every 512 tokens of the routing ids), which it takes from the caller's
// workspace.  Some callers have no way to provide one: code embedded in a
// host program that owns all device memory through its own pool and gives
// plug-ins no allocation hook, or code on a latency-critical path that must
// not call cudaMalloc (an allocation can stall until the device is idle and
// can fail when memory is tight).  This variant keeps its scratch in a
// fixed array compiled into the library instead.
//
// The array: MOE_NOALLOC_SCRATCH_INTS int32 values (1 MiB, the size the
// header states), declared below at file scope in device memory.  Every GPU
// that loads the library holds one copy of it until the process exits.  Host
// code cannot use the array's name as a device address (on the host it names
// a placeholder), so the first call on each device, with that device
// current, looks the address up with cudaGetSymbolAddress and keeps it;
// later calls on that device reuse it.  Make that first call before starting
// any stream capture.  The address is kept together with the id of the CUDA
// context it was looked up in: a device reset destroys that context and the
// module is loaded again elsewhere, so a call that finds another context
// looks the address up again (before any capture, like the first call).
//
// Sharing: every call on a device uses the same array and leaves its
// contents behind.  Nothing in it has to start at zero (each entry a call
// reads is written earlier in that same call), but two calls whose work
// overlaps on the GPU (different streams with no ordering between them, or
// several host threads) race on the array and corrupt each other's results.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "context.cuh"
#include "host_ctx.cuh"
#include "kernels.cuh"

namespace {

constexpr int64_t kNoallocScratchInts = MOE_NOALLOC_SCRATCH_INTS;  // 262144 int32 = 1 MiB
static_assert(kNoallocScratchInts == (1 << 18), "the header documents a 1 MiB array");

static __device__ __align__(256) int32_t g_permute_scratch[kNoallocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
int32_t* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context id the address belongs to

// Device address of the array on `device`, which must be the current device.
moe_status_t scratch_on_device(int device, int32_t** out) {
  if (device < 0 || device >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = moe::current_context_id();
  if (g_scratch_addr[device] == nullptr || ctx == 0 || ctx != g_scratch_ctx[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[device] = static_cast<int32_t*>(p);
    // the lookup made the device's primary context current if it was not
    g_scratch_ctx[device] = ctx != 0 ? ctx : moe::current_context_id();
  }
  *out = g_scratch_addr[device];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(moe_handle_t h, const moe_shape_t* s, const void* x,
                                            const int32_t* topk_idx, int32_t* counts,
                                            int32_t* offsets, int32_t* row_map, void* x_perm,
                                            moe_stream_t stream) {
  MOE_TRACE();
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_status_t shape_ok = moe::check_shape(s);
  if (shape_ok != MOE_OK) return shape_ok;
  if (x == nullptr || topk_idx == nullptr || counts == nullptr || offsets == nullptr ||
      row_map == nullptr || x_perm == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!moe::aligned(x, 16) || !moe::aligned(x_perm, 16)) return MOE_ERR_INVALID_ARG;
  const int T = s->T, d = s->d_model, E = s->n_experts, k = s->top_k;
  if (moe::route_scratch_ints(T, E) > kNoallocScratchInts) return MOE_ERR_WORKSPACE;  // > 1 MiB

  moe::DeviceGuard guard(h->device);
  if (!guard.ok) return MOE_ERR_CUDA;
  int32_t* sub = nullptr;
  const moe_status_t found = scratch_on_device(h->device, &sub);
  if (found != MOE_OK) return found;

  auto st = static_cast<cudaStream_t>(stream);
  h->launches += 2;
  if (moe::launch_route_count(topk_idx, T, k, E, moe::seg_align(s), sub, counts, offsets, h->ctl,
                              st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_route_rank_scatter(topk_idx, static_cast<const __nv_bfloat16*>(x), T, k, E, sub,
                                     offsets, counts, d, row_map,
                                     static_cast<__nv_bfloat16*>(x_perm), nullptr, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
