// moe_route_noalloc: moe_route for callers that cannot allocate device
// memory. moe_route needs a caller-allocated workspace for its per-block
// expert counts and bases; some callers have no way to provide one -- code
// that runs inside another library or runtime that owns all device memory
// and hands out none, hosts that plan every byte ahead and forbid new
// allocations, or paths where a cudaMalloc would implicitly synchronise the
// device. This entry point keeps that scratch in a fixed array compiled into
// the library instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its own copy (MOE_ROUTE_NOALLOC_MAX_SLOTS * 8 bytes, 2 MiB)
// until the process exits. Host code cannot use the variable's name as a
// device address, so the first call on each device looks the address up
// with cudaGetSymbolAddress (with that device current) and caches it with the
// id of the device's current context; make that first call before any stream
// capture. A later call in another context (after cudaDeviceReset the module
// is loaded again, at a new address) looks it up again. All calls on a device share the
// one array, so calls that overlap on the GPU (different streams, or
// concurrent host threads) race and must be serialised by the caller. Every
// entry the kernels read is written earlier in the same call, so nothing has
// to be cleared between calls.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// [0, MAX_SLOTS): per-block expert counts; [MAX_SLOTS, 2*MAX_SLOTS): bases.
static __device__ __align__(256) int32_t g_route_scratch[2 * MOE_ROUTE_NOALLOC_MAX_SLOTS];

std::mutex g_mu;
int32_t* g_scratch_of_device[kMaxDevices] = {};
unsigned long long g_ctx_of_device[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's copy of the array: looked up on the first
// call on the device and again whenever the device's context has changed.
int scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return moe::report_error(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return moe::report_error(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: device index out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  // makes the device's primary context current if no call has yet
  void* p = nullptr;
  if (!g_scratch_of_device[dev]) {
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p)
      return moe::report_error(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetSymbolAddress failed");
    g_scratch_of_device[dev] = static_cast<int32_t*>(p);
    g_ctx_of_device[dev] = current_context_id();
  } else {
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || ctx != g_ctx_of_device[dev]) {
      e = cudaGetSymbolAddress(&p, g_route_scratch);
      if (e != cudaSuccess || !p)
        return moe::report_error(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetSymbolAddress failed");
      g_scratch_of_device[dev] = static_cast<int32_t*>(p);
      g_ctx_of_device[dev] = ctx;
    }
  }
  *out = g_scratch_of_device[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_route_noalloc(const float* logits, int64_t T, int E, int k, int ep_groups,
                                 int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                                 int64_t* expert_offsets, int32_t* group_counts,
                                 int64_t* group_offsets, int32_t* row_of_pair,
                                 int32_t* pair_of_row, unsigned int* err_flags,
                                 cudaStream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E || ep_groups < 1)
    return moe::report_error(MOE_ERR_INVALID_ARG, "moe_route_noalloc: invalid T, E, k or ep_groups");
  if (E > MOE_MAX_EXPERTS || k > 32 || E % ep_groups != 0 || T * k >= (int64_t(1) << 31))
    return moe::report_error(MOE_ERR_UNSUPPORTED,
                             "moe_route_noalloc: E, k or ep_groups outside the supported set");
  const int64_t nb = (T + moe::kRouteTokensPerBlock - 1) / moe::kRouteTokensPerBlock;
  if (nb * E > MOE_ROUTE_NOALLOC_MAX_SLOTS)
    return moe::report_error(MOE_ERR_UNSUPPORTED,
                             "moe_route_noalloc: ceil(T/256)*E exceeds MOE_ROUTE_NOALLOC_MAX_SLOTS; "
                             "use moe_route with a workspace");
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w || !expert_counts || !expert_offsets || !group_counts ||
      !group_offsets || !row_of_pair || !pair_of_row)
    return moe::report_error(MOE_ERR_INVALID_ARG, "moe_route_noalloc: null pointer");
  int32_t* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  if (E > 768) {
    if (moe::route_set_smem_limits() != cudaSuccess)
      return moe::report_error(MOE_ERR_CUDA, "moe_route_noalloc: shared-memory limit");
  }
  cudaError_t e = moe::launch_route(logits, T, E, k, ep_groups, topk_idx, topk_w, expert_counts,
                                    expert_offsets, group_counts, group_offsets, row_of_pair,
                                    pair_of_row, scratch, scratch + MOE_ROUTE_NOALLOC_MAX_SLOTS,
                                    err_flags, stream);
  if (e != cudaSuccess) return moe::report_error(MOE_ERR_CUDA, cudaGetErrorString(e));
  moe::count_launches(3);
  return MOE_OK;
}
