// moe_dispatch_noalloc: the dispatch with its scratch in library-owned
// device memory instead of a caller workspace.
//
// Some callers cannot allocate device memory at all: a host framework that
// owns every byte of device memory and forbids allocation outside its own
// pool, or a latency-critical path where cudaMalloc's implicit device
// synchronisation is not acceptable. They can still provide the inputs and
// outputs, but not the workspace moe_dispatch needs for its per-block
// expert histograms. For them this file keeps that scratch in a fixed,
// file-scope __device__ array: every GPU that loads the library holds
// MOE_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// In host code `g_dispatch_scratch` names a host-side stand-in, not a
// device address, so the kernels are never given that name: on the first
// call on a device (with that device current) the address is looked up
// once with cudaGetSymbolAddress and cached for that device's current CUDA
// context. That first call should therefore be made before any stream
// capture. A device reset (cudaDeviceReset) ends the context and unloads
// the module; the next call, made in the new context, sees the context
// change and looks the address up again.
//
// Every call shares the one array, which keeps the last call's contents.
// The dispatch kernels write every histogram entry they later read, so
// nothing has to be cleared between calls; calls that overlap on the GPU
// (different streams, or different host threads on one device) race on the
// array and must be serialised by the caller.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_dispatch_scratch[MOE_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, looked up once (null if unavailable).
CtxGetCurrentFn ctx_get_current_fn() {
  static const CtxGetCurrentFn fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(ptr);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up
// once per device and context.
int scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return MOE_ERR_CUDA;
  // Null if the runtime has not yet made its context current on this thread.
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev] || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
    void *p = nullptr;
    // The lookup makes the device's primary context current if it was not.
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

bool dispatch_fits_noalloc_scratch(int64_t n_assign, int n_heavy) {
  return dispatch_workspace_bytes(n_assign, n_heavy) <= (size_t)MOE_NOALLOC_SCRATCH_BYTES;
}

int launch_dispatch_noalloc(const DispatchArgs &a, cudaStream_t stream) {
  if (!dispatch_fits_noalloc_scratch(a.n_assign, a.n_heavy)) return MOE_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  int st = scratch_on_current_device(&scratch);
  if (st != MOE_OK) return st;
  return launch_dispatch(a, scratch, stream);
}

}  // namespace moe
