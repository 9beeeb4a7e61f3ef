// The fixed scratch array behind any4_matmul_static_scratch.
//
// The prefill kernel's stream-K schedule needs device scratch (one fp32
// partial tile per block plus one flag word per block).  any4_matmul takes it
// from the caller; this file holds a file-scope array that serves instead for
// callers that cannot allocate at the call site: a step that must not call
// cudaMalloc/cudaFree (cudaFree synchronises the whole device, stalling every
// stream), or a plain C caller of the ABI that has no device allocator of its
// own.  Its size is fixed at build time (ANY4_STATIC_SCRATCH_BYTES); one copy
// exists per device (reserved when the library's module is loaded on that
// device, whether or not the entry point is ever called), so calls that
// overlap on the GPU share it and race.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kMaxScratchDevices = 64;

__device__ __align__(256) uint8_t g_static_scratch[ANY4_STATIC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Driver entry points for the identity of the current context (the array's
// address belongs to the context that loaded the module).
struct CtxFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

CtxFns ctx_fns() {
  static CtxFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

std::mutex g_scratch_mu;
struct ScratchEntry {
  unsigned long long ctx_id = 0;  // context the address was resolved in
  void* addr = nullptr;
};
ScratchEntry g_scratch[kMaxScratchDevices];

}  // namespace

// Device address of the array on `device`, which must be the current device.
// Resolved with cudaGetSymbolAddress on the first call on a device, and again
// whenever the device's current context has changed since (a device reset or
// a released and re-created primary context reloads the module, and the
// array may then sit at another address); otherwise the cached address.
any4_status static_scratch(int device, void** ptr) {
  if (device < 0 || device >= kMaxScratchDevices) return ANY4_ERR_CUDA;
  const CtxFns fns = ctx_fns();
  if (!fns.get_current || !fns.get_id) return ANY4_ERR_CUDA;
  // identity of the current context; 0 when the runtime has none yet
  auto current_id = [&fns](unsigned long long* id) {
    CUcontext ctx = nullptr;
    *id = 0;
    return fns.get_current(&ctx) == CUDA_SUCCESS &&
           (ctx == nullptr || fns.get_id(ctx, id) == CUDA_SUCCESS);
  };
  unsigned long long id = 0;
  if (!current_id(&id)) return ANY4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& e = g_scratch[device];
  if (id == 0 || e.addr == nullptr || e.ctx_id != id) {
    // cudaGetSymbolAddress also creates the device's primary context (and
    // loads the module) when there is none yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();  // leave no error behind for the caller's next CUDA call
      return ANY4_ERR_CUDA;
    }
    if (!current_id(&id) || id == 0) return ANY4_ERR_CUDA;
    e.addr = p;
    e.ctx_id = id;
  }
  *ptr = e.addr;
  return ANY4_OK;
}

}  // namespace any4
