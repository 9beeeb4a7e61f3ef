// The fixed scratch array behind any4_matmul_static_scratch.
//
// The prefill kernel's stream-K schedule needs device scratch (one fp32
// partial tile per block plus one flag word per block).  any4_matmul takes it
// from the caller; this file holds a file-scope array that serves instead for
// callers that cannot allocate at the call site: a step that must not call
// cudaMalloc/cudaFree (cudaFree synchronises the whole device, stalling every
// stream), or a plain C caller of the ABI that has no device allocator of its
// own.  Its size is fixed at build time (ANY4_STATIC_SCRATCH_BYTES); one copy
// exists per device, so calls that overlap on the GPU share it and race.
#include <mutex>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kMaxScratchDevices = 64;

__device__ __align__(256) uint8_t g_static_scratch[ANY4_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

}  // namespace

// Device address of the array on `device`, which must be the current device.
// Resolved once per device with cudaGetSymbolAddress (the first call on a
// device does this set-up); later calls return the cached address.
any4_status static_scratch(int device, void** ptr) {
  if (device < 0 || device >= kMaxScratchDevices) return ANY4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();  // leave no error behind for the caller's next CUDA call
      return ANY4_ERR_CUDA;
    }
    g_scratch_addr[device] = p;
  }
  *ptr = g_scratch_addr[device];
  return ANY4_OK;
}

}  // namespace any4
