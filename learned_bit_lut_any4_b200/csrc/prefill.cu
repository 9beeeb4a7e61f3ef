// Prefill-path any4 matmul (large M) -- tcgen05 tensor-core kernel goes here.
#include "common.cuh"

namespace any4 {

size_t prefill_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G) {
  (void)M; (void)N; (void)K; (void)G;
  return 0;
}

any4_status launch_prefill(const uint16_t*, const uint8_t*, const uint16_t*, int64_t,
                           const uint16_t*, const uint16_t*, uint16_t*, int64_t, int64_t,
                           int64_t, int64_t, void*, size_t, int32_t*, cudaStream_t,
                           const DeviceInfo&) {
  return ANY4_ERR_UNSUPPORTED;
}

}  // namespace any4
