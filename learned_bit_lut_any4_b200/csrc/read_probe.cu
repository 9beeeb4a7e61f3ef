// any4_read_probe: a read-only stream over a device buffer (sm_100a)
//
//   out = XOR of every 32-bit word of buf[0 .. bytes)
//
// The decode matmuls read about 250 bytes for every byte they write, so the
// ceiling that bounds them is the rate at which HBM delivers reads alone, which
// a copy (half reads, half writes) does not measure.  This kernel is that
// measurement: the smallest computation that needs every byte of the buffer,
// with a result that can be checked.
//
// Grid-stride 16-byte loads that skip L1, four independent loads in flight per
// thread and a full-occupancy grid (8 blocks of 256 threads per SM), so that
// roughly 128 KiB per SM are requested at any time: enough to cover the
// latency of a loaded HBM.  Each block folds its words with XOR (order does not
// matter for XOR, so the result is deterministic) and adds it to `out` with
// one atomic XOR.
#include "common.cuh"

namespace any4 {
namespace {

constexpr int kRpThreads = 256;
constexpr int kRpBlocksPerSm = 8;
constexpr int kRpUnroll = 4;

__device__ __forceinline__ uint4 ldg_stream_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t fold(uint4 v) { return v.x ^ v.y ^ v.z ^ v.w; }

__global__ void __launch_bounds__(kRpThreads) read_probe_kernel(const uint4* __restrict__ buf,
                                                                int64_t n16,
                                                                uint32_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * kRpThreads;
  int64_t i = (int64_t)blockIdx.x * kRpThreads + threadIdx.x;
  uint32_t acc = 0u;
  for (; i + (kRpUnroll - 1) * stride < n16; i += kRpUnroll * stride) {
    uint4 v[kRpUnroll];
#pragma unroll
    for (int u = 0; u < kRpUnroll; ++u) v[u] = ldg_stream_v4(buf + i + u * stride);
#pragma unroll
    for (int u = 0; u < kRpUnroll; ++u) acc ^= fold(v[u]);
  }
  for (; i < n16; i += stride) acc ^= fold(ldg_stream_v4(buf + i));

  acc = __reduce_xor_sync(0xffffffffu, acc);
  __shared__ uint32_t s_warp[kRpThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_warp[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t blk = 0u;
#pragma unroll
    for (int w = 0; w < kRpThreads / 32; ++w) blk ^= s_warp[w];
    atomicXor(out, blk);
  }
}

}  // namespace

any4_status launch_read_probe(const void* buf, int64_t bytes, uint32_t* out, cudaStream_t stream,
                              const DeviceInfo& dev) {
  if (cudaMemsetAsync(out, 0, sizeof(uint32_t), stream) != cudaSuccess) return ANY4_ERR_CUDA;
  const int64_t n16 = bytes / 16;
  if (n16 == 0) return ANY4_OK;
  const int64_t full = (int64_t)dev.sm_count * kRpBlocksPerSm;
  const int64_t need = (n16 + kRpThreads - 1) / kRpThreads;
  const int grid = (int)(need < full ? need : full);
  read_probe_kernel<<<grid, kRpThreads, 0, stream>>>(static_cast<const uint4*>(buf), n16, out);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
