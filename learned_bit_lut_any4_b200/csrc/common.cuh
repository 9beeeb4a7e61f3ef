// Shared device helpers of libany4 (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "any4.h"

namespace any4 {

constexpr unsigned kFullMask = 0xffffffffu;

// bf16 bit pattern -> fp32 (exact: the pattern is the high half of the fp32).
__device__ __forceinline__ float bf16_lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2 with round-to-nearest-even (cvt.rn.bf16x2.f32);
// `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float v) {
  return (uint16_t)(pack_bf16x2_rn(v, 0.0f) & 0xffffu);
}

// Warp shuffle by index; only bits 4..0 of `src` select the lane.  With a
// 16-entry table held twice across the warp (lane l holds entry l & 15), the
// low nibble of `src` is the table index and the bits above it are ignored,
// so a code word shifted right needs no masking.
__device__ __forceinline__ float shfl_idx(float v, uint32_t src) {
  float r;
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=f"(r) : "f"(v), "r"(src));
  return r;
}

// Read-only 16-byte load through the non-coherent path.
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) {
  uint16_t r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ void stg_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
               :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void report_status(int32_t* dev_status, int32_t code) {
  if (dev_status != nullptr) atomicOr(dev_status, code);
}

}  // namespace any4

// Host-side: launch helpers shared by the translation units.
namespace any4 {
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0;
  int cc_minor = 0;
  size_t smem_optin = 0;
};
// Cached properties of the current device (one lookup per device).
any4_status current_device(DeviceInfo* info);

any4_status launch_pack(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                        int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev);
any4_status launch_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                           const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                           int64_t N, int64_t K, int64_t G, cudaStream_t stream,
                           const DeviceInfo& dev);
any4_status launch_decode(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t G, bool overlap,
                          int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev);
bool decode_tma_supported(int64_t M, int64_t N, int64_t K, int64_t G);
any4_status launch_decode_tma(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                              int64_t lut_row_stride, const uint16_t* scale,
                              const uint16_t* offset, uint16_t* y, int64_t N, int64_t K,
                              int64_t G, bool overlap, int32_t* dev_status, cudaStream_t stream,
                              const DeviceInfo& dev);
size_t prefill_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G);
// Device address of the fixed scratch array of any4_matmul_static_scratch on
// `device` (the current device); resolved on first use per device.
any4_status static_scratch(int device, void** ptr);

any4_status launch_prefill(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                           int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev);
}  // namespace any4
