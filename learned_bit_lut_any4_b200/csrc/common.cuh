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

// Table lookup in registers, no memory traffic: tl/th are the low/high byte
// planes of a 16-entry bf16 table (tl[i] holds the low bytes of entries
// 4i..4i+3).  For the 8 codes of w (code i at bits 4i..4i+3) returns the 8
// entries as 4 bf16 pairs, pair p = (entry of code 2p) | (entry of code 2p+1) << 16.
// Per 4 codes: byte permutes pick each byte from entries 0..7 and 8..15 by the
// code's low 3 bits, a sign-replicating permute turns each code's bit 3 into a
// byte mask, and a bitwise select keeps the right half-table's byte.
__device__ __forceinline__ void lookup8(uint32_t w, const uint32_t (&tl)[4],
                                        const uint32_t (&th)[4], uint32_t (&pair)[4]) {
  const uint32_t u = w << 4;  // bit 3 of codes 0, 2, 4, 6 into byte sign bits
#pragma unroll
  for (int hv = 0; hv < 2; ++hv) {
    const uint32_t sel = (hv ? (w >> 16) : w) & 0x7777u;
    // prmt's default mode: a selector nibble with bit 3 set replicates the
    // sign bit of the chosen byte (the __byte_perm intrinsic ignores bit 3)
    uint32_t m;
    if (hv)
      asm("prmt.b32 %0, %1, %2, 0xFBEA;" : "=r"(m) : "r"(u), "r"(w));
    else
      asm("prmt.b32 %0, %1, %2, 0xD9C8;" : "=r"(m) : "r"(u), "r"(w));
    const uint32_t x0 = __byte_perm(tl[0], tl[1], sel), x1 = __byte_perm(tl[2], tl[3], sel);
    const uint32_t y0 = __byte_perm(th[0], th[1], sel), y1 = __byte_perm(th[2], th[3], sel);
    const uint32_t lo = (x0 & ~m) | (x1 & m);
    const uint32_t hi = (y0 & ~m) | (y1 & m);
    pair[2 * hv] = __byte_perm(lo, hi, 0x5140u);
    pair[2 * hv + 1] = __byte_perm(lo, hi, 0x7362u);
  }
}

// The byte planes tl/th of lookup8 from a 16-entry bf16 table given as two
// 16-byte halves (entries 0-7 in e0, 8-15 in e1).
__device__ __forceinline__ void table_planes(const uint4& e0, const uint4& e1, uint32_t (&tl)[4],
                                             uint32_t (&th)[4]) {
  const uint32_t e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    tl[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x6420);
    th[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x7531);
  }
}

// Two bf16x2 lanes: a * b + c rounded once (bf16x2 fused multiply-add).
__device__ __forceinline__ uint32_t hfma2_bf16(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
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
// streaming: W written with evict-first stores (any4_dequant); false keeps
// what fits of W in L2 for a kernel that reads it next (the two-pass prefill).
any4_status launch_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                           const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                           int64_t N, int64_t K, int64_t G, cudaStream_t stream,
                           const DeviceInfo& dev, bool streaming = true);
any4_status launch_group_sums(const uint16_t* x, float* xsum, int64_t M, int64_t K, int64_t G,
                              cudaStream_t stream, const DeviceInfo& dev);
// out = XOR of the 32-bit words of buf[0 .. bytes) (bytes a multiple of 16);
// zeroes *out first, on the stream.
any4_status launch_read_probe(const void* buf, int64_t bytes, uint32_t* out, cudaStream_t stream,
                              const DeviceInfo& dev);
// The decode path (M <= 16).  y32, when not NULL, receives the fp32 sums
// instead of y (the unrounded results).  A workspace of at least
// decode_pair_workspace_size bytes selects the pair-table kernel for M <= 2.
any4_status launch_decode(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                          void* workspace, size_t workspace_bytes, bool overlap, bool pair_at_m1,
                          int32_t* dev_status, bool test_stall, cudaStream_t stream,
                          const DeviceInfo& dev);
// Pair-table decode for M <= 2 (decode_pair.cu): workspace bytes it needs on
// `dev` (0 when the shape is not supported).
bool decode_pair_supported(int64_t M, int64_t N, int64_t K, int64_t G);
size_t decode_pair_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G,
                                  const DeviceInfo& dev);
any4_status launch_decode_pair(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                               int64_t lut_row_stride, const uint16_t* scale,
                               const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                               int64_t N, int64_t K, int64_t G, void* workspace, bool overlap,
                               int32_t* dev_status, bool test_stall, cudaStream_t stream,
                               const DeviceInfo& dev);
// The weight-streaming decode kernel takes the shape (bits: code width 2..4).
bool decode_tma_supported(int64_t M, int64_t N, int64_t K, int64_t G, int bits = 4);
// One weight matrix of a grouped decode launch (y32, when not NULL, receives
// the fp32 sums instead of y).
struct DecodeWeights {
  const uint8_t* packed;
  const uint16_t* lut;
  int64_t lut_row_stride;
  const uint16_t* scale;
  const uint16_t* offset;
  uint16_t* y;
  float* y32;
  int64_t N;
};
// M = 1 on the weight-streaming kernel for up to ANY4_GROUP_MAX matrices that
// share x, K and G, in one launch (decode_layout: the codes are in
// any4_repack's layout; only where decode_layout_supported).
any4_status launch_decode_tma_group(const uint16_t* x, const DecodeWeights* w, int count,
                                    int64_t K, int64_t G, int bits, bool overlap,
                                    int32_t* dev_status, bool test_stall, cudaStream_t stream,
                                    const DeviceInfo& dev, bool decode_layout = false);
any4_status launch_decode_tma(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                              int64_t lut_row_stride, const uint16_t* scale,
                              const uint16_t* offset, uint16_t* y, float* y32, int64_t N,
                              int64_t K, int64_t G, bool overlap, int32_t* dev_status,
                              bool test_stall, cudaStream_t stream, const DeviceInfo& dev,
                              bool decode_layout = false);
// The folded-table M = 1 kernel takes the shape, so codes in any4_repack's
// layout can be used (M = 1, G = 128, K a multiple of 1024).
bool decode_layout_supported(int64_t M, int64_t N, int64_t K, int64_t G);
// any4_repack: packed codes into the decode layout (pack_dequant.cu).
any4_status launch_repack(const uint8_t* packed, uint8_t* repacked, int64_t N, int64_t K,
                          cudaStream_t stream, const DeviceInfo& dev);
size_t prefill_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G);
// n-bit (2 or 3) dequant into a bf16 W (nbit.cu).
any4_status launch_dequant_bits(const uint8_t* packed, const uint16_t* lut,
                                int64_t lut_row_stride, const uint16_t* scale,
                                const uint16_t* offset, uint16_t* W, int64_t N, int64_t K,
                                int64_t G, int bits, cudaStream_t stream, const DeviceInfo& dev);
// Skinny matmul for 2 <= M <= 16 (standard tensor-core mapping, table
// lookups by byte permute): skinny.cu.
any4_status launch_skinny(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                          bool overlap, cudaStream_t stream, const DeviceInfo& dev);

// cudaOccupancyMaxActiveBlocksPerMultiprocessor, remembered per (kernel,
// threads, dynamic shared memory) so that launches after the first of a shape
// make no occupancy query (it costs microseconds of host time per call).
// Returns 0 when the query fails.
int cached_occupancy(const void* kernel, int threads, size_t smem);

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) on the
// current device, skipped when that device already allows `kernel` at least
// `bytes`.  Function attributes belong to a device, so a process that
// launches on several GPUs opts each one in; the cache is keyed per (kernel,
// device) and guarded by a mutex (callers may be on several host threads).
any4_status ensure_dynamic_smem(const void* kernel, size_t bytes);

// Device address of the fixed scratch array of any4_matmul_static_scratch on
// `device` (the current device); resolved on first use per device.
any4_status static_scratch(int device, void** ptr);

any4_status launch_prefill(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                           int64_t N, int64_t K, int64_t G, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, bool test_stall,
                           cudaStream_t stream, const DeviceInfo& dev);
}  // namespace any4
