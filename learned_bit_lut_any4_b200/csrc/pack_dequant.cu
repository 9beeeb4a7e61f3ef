// any4_pack and any4_dequant kernels (sm_100a).
//
// Both are streaming, HBM-bound transforms over the flat row-major arrays:
//   pack     reads N*K code bytes, writes N*K/2 bytes
//   dequant  reads N*K/2 code bytes (+ tables, scales, offsets), writes 2*N*K bytes
// Each thread handles one 16-byte packed chunk (32 codes).  K % 32 == 0, so a
// chunk never straddles a row, and G % 32 == 0, so it never straddles a group.
// Grids are a multiple of the SM count and loop (grid-stride) over chunks.
#include "common.cuh"

namespace any4 {
namespace {

// ---------------------------------------------------------------------------
// pack: byte j of row n = code(2j) | code(2j+1) << 4   (paper §4.2: two any4
// codes per byte; the even column goes to the low nibble)
// ---------------------------------------------------------------------------

// 4 code bytes c0..c3 (c0 in bits 0..7) -> 16 bits c0 | c1<<4 | c2<<8 | c3<<12.
__device__ __forceinline__ uint32_t pack4(uint32_t w) {
  uint32_t t = (w | (w >> 4)) & 0x00ff00ffu;  // byte0 = c0|c1<<4, byte2 = c2|c3<<4
  return (t & 0xffu) | (t >> 8);
}

__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ idx,
                                                    uint8_t* __restrict__ packed,
                                                    int64_t chunks, int32_t* dev_status) {
  uint32_t bad = 0;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = ldg_stream_v4(idx + c * 32);
    const uint4 b = ldg_stream_v4(idx + c * 32 + 16);
    bad |= a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w;
    uint4 o;
    o.x = pack4(a.x & 0x0f0f0f0fu) | (pack4(a.y & 0x0f0f0f0fu) << 16);
    o.y = pack4(a.z & 0x0f0f0f0fu) | (pack4(a.w & 0x0f0f0f0fu) << 16);
    o.z = pack4(b.x & 0x0f0f0f0fu) | (pack4(b.y & 0x0f0f0f0fu) << 16);
    o.w = pack4(b.z & 0x0f0f0f0fu) | (pack4(b.w & 0x0f0f0f0fu) << 16);
    stg_stream_v4(packed + c * 16, o);
  }
  // any code byte above 15 has a bit set in its high nibble
  if (__any_sync(kFullMask, (bad & 0xf0f0f0f0u) != 0u)) {
    if ((threadIdx.x & 31) == 0) report_status(dev_status, (int32_t)ANY4_ERR_RANGE);
  }
}

// ---------------------------------------------------------------------------
// dequant: W = bf16_rne(fmaf(LUT[n][c], scale[n][g], offset[n][g]))
// (paper §2.5.2 dequant(w_Q) = alpha*w_Q + beta with w_Q = LUT[c], §2.4.1)
// ---------------------------------------------------------------------------

constexpr int kDqThreads = 256;
// A block covers 256 consecutive chunks; with K >= 32 (one chunk per row at
// least) that touches at most 256 rows.
constexpr int kDqMaxRows = kDqThreads;

__global__ void __launch_bounds__(kDqThreads) dequant_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ W, int64_t N, int64_t K, int64_t G) {
  __shared__ float s_lut[kDqMaxRows][16];
  const int64_t chunks_per_row = K / 32;
  const int64_t chunks = N * chunks_per_row;
  const int64_t groups = K / G;
  for (int64_t base = (int64_t)blockIdx.x * kDqThreads; base < chunks;
       base += (int64_t)gridDim.x * kDqThreads) {
    const int64_t row0 = base / chunks_per_row;
    const int64_t last = min(base + kDqThreads, chunks) - 1;
    const int nrows = (int)(last / chunks_per_row - row0 + 1);
    __syncthreads();  // previous iteration's readers are done with s_lut
    for (int i = threadIdx.x; i < nrows * 16; i += kDqThreads) {
      const int64_t n = row0 + i / 16;
      s_lut[i / 16][i % 16] = bf16_lo_to_f32(ldg_u16(lut + n * lut_row_stride + (i % 16)));
    }
    __syncthreads();
    const int64_t c = base + threadIdx.x;
    if (c < chunks) {
      const int64_t n = c / chunks_per_row;
      const int64_t k0 = (c - n * chunks_per_row) * 32;
      const int64_t g = k0 / G;
      const float s = bf16_lo_to_f32(ldg_u16(scale + n * groups + g));
      const float o = bf16_lo_to_f32(ldg_u16(offset + n * groups + g));
      const float* t = s_lut[n - row0];
      const uint4 q = ldg_stream_v4(packed + c * 16);
      const uint32_t words[4] = {q.x, q.y, q.z, q.w};
      uint32_t out[16];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          // byte p of word w holds the codes of columns k0 + 8w + 2p (low
          // nibble) and k0 + 8w + 2p + 1 (high nibble)
          const uint32_t byte = (words[w] >> (8 * p)) & 0xffu;
          const float lo = __fmaf_rn(t[byte & 15u], s, o);
          const float hi = __fmaf_rn(t[byte >> 4], s, o);
          out[4 * w + p] = pack_bf16x2_rn(lo, hi);
        }
      }
      uint16_t* dst = W + n * K + k0;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        stg_stream_v4(dst + 8 * v, make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2],
                                              out[4 * v + 3]));
      }
    }
  }
}

int grid_for(int64_t work_items, int threads, const DeviceInfo& dev, int blocks_per_sm) {
  const int64_t want = (work_items + threads - 1) / threads;
  const int64_t cap = (int64_t)dev.sm_count * blocks_per_sm;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

any4_status launch_pack(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                        int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t chunks = N * K / 32;
  pack_kernel<<<grid_for(chunks, 256, dev, 8), 256, 0, stream>>>(idx, packed, chunks,
                                                                  dev_status);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

any4_status launch_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                           const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                           int64_t N, int64_t K, int64_t G, cudaStream_t stream,
                           const DeviceInfo& dev) {
  const int64_t chunks = N * K / 32;
  dequant_kernel<<<grid_for(chunks, kDqThreads, dev, 8), kDqThreads, 0, stream>>>(
      packed, lut, lut_row_stride, scale, offset, W, N, K, G);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
