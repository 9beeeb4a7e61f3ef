// any4_pack and any4_dequant kernels (sm_100a).
//
// Both are streaming, HBM-bound transforms over the flat row-major arrays:
//   pack     reads N*K code bytes, writes N*K/2 bytes
//   dequant  reads N*K/2 code bytes (+ tables, scales, offsets), writes 2*N*K bytes
// pack: each thread handles one 16-byte packed chunk (32 codes); K % 32 == 0,
// so a chunk never straddles a row.  dequant: a warp per 1024-column segment
// (below).  Grids are a multiple of the SM count and loop (grid-stride).
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

// One warp per 1024-column segment of a row.  Lane l converts the 8 codes at
// columns 256 v + 8 l .. + 7 of the segment (v = 0..3), so each of the warp's
// 4-byte code loads covers 128 consecutive bytes and each 16-byte result lands
// next to its neighbour lane's in a shared-memory copy of the segment's bf16
// row; one bulk copy (cp.async.bulk) then writes the whole segment, 2 KiB in
// one piece, while the warp goes on with its next segment (two staging
// buffers per warp).  The row's table sits in shared memory as fp32 (16
// entries, 16 banks: conflict free).
constexpr int kDqWarps = 8;
constexpr int kDqThreads = kDqWarps * 32;
constexpr int kDqSeg = 1024;

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__global__ void __launch_bounds__(kDqThreads) dequant_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ W, int64_t N, int64_t K, int64_t G) {
  __shared__ __align__(128) uint16_t s_out[kDqWarps][2][kDqSeg];
  __shared__ float s_lut[kDqWarps][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t segs_per_row = (K + kDqSeg - 1) / kDqSeg;
  const int64_t nseg = N * segs_per_row;
  const int64_t groups = K / G;
  int64_t cur_row = -1;
  int buf = 0;
  for (int64_t sg = (int64_t)blockIdx.x * kDqWarps + warp; sg < nseg;
       sg += (int64_t)gridDim.x * kDqWarps) {
    const int64_t n = sg / segs_per_row;
    const int64_t col0 = (sg - n * segs_per_row) * kDqSeg;
    const int cols = (int)min((int64_t)kDqSeg, K - col0);  // a multiple of 32
    uint32_t w[4];
    float sv[4], ov[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = 256 * v + 8 * lane;
      w[v] = 0u;
      sv[v] = ov[v] = 0.f;
      if (c < cols) {
        const int64_t k = col0 + c;
        w[v] = ldg_nc_u32(packed + (n * K + k) / 2);
        const int64_t gi = n * groups + k / G;
        sv[v] = bf16_lo_to_f32(ldg_u16(scale + gi));
        ov[v] = bf16_lo_to_f32(ldg_u16(offset + gi));
      }
    }
    if (n != cur_row) {  // this warp moves to a new row: its table as fp32
      __syncwarp();
      if (lane < 16) s_lut[warp][lane] = bf16_lo_to_f32(ldg_u16(lut + n * lut_row_stride + lane));
      __syncwarp();
      cur_row = n;
    }
    // the bulk copy that last read this buffer (two segments ago) must be done
    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    __syncwarp();
    const float* t = s_lut[warp];
    uint16_t* out = s_out[warp][buf];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = 256 * v + 8 * lane;
      if (c < cols) {
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          // byte p of the word: codes of columns c + 2p (low nibble), c + 2p + 1
          const uint32_t byte = (w[v] >> (8 * p)) & 0xffu;
          const float lo = __fmaf_rn(t[byte & 15u], sv[v], ov[v]);
          const float hi = __fmaf_rn(t[byte >> 4], sv[v], ov[v]);
          o[p] = pack_bf16x2_rn(lo, hi);
        }
        *reinterpret_cast<uint4*>(out + c) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                   :: "l"(W + n * K + col0), "r"((uint32_t)__cvta_generic_to_shared(out)),
                      "r"((uint32_t)cols * 2u) : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    buf ^= 1;
  }
  // every bulk copy of this warp has finished before the block's shared memory goes
  if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  __syncwarp();
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
  const int64_t segs = N * ((K + kDqSeg - 1) / kDqSeg);
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(dequant_kernel), kDqThreads, 0);
  if (per_sm < 1) per_sm = 1;
  dequant_kernel<<<grid_for(segs * 32, kDqThreads, dev, per_sm), kDqThreads, 0, stream>>>(
      packed, lut, lut_row_stride, scale, offset, W, N, K, G);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
