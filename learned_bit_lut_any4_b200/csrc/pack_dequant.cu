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

// One warp per 1024-column segment of a row, segments walked grid-stride.
// Lane l converts the 8 codes at columns 256 v + 8 l .. + 7 (v = 0..3): each
// of the warp's 4-byte code loads covers 128 consecutive bytes and each of
// its 16-byte streaming stores 512 consecutive bytes of W.  The loads of the
// warp's next segment are issued before the current one is converted (one
// segment ahead, in registers).  The kernel moves 4 bytes of W out per byte
// of codes in, and on B200 that mix of reads and writes streams at about
// 5 TB/s with no arithmetic at all; a deeper prefetch (in registers, or
// through a shared-memory ring fed by bulk copies) and bulk-copy stores were
// both measured slower: they cost resident warps.  The row's table sits in
// shared memory as fp32 (16 entries, 16 banks: conflict free).
constexpr int kDqWarps = 8;
constexpr int kDqThreads = kDqWarps * 32;
constexpr int kDqSeg = 1024;

__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ void stg_cs_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
               :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// group of column k: a shift when G is a power of two (g_shift >= 0)
__device__ __forceinline__ uint32_t group_of(uint32_t k, int g_shift, uint32_t G) {
  return g_shift >= 0 ? (k >> g_shift) : k / G;
}

// kFull: K is a multiple of the segment width, so no lane needs a bounds test;
// kStream: streaming stores (W is not read again soon) or plain write-back
// stores (the two-pass prefill reads W right after: what stays in L2 helps)
template <bool kFull, bool kStream>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ W, int64_t N, int K, int G, int g_shift) {
  __shared__ float s_lut[kDqWarps][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int segs_per_row = (K + kDqSeg - 1) / kDqSeg;
  const int64_t nseg = N * segs_per_row;
  const int groups = K / G;
  const int64_t first = (int64_t)blockIdx.x * kDqWarps + warp;
  const int64_t stride = (int64_t)gridDim.x * kDqWarps;
  if (first >= nseg) return;
  // codes and the groups' scale (low half) and offset (high half) of one
  // segment, per lane
  struct Seg {
    uint32_t w[4];
    uint32_t so[4];
  };
  auto load = [&](int64_t n, int si, Seg& d) {
    const int col0 = si * kDqSeg;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = 256 * v + 8 * lane;
      if (kFull || c < K - col0) {
        const uint32_t k = (uint32_t)(col0 + c);
        d.w[v] = ldg_nc_u32(packed + (n * K + k) / 2);
        const int64_t gi = n * groups + group_of(k, g_shift, (uint32_t)G);
        d.so[v] = (uint32_t)ldg_u16(scale + gi) | ((uint32_t)ldg_u16(offset + gi) << 16);
      } else {
        d.w[v] = 0u;
        d.so[v] = 0u;
      }
    }
  };
  // the next segment's (row, segment of the row), advanced by the grid
  // stride without a division per segment
  const int64_t step_rows = stride / segs_per_row;
  const int step_segs = (int)(stride - step_rows * segs_per_row);
  int64_t n_nxt = first / segs_per_row;
  int si_nxt = (int)(first - n_nxt * segs_per_row);
  Seg nxt;
  load(n_nxt, si_nxt, nxt);
  int64_t cur_row = -1;
  for (int64_t sg = first; sg < nseg; sg += stride) {
    const int64_t n = n_nxt;
    const int col0 = si_nxt * kDqSeg;
    n_nxt += step_rows;
    si_nxt += step_segs;
    if (si_nxt >= segs_per_row) {
      si_nxt -= segs_per_row;
      ++n_nxt;
    }
    if (n != cur_row) {  // this warp moves to a new row: its table as fp32
      __syncwarp();
      if (lane < 16) s_lut[warp][lane] = bf16_lo_to_f32(ldg_u16(lut + n * lut_row_stride + lane));
      __syncwarp();
      cur_row = n;
    }
    const Seg cur = nxt;
    if (sg + stride < nseg) load(n_nxt, si_nxt, nxt);  // out before this segment's math
    const float* t = s_lut[warp];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = 256 * v + 8 * lane;
      if (kFull || c < K - col0) {
        const float sv = bf16_lo_to_f32(cur.so[v]), ov = bf16_hi_to_f32(cur.so[v]);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          // byte p of the word: codes of columns c + 2p (low nibble), c + 2p + 1
          const uint32_t byte = (cur.w[v] >> (8 * p)) & 0xffu;
          const float lo = __fmaf_rn(t[byte & 15u], sv, ov);
          const float hi = __fmaf_rn(t[byte >> 4], sv, ov);
          o[p] = pack_bf16x2_rn(lo, hi);
        }
        if (kStream)
          stg_cs_v4(W + n * K + col0 + c, o[0], o[1], o[2], o[3]);
        else
          *reinterpret_cast<uint4*>(W + n * K + col0 + c) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// G a multiple of 128 and K a multiple of 1024: the table folded with the
// group's scale and offset.  A warp still owns 1024-column segments and writes
// them with the same 512-byte warp stores, but step p (0..3) of a lane in half
// h covers columns 256 p + 128 h + 8 (lane & 15) .. + 7, so a half-warp spans
// 128 columns of one group at a time.  Source lane e of half h then holds, for
// its half's groups of steps 2i and 2i + 1, the bf16 pair
//   (bf16(fmaf(LUT[e], s, o)) of step 2i, the same of step 2i + 1),
// the weight of the definition for code e, and a lookup is one shuffle inside
// the half-warp (segment mask 16) with the shifted code word, a byte permute
// pairing two weights in the half of the step.  Per weight that is a shift, a
// shuffle and half a permute instead of a table load, an fp32 FMA and half a
// conversion: the arithmetic no longer competes with the memory stream.
template <bool kStream>
__global__ void __launch_bounds__(kDqThreads) dequant_fold_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ W, int64_t N, int K, int G, int g_shift) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = lane >> 4, e = lane & 15;
  const int segs_per_row = K / kDqSeg;
  const int64_t nseg = N * segs_per_row;
  const int groups = K / G;
  const int64_t first = (int64_t)blockIdx.x * kDqWarps + warp;
  const int64_t stride = (int64_t)gridDim.x * kDqWarps;
  if (first >= nseg) return;
  // codes, and the scale (low half) and offset (high half) of the lane's
  // group at each step, of one segment
  struct Seg {
    uint32_t w[4];
    uint32_t so[4];
  };
  auto load = [&](int64_t n, int si, Seg& d) {
    const int col0 = si * kDqSeg;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t k = (uint32_t)(col0 + 256 * p + 128 * h + 8 * e);
      d.w[p] = ldg_nc_u32(packed + (n * K + k) / 2);
      const int64_t gi = n * groups + group_of(k, g_shift, (uint32_t)G);
      d.so[p] = (uint32_t)ldg_u16(scale + gi) | ((uint32_t)ldg_u16(offset + gi) << 16);
    }
  };
  // the next segment's (row, segment of the row), advanced by the grid
  // stride without a division per segment
  const int64_t step_rows = stride / segs_per_row;
  const int step_segs = (int)(stride - step_rows * segs_per_row);
  int64_t n_nxt = first / segs_per_row;
  int si_nxt = (int)(first - n_nxt * segs_per_row);
  Seg nxt;
  load(n_nxt, si_nxt, nxt);
  int64_t cur_row = -1;
  float lv = 0.f;  // LUT[row][e]
  for (int64_t sg = first; sg < nseg; sg += stride) {
    const int64_t n = n_nxt;
    const int col0 = si_nxt * kDqSeg;
    n_nxt += step_rows;
    si_nxt += step_segs;
    if (si_nxt >= segs_per_row) {
      si_nxt -= segs_per_row;
      ++n_nxt;
    }
    if (n != cur_row) {
      lv = bf16_lo_to_f32(ldg_u16(lut + n * lut_row_stride + e));
      cur_row = n;
    }
    const Seg cur = nxt;
    if (sg + stride < nseg) load(n_nxt, si_nxt, nxt);  // out before this segment's math
    uint32_t tab[2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
      tab[i] = pack_bf16x2_rn(
          __fmaf_rn(lv, bf16_lo_to_f32(cur.so[2 * i]), bf16_hi_to_f32(cur.so[2 * i])),
          __fmaf_rn(lv, bf16_lo_to_f32(cur.so[2 * i + 1]), bf16_hi_to_f32(cur.so[2 * i + 1])));
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t sel = (p & 1) ? 0x7632u : 0x5410u;
      uint32_t o[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t a, b;
        asm("shfl.sync.idx.b32 %0, %1, %2, 0x101f, 0xffffffff;"
            : "=r"(a) : "r"(tab[p >> 1]), "r"(cur.w[p] >> (8 * m)));
        asm("shfl.sync.idx.b32 %0, %1, %2, 0x101f, 0xffffffff;"
            : "=r"(b) : "r"(tab[p >> 1]), "r"(cur.w[p] >> (8 * m + 4)));
        o[m] = __byte_perm(a, b, sel);
      }
      uint16_t* dst = W + n * K + col0 + 256 * p + 128 * h + 8 * e;
      if (kStream)
        stg_cs_v4(dst, o[0], o[1], o[2], o[3]);
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

int pow2_shift(int64_t G) {
  for (int s = 0; s < 31; ++s)
    if ((int64_t(1) << s) == G) return s;
  return -1;
}

int grid_for(int64_t work_items, int threads, const DeviceInfo& dev, int blocks_per_sm) {
  const int64_t want = (work_items + threads - 1) / threads;
  const int64_t cap = (int64_t)dev.sm_count * blocks_per_sm;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

// any4_repack: one thread per 16-byte chunk of the decode layout (chunk l of
// a row's 1024-column slice: the slice's words 16 (4h + (t ^ h)) + e for
// t = 0..3, h = l / 16, e = l mod 16).  The four gathered words of a warp's
// threads come from the same 512-byte slice (one cache line set), the store
// is one coalesced 16-byte write per thread.
__global__ void __launch_bounds__(256) repack_kernel(const uint32_t* __restrict__ in,
                                                      uint4* __restrict__ out, int64_t chunks) {
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int l = (int)(c & 31);
    const int h = l >> 4, e = l & 15;
    const uint32_t* slice = in + (c >> 5) * 128;
    uint4 v;
    v.x = __ldg(slice + 16 * (4 * h + (0 ^ h)) + e);
    v.y = __ldg(slice + 16 * (4 * h + (1 ^ h)) + e);
    v.z = __ldg(slice + 16 * (4 * h + (2 ^ h)) + e);
    v.w = __ldg(slice + 16 * (4 * h + (3 ^ h)) + e);
    out[c] = v;
  }
}

}  // namespace

any4_status launch_repack(const uint8_t* packed, uint8_t* repacked, int64_t N, int64_t K,
                          cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t chunks = N * (K / 1024) * 32;  // a slice is 1024 codes = 32 chunks of 16 bytes
  repack_kernel<<<grid_for(chunks, 256, dev, 8), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<uint4*>(repacked), chunks);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

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
                           const DeviceInfo& dev, bool streaming) {
  if (K > INT32_MAX / 2) return ANY4_ERR_SHAPE;
  const int64_t segs = N * ((K + kDqSeg - 1) / kDqSeg);
  // the folded-table kernel where a half-warp step stays inside one group
  const bool fold = K % kDqSeg == 0 && G % 128 == 0;
  auto kern = fold ? (streaming ? dequant_fold_kernel<true> : dequant_fold_kernel<false>)
            : K % kDqSeg == 0
                ? (streaming ? dequant_kernel<true, true> : dequant_kernel<true, false>)
                : (streaming ? dequant_kernel<false, true> : dequant_kernel<false, false>);
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(kern), kDqThreads, 0);
  if (per_sm < 1) per_sm = 1;
  kern<<<grid_for(segs * 32, kDqThreads, dev, per_sm), kDqThreads, 0, stream>>>(
      packed, lut, lut_row_stride, scale, offset, W, N, (int)K, (int)G, pow2_shift(G));
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
