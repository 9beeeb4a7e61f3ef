// n-bit storage below 4 bits (any3, any2): pack and dequant kernels (sm_100a).
//
// "any4: Learned 4-bit Numeric Representation for LLMs" states the table for
// any bit width (§4.1 Eq. 9: 2^n values per row) and evaluates any3 and any2
// (§5); it gives no storage layout below 4 bits.  Layout here: the codes of a
// row form one little-endian bit stream, code k in bits [n k, n k + n), so a
// row of K codes takes n K / 8 bytes (for n = 4 this is any4's nibble order,
// which any4_pack / any4_dequant already serve).  A thread handles one chunk
// of 32 codes: n 32-bit words, inside one row (K % 32 == 0) and one group
// (G % 32 == 0).  Both kernels are streaming and HBM-bound; grids are a
// multiple of the SM count and loop over the chunks (pack) or over 1024-column
// segments of rows (dequant, a warp per segment).
#include <algorithm>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kNbThreads = 256;

template <int BITS>
__device__ __forceinline__ void load_chunk(const uint8_t* p, uint32_t (&v)[BITS]) {
  if constexpr (BITS == 2) {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = t.x;
    v[1] = t.y;
  } else {
#pragma unroll
    for (int b = 0; b < BITS; ++b) v[b] = __ldg(reinterpret_cast<const uint32_t*>(p) + b);
  }
}

template <int BITS>
__device__ __forceinline__ void store_chunk(uint8_t* p, const uint32_t (&v)[BITS]) {
  if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(p) = make_uint2(v[0], v[1]);
  } else {
#pragma unroll
    for (int b = 0; b < BITS; ++b) reinterpret_cast<uint32_t*>(p)[b] = v[b];
  }
}

// Code k (0..31) of a chunk held in BITS words.
template <int BITS>
__device__ __forceinline__ uint32_t code_of(const uint32_t (&v)[BITS], int k) {
  const int bit = BITS * k, w = bit >> 5, off = bit & 31;
  uint32_t c = v[w] >> off;
  if (off + BITS > 32) c |= v[w + 1] << (32 - off);
  return c & ((1u << BITS) - 1u);
}

template <int BITS>
__global__ void __launch_bounds__(kNbThreads)
pack_bits_kernel(const uint8_t* __restrict__ idx, uint8_t* __restrict__ packed, int64_t chunks,
                 int32_t* dev_status) {
  constexpr uint32_t kMask = (1u << BITS) - 1u;
  constexpr uint32_t kHigh = (~kMask & 0xffu) * 0x01010101u;  // bits no code may set
  uint32_t bad = 0;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = ldg_stream_v4(idx + c * 32);
    const uint4 b = ldg_stream_v4(idx + c * 32 + 16);
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t v[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) v[i] = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint32_t cd = (in[k >> 2] >> (8 * (k & 3))) & kMask;
      const int bit = BITS * k, w = bit >> 5, off = bit & 31;
      v[w] |= cd << off;
      if (off + BITS > 32) v[w + 1] |= cd >> (32 - off);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) bad |= in[i] & kHigh;
    store_chunk<BITS>(packed + c * (4 * BITS), v);
  }
  if (__any_sync(kFullMask, bad != 0u)) {
    if ((threadIdx.x & 31) == 0) report_status(dev_status, (int32_t)ANY4_ERR_RANGE);
  }
}

// dequant: one warp per 1024-column segment of a row, lane l on the segment's
// 32-code chunk l (its n words are the n * 4 bytes after lane l - 1's, so the
// warp's code loads are contiguous).  The loads of the warp's next segment
// (codes, the chunk's scale and offset, the row's table) are issued before the
// current one is converted.  The 64 output bytes of a lane go to a
// shared-memory copy of the segment's bf16 row, 16 bytes at a time in a
// lane-rotated order (lanes 2i and 2i + 1 start at the 16-byte unit i mod 4
// of their 64 bytes), which keeps every phase of 8 lanes on 8 distinct bank
// groups; the warp then writes the segment with 16-byte streaming stores,
// 512 consecutive bytes per instruction.
constexpr int kNbWarps = 8;
constexpr int kNbSeg = 1024;

__device__ __forceinline__ void nb_stg_cs_v4(void* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
               :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

template <int BITS>
__global__ void __launch_bounds__(kNbWarps * 32)
dequant_bits_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ lut,
                    int64_t lut_row_stride, const uint16_t* __restrict__ scale,
                    const uint16_t* __restrict__ offset, uint16_t* __restrict__ W, int64_t N,
                    int K, int G, int g_shift) {
  __shared__ __align__(128) uint16_t s_out[kNbWarps][kNbSeg];
  __shared__ float s_lut[kNbWarps][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int segs_per_row = (K + kNbSeg - 1) / kNbSeg;
  const int64_t nseg = N * segs_per_row;
  const int groups = K / G;
  const int64_t first = (int64_t)blockIdx.x * kNbWarps + warp;
  const int64_t stride = (int64_t)gridDim.x * kNbWarps;
  if (first >= nseg) return;
  // (row, segment) of the warp's segments without a division per step
  const int64_t n_step = stride / segs_per_row;
  const int s_step = (int)(stride % segs_per_row);
  auto advance = [&](int64_t& n, int& seg) {
    n += n_step;
    seg += s_step;
    if (seg >= segs_per_row) {
      seg -= segs_per_row;
      ++n;
    }
  };
  // one segment's inputs, per lane
  constexpr int NQ = 1 << BITS;
  struct Seg {
    uint32_t v[BITS];
    uint32_t lv;  // lanes 0 .. NQ-1: entry `lane` of the row's table (bf16 bits)
    uint32_t so;  // scale (low half) and offset (high half)
  };
  auto load = [&](int64_t n, int seg, Seg& d) {
    const int col0 = seg * kNbSeg;
    const int k0 = col0 + 32 * lane;
    d.lv = lane < NQ ? (uint32_t)ldg_u16(lut + n * lut_row_stride + lane) : 0u;
#pragma unroll
    for (int b = 0; b < BITS; ++b) d.v[b] = 0u;
    d.so = 0u;
    if (32 * lane < min(kNbSeg, K - col0)) {
      const uint32_t g = g_shift >= 0 ? ((uint32_t)k0 >> g_shift) : (uint32_t)k0 / (uint32_t)G;
      d.so = (uint32_t)ldg_u16(scale + n * groups + g) |
             ((uint32_t)ldg_u16(offset + n * groups + g) << 16);
      load_chunk<BITS>(packed + (n * K + k0) / 8 * BITS, d.v);
    }
  };
  int64_t n = first / segs_per_row, ln = n;
  int seg = (int)(first % segs_per_row), lseg = seg;
  Seg nxt;
  load(ln, lseg, nxt);
  advance(ln, lseg);
  int64_t cur_row = -1;
  for (int64_t sg = first; sg < nseg; sg += stride) {
    const int col0 = seg * kNbSeg;
    const int cols = min(kNbSeg, K - col0);  // a multiple of 32
    const bool on = 32 * lane < cols;
    const Seg cur = nxt;
    if (sg + stride < nseg) {  // the next segment's loads go out before this one's math
      load(ln, lseg, nxt);
      advance(ln, lseg);
    }
    uint16_t* seg_out = s_out[warp];
    float* tab = s_lut[warp];
    __syncwarp();  // the previous segment's row and table have been read
    if (n != cur_row) {  // a new row: its table as fp32 in shared memory
      if (lane < NQ) tab[lane] = bf16_lo_to_f32(cur.lv);
      __syncwarp();
      cur_row = n;
    }
    const float s = bf16_lo_to_f32(cur.so), o = bf16_hi_to_f32(cur.so);
    uint32_t out[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const float lo = __fmaf_rn(tab[code_of<BITS>(cur.v, 2 * p)], s, o);
      const float hi = __fmaf_rn(tab[code_of<BITS>(cur.v, 2 * p + 1)], s, o);
      out[p] = pack_bf16x2_rn(lo, hi);
    }
    if (on) {
#pragma unroll
      for (int step = 0; step < 4; ++step) {
        const int q = (step + (lane >> 1)) & 3;  // 16-byte unit of this lane's 64 bytes
        const uint4 val = q == 0 ? make_uint4(out[0], out[1], out[2], out[3])
                        : q == 1 ? make_uint4(out[4], out[5], out[6], out[7])
                        : q == 2 ? make_uint4(out[8], out[9], out[10], out[11])
                                 : make_uint4(out[12], out[13], out[14], out[15]);
        *reinterpret_cast<uint4*>(seg_out + 32 * lane + 8 * q) = val;
      }
    }
    __syncwarp();
    // 16-byte unit u = 32 q + lane of the segment's row: 512 contiguous bytes per q
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = 8 * (32 * q + lane);
      if (c < cols)
        nb_stg_cs_v4(W + n * K + col0 + c, *reinterpret_cast<const uint4*>(seg_out + c));
    }
    advance(n, seg);
  }
}

int nb_pow2_shift(int64_t G) {
  for (int s = 0; s < 31; ++s)
    if ((int64_t(1) << s) == G) return s;
  return -1;
}

int nb_grid(int64_t chunks, const DeviceInfo& dev) {
  const int64_t want = (chunks + kNbThreads - 1) / kNbThreads;
  const int64_t cap = (int64_t)dev.sm_count * 8;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

any4_status launch_pack_bits(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                             int bits, int32_t* dev_status, cudaStream_t stream,
                             const DeviceInfo& dev) {
  const int64_t chunks = N * K / 32;
  if (bits == 3)
    pack_bits_kernel<3><<<nb_grid(chunks, dev), kNbThreads, 0, stream>>>(idx, packed, chunks,
                                                                          dev_status);
  else if (bits == 2)
    pack_bits_kernel<2><<<nb_grid(chunks, dev), kNbThreads, 0, stream>>>(idx, packed, chunks,
                                                                          dev_status);
  else
    return ANY4_ERR_SHAPE;
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

any4_status launch_dequant_bits(const uint8_t* packed, const uint16_t* lut,
                                int64_t lut_row_stride, const uint16_t* scale,
                                const uint16_t* offset, uint16_t* W, int64_t N, int64_t K,
                                int64_t G, int bits, cudaStream_t stream, const DeviceInfo& dev) {
  // a warp per 1024-column segment; 8 warps per block
  const int64_t segs = N * ((K + kNbSeg - 1) / kNbSeg);
  auto kern = bits == 3 ? dequant_bits_kernel<3> : dequant_bits_kernel<2>;
  if (bits != 3 && bits != 2) return ANY4_ERR_SHAPE;
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(kern), kNbWarps * 32, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t want = (segs + kNbWarps - 1) / kNbWarps;
  const int64_t cap = (int64_t)dev.sm_count * per_sm;
  if (K > INT32_MAX / 2) return ANY4_ERR_SHAPE;
  kern<<<(unsigned)std::max<int64_t>(1, std::min(want, cap)), kNbWarps * 32, 0, stream>>>(
      packed, lut, lut_row_stride, scale, offset, W, N, (int)K, (int)G, nb_pow2_shift(G));
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
