// Decode-path any4 matmul, M <= 16: y[m][n] = sum_k x[m][k] * W[n][k] with
// W[n][k] = LUT[n][c] * scale[n][k/G] + offset[n][k/G] never materialised.
//
// Paper: "any4: Learned 4-bit Numeric Representation for LLMs", §4.1 Eq. 8
// (y_i = sum_j dequant(w_Q[i,j]) x_j), §2.5.2 (dequant = alpha*w_Q + beta),
// §4.2 (memory-bound at small M; 16-byte coalesced loads; the 16-entry table
// held in one register and read with a warp shuffle, the 4-bit code being the
// source lane).
//
// Work decomposition (B200: 148 SMs, HBM-bound at small M):
//  * A lane owns a fixed KL-code chunk of K (KL = 32: one 16-byte load per
//    row); a warp covers a "slice" of 32*KL columns; the warps of a block
//    split K into slices.  A block owns R consecutive rows at a time and
//    loops over row blocks (grid = a multiple of the SM count).
//  * x for the lane's chunk lives in fp32 registers and is reused by every
//    row the warp visits.
//  * Each row's table sits in one register per lane: lane l holds entry
//    l & 15, so both half-warps hold the full table and `shfl` with the code
//    word shifted right selects the entry with no masking (the shuffle reads
//    only the low 5 bits of the source lane).
//  * Each weight is dequantised exactly as the definition rounds it,
//      W' = bf16(fmaf(LUT[c], scale, offset)),
//    two at a time (one cvt.rn.bf16x2), and multiplied with x in fp32 by the
//    mixed-precision bf16 x bf16 -> f32 FMA of sm_100 (products exact).
//    (Factoring the group scale out of the sum -- one FMA per weight --
//    skips that rounding and misses the tolerance on heavy-tailed tables.)
//  * Reduction: butterfly shuffles within the warp, then a fixed-order sum
//    over warps in shared memory.  No atomics: bitwise deterministic.
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kMaxWarps = 8;

template <int KL> struct CodeLoad;
template <> struct CodeLoad<32> {
  static constexpr int kWords = 4;
  __device__ __forceinline__ static void load(const uint8_t* p, uint32_t (&w)[4]) {
    const uint4 v = ldg_stream_v4(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
};
template <> struct CodeLoad<16> {
  static constexpr int kWords = 2;
  __device__ __forceinline__ static void load(const uint8_t* p, uint32_t (&w)[2]) {
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w[0]), "=r"(w[1]) : "l"(p));
  }
};
template <> struct CodeLoad<8> {
  static constexpr int kWords = 1;
  __device__ __forceinline__ static void load(const uint8_t* p, uint32_t (&w)[1]) {
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
  }
};

// W' = bf16(fmaf(LUT[c], s, o)) for two codes, packed as bf16x2 (first code
// in the low half): exactly the dequantised weights of the definition.
__device__ __forceinline__ uint32_t dequant_pair(float lut_lane, uint32_t c_lo, uint32_t c_hi,
                                                 float s, float o) {
  const float a = shfl_idx(lut_lane, c_lo);
  const float b = shfl_idx(lut_lane, c_hi);
  return pack_bf16x2_rn(__fmaf_rn(a, s, o), __fmaf_rn(b, s, o));
}

// acc_lo += W'.lo * x.lo ; acc_hi += W'.hi * x.hi  -- bf16 x bf16 products
// (exact) accumulated in fp32 by the mixed-precision FMA of sm_100.
__device__ __forceinline__ void fma_bf16x2_f32(float& acc_lo, float& acc_hi, uint32_t w,
                                               uint32_t xv) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %2;\n\tmov.b32 {xl, xh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, wl, xl, %0;\n\tfma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi) : "r"(w), "r"(xv));
}

template <int MT, int KL, int R>
__global__ void __launch_bounds__(kMaxWarps * 32) decode_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ y, int M, int64_t N, int64_t K, int64_t G, int nslices) {
  constexpr int KW = CodeLoad<KL>::kWords;
  __shared__ float s_part[kMaxWarps][R][MT];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t groups = K / G;
  const int64_t row_bytes = K / 2;
  const int64_t nblocks = (N + R - 1) / R;

  uint32_t xw[MT][KL / 2];  // x of the lane's chunk as bf16 pairs (even k low)
  int cur_slice = -1;

  for (int64_t rb = blockIdx.x; rb < nblocks; rb += gridDim.x) {
    const int64_t n0 = rb * R;
    float acc[R][MT][2];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m][0] = acc[r][m][1] = 0.f;

    for (int s = warp; s < nslices; s += nwarps) {
      const int64_t k0 = (int64_t)s * 32 * KL + (int64_t)lane * KL;
      const bool kin = k0 < K;

      // codes, tables and group parameters of the R rows (issued together)
      uint32_t code[R][KW];
      float lv[R], sv[R], ov[R];
      const int64_t g = kin ? k0 / G : 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t n = n0 + r;
        const bool rin = n < N;
        if (rin && kin) {
          CodeLoad<KL>::load(packed + n * row_bytes + k0 / 2, code[r]);
          sv[r] = bf16_lo_to_f32(ldg_u16(scale + n * groups + g));
          ov[r] = bf16_lo_to_f32(ldg_u16(offset + n * groups + g));
        } else {
#pragma unroll
          for (int w = 0; w < KW; ++w) code[r][w] = 0u;
          sv[r] = 0.f;
          ov[r] = 0.f;
        }
        lv[r] = rin ? bf16_lo_to_f32(ldg_u16(lut + n * lut_row_stride + (lane & 15))) : 0.f;
      }

      if (s != cur_slice) {  // activations of this chunk, reused across rows
        cur_slice = s;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < M && kin) {
            const uint16_t* xp = x + (int64_t)m * K + k0;
#pragma unroll
            for (int v = 0; v < KL / 8; ++v) {
              const uint4 q = ldg_nc_v4(xp + 8 * v);
              xw[m][4 * v] = q.x;
              xw[m][4 * v + 1] = q.y;
              xw[m][4 * v + 2] = q.z;
              xw[m][4 * v + 3] = q.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < KL / 2; ++i) xw[m][i] = 0u;
          }
        }
      }

#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int w = 0; w < KW; ++w) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // byte j of the word: codes of columns k0 + 8w + 2j (low nibble)
            // and k0 + 8w + 2j + 1 (high nibble)
            const uint32_t wp = dequant_pair(lv[r], code[r][w] >> (8 * j),
                                             code[r][w] >> (8 * j + 4), sv[r], ov[r]);
#pragma unroll
            for (int m = 0; m < MT; ++m)
              fma_bf16x2_f32(acc[r][m][0], acc[r][m][1], wp, xw[m][4 * w + j]);
          }
        }
      }
    }

    // reduce over the 32 lanes, then over warps in a fixed order
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float v = acc[r][m][0] + acc[r][m][1];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFullMask, v, off);
        if (lane == 0) s_part[warp][r][m] = v;
      }
    __syncthreads();
    if (threadIdx.x < R * MT) {
      const int r = threadIdx.x / MT;
      const int m = threadIdx.x % MT;
      const int64_t n = n0 + r;
      if (n < N && m < M) {
        float t = 0.f;
        for (int w = 0; w < nwarps; ++w) t += s_part[w][r][m];
        y[(int64_t)m * N + n] = f32_to_bf16_rn(t);
      }
    }
    __syncthreads();
  }
}

struct LaunchCfg {
  int threads;
  int grid;
};

template <int MT, int KL, int R>
any4_status run(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                uint16_t* y, int M, int64_t N, int64_t K, int64_t G, cudaStream_t stream,
                const DeviceInfo& dev) {
  const int64_t slice = 32LL * KL;
  const int nslices = (int)((K + slice - 1) / slice);
  const int nwarps = std::min(nslices, kMaxWarps);
  const int threads = nwarps * 32;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<MT, KL, R>, threads,
                                                    0) != cudaSuccess ||
      per_sm < 1) {
    per_sm = 1;
  }
  const int64_t nblocks = (N + R - 1) / R;
  const int64_t cap = (int64_t)dev.sm_count * per_sm;
  const int grid = (int)std::min<int64_t>(nblocks, cap);
  decode_kernel<MT, KL, R><<<grid, threads, 0, stream>>>(x, packed, lut, lut_row_stride, scale,
                                                         offset, y, M, N, K, G, nslices);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

any4_status launch_decode(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t G,
                          cudaStream_t stream, const DeviceInfo& dev) {
  // rows of x beyond 8 are handled by further launches over the same weights
  for (int64_t m0 = 0; m0 < M; m0 += 8) {
    const int mb = (int)std::min<int64_t>(M - m0, 8);
    const uint16_t* xb = x + m0 * K;
    uint16_t* yb = y + m0 * N;
    any4_status st;
    const bool few_rows = (N + 7) / 8 < 2LL * dev.sm_count;
    if (mb == 1) {
      st = few_rows ? run<1, 32, 4>(xb, packed, lut, lut_row_stride, scale, offset, yb, mb, N,
                                    K, G, stream, dev)
                    : run<1, 32, 8>(xb, packed, lut, lut_row_stride, scale, offset, yb, mb, N,
                                    K, G, stream, dev);
    } else if (mb == 2) {
      st = run<2, 32, 4>(xb, packed, lut, lut_row_stride, scale, offset, yb, mb, N, K, G,
                         stream, dev);
    } else if (mb <= 4) {
      st = run<4, 16, 4>(xb, packed, lut, lut_row_stride, scale, offset, yb, mb, N, K, G,
                         stream, dev);
    } else {
      st = run<8, 8, 4>(xb, packed, lut, lut_row_stride, scale, offset, yb, mb, N, K, G,
                        stream, dev);
    }
    if (st != ANY4_OK) return st;
  }
  return ANY4_OK;
}

}  // namespace any4
