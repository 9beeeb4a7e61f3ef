// Decode-path any4 matmul, M <= 16: y[m][n] = sum_k x[m][k] * W[n][k] with
// W[n][k] = LUT[n][c] * scale[n][k/G] + offset[n][k/G] never materialised.
//
// launch_decode dispatches: M = 1 goes to the weight-streaming kernel of
// decode_tma.cu where its shape rules allow (G in {32, 64, 128}, K/G a
// multiple of 8), else to the kernel below (instantiated for one row of x);
// 2 <= M <= 16 goes to skinny.cu, which dequantises each weight once for all
// rows of x.
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
//  * Each weight is dequantised as W' = LUT[c] * scale + offset rounded once
//    to bf16, two at a time (one bf16x2 fused multiply-add; this equals the
//    definition's bf16(fmaf(...)) except when that fp32 fmaf is inexact and
//    lands on a bf16 rounding tie), and the products with x are exact in the
//    tensor core's fp32 accumulation.
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
constexpr int kMaxRowsMT = 1024;  // rows_per_block * MT bound (shared memory partials)

template <int KL> struct CodeLoad;
template <> struct CodeLoad<32> {
  static constexpr int kWords = 4;
  __device__ __forceinline__ static void load(const uint8_t* p, uint32_t (&w)[4]) {
    const uint4 v = ldg_stream_v4(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
};
// W' = LUT[c] * s + o for two codes, packed as bf16x2 (first code in the low
// half): both table entries (bf16 bits, lane l holding entry l & 15) fetched
// by shuffle, paired, and one bf16x2 fused multiply-add rounds the exact
// value once to bf16 -- bf16(fmaf(LUT, s, o)) unless that fp32 fmaf is
// inexact and lands on a bf16 rounding tie.  s2, o2: scale, offset in both halves.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t lut_lane, uint32_t c_lo, uint32_t c_hi,
                                                 uint32_t s2, uint32_t o2) {
  uint32_t a, b, w;
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=r"(a) : "r"(lut_lane), "r"(c_lo));
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=r"(b) : "r"(lut_lane), "r"(c_hi));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(w) : "r"(__byte_perm(a, b, 0x5410)), "r"(s2), "r"(o2));
  return w;
}

// Sum V = 2^v per-lane values over the 32 lanes, leaving value i's total in
// the lanes whose bits 4, 3, ... (one per halving step) spell i (most
// significant first).  V - 1 + 5 - log2(V) shuffles instead of 5 V.
// D += A * B on the legacy warp-level tensor-core instruction (bf16 inputs,
// fp32 accumulation): m16n8k16, A row-major 16 x 16, B column-major 16 x 8.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V], int lane) {
  int n = V;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (lane & off) != 0;
      const int half = n / 2;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < half) {
          const float give = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(kFullMask, give, off);
        }
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(kFullMask, v[0], off);
    }
  }
  return v[0];
}

// Which of the V values lane `lane` holds after transpose_reduce<V>.
template <int V>
__device__ __forceinline__ int transpose_reduce_index(int lane) {
  int idx = 0;
  int n = V;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      idx = 2 * idx + ((lane & off) ? 1 : 0);
      n /= 2;
    }
  }
  return idx;
}

// The per-row loads of one lane: its KL codes, the row's table entry for
// this lane, and the group scale/offset of its chunk.
template <int KW>
struct RowRegs {
  uint32_t code[KW];
  uint32_t lv;      // table entry lane & 15 (bf16 bits)
  uint32_t sv, ov;  // group scale and offset, bf16 bits in both halves
};

// Where one lane's data of the current row lives; advanced row by row.
struct RowPtrs {
  const uint8_t* pk;   // the lane's KL codes
  const uint16_t* lt;  // table entry lane & 15
  const uint16_t* sc;  // scale of the chunk's group
  const uint16_t* of;  // offset of the chunk's group
};

template <int KL>
__device__ __forceinline__ void load_row(RowRegs<CodeLoad<KL>::kWords>& rr, const RowPtrs& p,
                                         bool valid, bool kin) {
  constexpr int KW = CodeLoad<KL>::kWords;
  if (valid && kin) {
    CodeLoad<KL>::load(p.pk, rr.code);
    rr.sv = (uint32_t)ldg_u16(p.sc) * 0x10001u;
    rr.ov = (uint32_t)ldg_u16(p.of) * 0x10001u;
  } else {
#pragma unroll
    for (int w = 0; w < KW; ++w) rr.code[w] = 0u;
    rr.sv = 0u;
    rr.ov = 0u;
  }
  rr.lv = valid ? (uint32_t)ldg_u16(p.lt) : 0u;
}

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// A block owns a contiguous range of weight rows (sized so that the grid is
// one wave).  Warp w handles the K-slices w, w + nwarps, ... of every row in
// the range: it keeps the loads of the next P rows in flight (a row's
// registers are refilled with the row P further on as soon as it has been
// consumed) across the whole range, and reduces the lane partials of every P
// rows with one transposed shuffle reduction.  Slice partials meet in shared
// memory and are summed in a fixed order.
//
// Programmatic dependent launch: the weight-side loads of the first P rows
// are issued before griddepcontrol.wait, x is read only after it, and y is
// written only after it.  (When the kernel is launched without the
// programmatic attribute the wait returns at once.)
template <int MT, int KL, int P>
__global__ void __launch_bounds__(kMaxWarps * 32) decode_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ y, float* __restrict__ y32, int M, int64_t N, int64_t K, int64_t G,
    int nslices, int rows_per_block) {
  constexpr int KW = CodeLoad<KL>::kWords;
  constexpr int V = P * MT;
  static_assert(V <= 32 && (V & (V - 1)) == 0, "P * MT must be a power of two <= 32");
  static_assert(P % 2 == 0 && KL % 8 == 0, "rows go to the tensor core in pairs");
  extern __shared__ float s_part[];  // [nwarps][RTP][MT]

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t groups = K / G;
  const int64_t row_bytes = K / 2;
  const int RT = rows_per_block;
  const int RTP = ((RT + P - 1) / P) * P;
  const int64_t nblocks = (N + RT - 1) / RT;
  const int my_idx = transpose_reduce_index<V>(lane);
  const bool writer = (lane & ((32 / V) - 1)) == 0;  // one lane per reduced value
  bool waited = false;

  for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const int64_t row0 = blk * RT;
    const int nrows = (int)((N - row0) < (int64_t)RT ? (N - row0) : (int64_t)RT);
    bool first_slice = true;
    for (int s = warp; s < nslices; s += nwarps) {
      const int64_t k0 = (int64_t)s * 32 * KL + (int64_t)lane * KL;
      const bool kin = k0 < K;
      const int64_t g = kin ? k0 / G : 0;
      RowPtrs nxt;  // the row after the ones in flight
      nxt.pk = packed + row0 * row_bytes + (kin ? k0 / 2 : 0);
      nxt.lt = lut + row0 * lut_row_stride + (lane & 15);
      nxt.sc = scale + row0 * groups + g;
      nxt.of = offset + row0 * groups + g;

      RowRegs<KW> buf[P];
#pragma unroll
      for (int j = 0; j < P; ++j) {
        load_row<KL>(buf[j], nxt, j < nrows, kin);
        nxt.pk += row_bytes;
        nxt.lt += lut_row_stride;
        nxt.sc += groups;
        nxt.of += groups;
      }
      if (!waited) {  // x (and y) may belong to the preceding kernel
        grid_dependency_wait();
        grid_dependents_launch();
        waited = true;
      }

      uint32_t xw[MT][KL / 2];  // activations of this chunk, bf16 pairs (even k low)
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

      for (int i = 0; i < RTP; i += P) {
        float part[V];
#pragma unroll
        for (int j = 0; j < P; j += 2) {
          // Rows j (A rows 0..7) and j + 1 (A rows 8..15) of this group on the
          // tensor core.  mma step st covers codes 4st .. 4st+3 of every lane's
          // chunk: lane (q = lane/4, t = lane%4) supplies A[q][2t, 2t+1, 2t+8,
          // 2t+9] = W'(its codes 4st..4st+3) of row j, A[q+8][same] = those of
          // row j+1, and B[2t, 2t+1, 2t+8, 2t+9][q] = x at the same four
          // columns.  Every product therefore pairs a weight with its own x,
          // and the diagonals C[q][q], C[q+8][q] (summed over q) are the two
          // rows' partial dot products; the other entries are not used.
          float c[MT][4];
#pragma unroll
          for (int m = 0; m < MT; ++m) c[m][0] = c[m][1] = c[m][2] = c[m][3] = 0.f;
          const bool va = i + j < nrows, vb = i + j + 1 < nrows;  // warp-uniform
          if (va || vb) {
#pragma unroll
            for (int st = 0; st < KL / 4; ++st) {
              const uint32_t ca = buf[j].code[st / 2] >> (16 * (st & 1));
              const uint32_t cb = buf[j + 1].code[st / 2] >> (16 * (st & 1));
              const uint32_t a01 = dequant_pair(buf[j].lv, ca, ca >> 4, buf[j].sv, buf[j].ov);
              const uint32_t a45 = dequant_pair(buf[j].lv, ca >> 8, ca >> 12, buf[j].sv, buf[j].ov);
              const uint32_t a23 =
                  dequant_pair(buf[j + 1].lv, cb, cb >> 4, buf[j + 1].sv, buf[j + 1].ov);
              const uint32_t a67 =
                  dequant_pair(buf[j + 1].lv, cb >> 8, cb >> 12, buf[j + 1].sv, buf[j + 1].ov);
#pragma unroll
              for (int m = 0; m < MT; ++m)
                mma_16816(c[m], a01, a23, a45, a67, xw[m][2 * st], xw[m][2 * st + 1]);
            }
          }
          const int q = lane >> 2;
          const bool diag = (lane & 3) == (q >> 1);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float da = (q & 1) ? c[m][1] : c[m][0];
            const float db = (q & 1) ? c[m][3] : c[m][2];
            part[j * MT + m] = diag ? da : 0.f;
            part[(j + 1) * MT + m] = diag ? db : 0.f;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (i + j + h + P < nrows) {  // refill with the row P further on
              load_row<KL>(buf[j + h], nxt, true, kin);
              nxt.pk += row_bytes;
              nxt.lt += lut_row_stride;
              nxt.sc += groups;
              nxt.of += groups;
            }
          }
        }
        const float tot = transpose_reduce<V>(part, lane);
        if (writer) {
          const int r = i + my_idx / MT;
          const int m = my_idx % MT;
          float* dst = s_part + ((size_t)warp * RTP + r) * MT + m;
          *dst = first_slice ? tot : *dst + tot;
        }
      }
      first_slice = false;
    }
    __syncthreads();
    const int nw_used = min(nwarps, nslices);
    for (int t = threadIdx.x; t < nrows * MT; t += blockDim.x) {
      const int r = t / MT;
      const int m = t % MT;
      if (m < M) {
        float tot = 0.f;
        for (int w = 0; w < nw_used; ++w) tot += s_part[((size_t)w * RTP + r) * MT + m];
        if (y32 != nullptr)
          y32[(int64_t)m * N + row0 + r] = tot;
        else
          y[(int64_t)m * N + row0 + r] = f32_to_bf16_rn(tot);
      }
    }
    __syncthreads();
  }
  if (!waited) {
    grid_dependency_wait();
    grid_dependents_launch();
  }
}

template <int MT, int KL, int P>
any4_status run(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                uint16_t* y, float* y32, int M, int64_t N, int64_t K, int64_t G, bool overlap,
                cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t slice = 32LL * KL;
  const int nslices = (int)((K + slice - 1) / slice);
  // the fewest warps that keep every warp's share of slices equal (<= 8)
  const int per_warp = (nslices + kMaxWarps - 1) / kMaxWarps;
  const int nwarps = (nslices + per_warp - 1) / per_warp;
  const int threads = nwarps * 32;
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(decode_kernel<MT, KL, P>), threads,
                                (size_t)kMaxRowsMT * sizeof(float) * nwarps);
  if (per_sm < 1) per_sm = 1;
  // one wave: every resident block owns an equal contiguous range of rows
  const int64_t wave = (int64_t)dev.sm_count * per_sm;
  int64_t rt = (N + wave - 1) / wave;
  rt = std::min<int64_t>(rt, kMaxRowsMT / MT);
  const int64_t rtp = ((rt + P - 1) / P) * P;
  const int64_t nblocks = (N + rt - 1) / rt;
  const int grid = (int)std::min<int64_t>(nblocks, wave);
  const size_t smem = (size_t)nwarps * rtp * MT * sizeof(float);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, decode_kernel<MT, KL, P>, x, packed, lut,
                                             lut_row_stride, scale, offset, y, y32, M, N, K,
                                             G, nslices, (int)rt);
  return err == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

any4_status launch_decode(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                          void* workspace, size_t workspace_bytes, bool overlap, bool pair_at_m1,
                          int32_t* dev_status, bool test_stall, cudaStream_t stream,
                          const DeviceInfo& dev) {
  // The kernel measured fastest for each M on B200 where several apply:
  //   M = 1  the weight-streaming shuffle kernel (decode_tma.cu), unless the
  //          caller asks for the pair-table kernel;
  //   M = 2  the pair-table kernel (decode_pair.cu), stream-K over 64-row
  //          sets, when the caller passes its workspace.
  const size_t pair_ws = decode_pair_workspace_size(M, N, K, G, dev);
  const bool pair_ok = pair_ws > 0 && workspace != nullptr && workspace_bytes >= pair_ws;
  const bool tma_ok = decode_tma_supported(M, N, K, G);
  if (pair_ok && (M == 2 || pair_at_m1 || !tma_ok))
    return launch_decode_pair(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                              workspace, overlap, dev_status, test_stall, stream, dev);
  // M = 1 with a 1024-column slice holding whole 16-byte runs of scales:
  // weights streamed by the tensor-memory-access engine
  if (tma_ok)
    return launch_decode_tma(x, packed, lut, lut_row_stride, scale, offset, y, y32, N, K, G,
                             overlap, dev_status, test_stall, stream, dev);
  // M >= 2: the skinny kernel (one dequantisation of the weights for all rows
  // of x, standard tensor-core mapping; skinny.cu)
  if (M >= 2)
    return launch_skinny(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                         overlap, stream, dev);
  return run<1, 32, 8>(x, packed, lut, lut_row_stride, scale, offset, y, y32, 1, N, K, G, overlap,
                       stream, dev);
}

}  // namespace any4
