// Learning the table of each row: the quantiser that produces the packed codes,
// tables, scales and offsets the matmul consumes.
//
// "any4: Learned 4-bit Numeric Representation for LLMs", for n-bit codes
// (§4.1 Eq. 9: 2^n table entries per row; n = 4 is any4, §5 evaluates any3
// and any2):
//   §2.5.1 Eq. 1-2   group-wise scaling: alpha = (max - min) / (2^n - 1),
//                    beta = min, scaled weight w_S = (w - beta) / alpha;
//   §4.1 Eq. 18      E-step: each scaled weight takes its nearest table entry;
//   §4.1 Eq. 23      M-step: an entry becomes the mean of its cluster's scaled
//                    weights, weighted by alpha_{i,j} * E|x_j|;
//   Appendix A.1     rows are independent (Alg. 1 runs k-means row by row).
//
// One thread block per row, the row held in shared memory.  Every floating-point
// step is one correctly rounded IEEE operation written with an explicit-rounding
// intrinsic (nothing is contracted into a fused multiply-add), taken in the order
// of a sequential loop, so the results are bit-identical to a plain sequential
// statement of the same steps:
//   - alpha = bf16(fp32(fp32(max - min) / (2^n - 1))), beta = min (exact in bf16);
//     w is read with -0 as +0;
//   - w_S = ((double)w - beta) / alpha in fp64, 0 in a group whose alpha is 0;
//   - initial table: entry q = the element at position
//     floor(q (K - 1) / (2^n - 1)) of the sorted row (a bitonic sort in
//     shared memory);
//   - E-step: nearest by |w_S - c_q| in fp64, ties to the lowest q;
//   - M-step: sample weight u_j = alpha_{g(j)} * E|x_j| (exact in fp64);
//     numerator sum(u_j * w_S_j) and denominator sum(u_j) over ascending j,
//     one lane per cluster adding both sums, so the rounding order is the
//     sequential one (the block first sorts each batch of columns' terms by
//     cluster, keeping the column order within a cluster); a cluster whose
//     weights sum to 0 keeps its entry;
//   - stop after max_iter M-steps, or when an E-step changes no code;
//   - LUT_q = bf16(fp32(c_q)); the codes are a final E-step against the stored
//     LUT, packed as one little-endian bit stream per row (code k in bits
//     [n k, n k + n); for n = 4 two per byte, even column in the low nibble).
#include <cstdint>

#include "common.cuh"

namespace any4 {
namespace {

// Threads per block (one block per row): 256, or 512 when the row's shared
// memory leaves room for one block per SM only (long rows), so that the one
// resident block has more warps to hide the M-step's add chains; the staging
// row is sized for the larger count.
constexpr int kQuantThreadsMax = 512;

// Shared-memory layout of one row (K columns, NG = K / G groups, P = the
// power of two >= K the sort runs over; cpt M-step columns per thread and
// batch, 2 where the row leaves room, else 1).
struct QuantSmem {
  size_t xs, ex, alpha, beta, cent, table, stage, cnt, off, code, total;
};

__host__ __device__ inline int64_t pow2_at_least(int64_t K) {
  int64_t p = 32;
  while (p < K) p <<= 1;
  return p;
}

__host__ __device__ inline QuantSmem quant_smem_layout(int64_t K, int64_t G, int cpt) {
  QuantSmem s;
  const int64_t NG = K / G;
  s.xs = 0;                                            // double [P]
  s.cent = s.xs + 8 * (size_t)pow2_at_least(K);        // double [16]
  s.table = s.cent + 8 * 16;                           // double [16]
  const size_t chunks = (size_t)cpt * (kQuantThreadsMax / 32);  // 32 columns each
  s.stage = s.table + 8 * 16;                          // double2 [32 chunks] (M-step)
  s.cnt = s.stage + 16 * 32 * chunks;                  // int [chunks][16] (M-step)
  s.off = s.cnt + 4 * 16 * chunks;                     // int [chunks][16]
  s.ex = s.off + 4 * 16 * chunks;                      // float [K]
  s.alpha = s.ex + 4 * (size_t)K;                      // float [NG]
  s.beta = s.alpha + 4 * (size_t)NG;                   // float [NG]
  s.code = s.beta + 4 * (size_t)NG;                    // uint8 [K]
  s.total = (s.code + (size_t)K + 15) & ~(size_t)15;
  return s;
}

// bf16 value with -0 read as +0 (x + 0 rounds -0 to +0 and leaves all else).
__device__ __forceinline__ float bf16_canon(uint16_t h) {
  return __fadd_rn(__uint_as_float((uint32_t)h << 16), 0.0f);
}

__device__ __forceinline__ double scaled_weight(float w, float alpha, float beta) {
  return alpha > 0.0f ? __ddiv_rn(__dsub_rn((double)w, (double)beta), (double)alpha) : 0.0;
}

// E-step over the row: nearest of the NQ entries of c (ties to the lowest
// index).  Returns (uniformly across the block) whether any code changed.
template <int NQ, int kQuantThreads>
__device__ __forceinline__ bool estep(const double* xs, int K, const double* c, uint8_t* code) {
  double cr[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) cr[q] = c[q];
  int changed = 0;
  for (int j = threadIdx.x; j < K; j += kQuantThreads) {
    const double x = xs[j];
    double best = fabs(__dsub_rn(x, cr[0]));
    int bq = 0;
#pragma unroll
    for (int q = 1; q < NQ; ++q) {
      const double d = fabs(__dsub_rn(x, cr[q]));
      if (d < best) {
        best = d;
        bq = q;
      }
    }
    if (code[j] != (uint8_t)bq) changed = 1;
    code[j] = (uint8_t)bq;
  }
  return __syncthreads_or(changed) != 0;
}

// NQ = 2^n table entries (4, 8 or 16); the packed row has n K / 8 bytes.
template <int NQ, int kQuantThreads, int kCPT>
__global__ void __launch_bounds__(kQuantThreads)
quantize_kernel(const uint16_t* __restrict__ w, const float* __restrict__ ex, int K, int G,
                int max_iter, uint8_t* __restrict__ packed, uint16_t* __restrict__ lut,
                uint16_t* __restrict__ scale, uint16_t* __restrict__ offset,
                int32_t* __restrict__ iters) {
  constexpr int kQuantWarps = kQuantThreads / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const QuantSmem L = quant_smem_layout(K, G, kCPT);
  double* xs = reinterpret_cast<double*>(smem + L.xs);
  double* cent = reinterpret_cast<double*>(smem + L.cent);
  double* table = reinterpret_cast<double*>(smem + L.table);
  float* ex_s = reinterpret_cast<float*>(smem + L.ex);
  float* alpha_s = reinterpret_cast<float*>(smem + L.alpha);
  float* beta_s = reinterpret_cast<float*>(smem + L.beta);
  uint8_t* code = smem + L.code;
  double2* stage = reinterpret_cast<double2*>(smem + L.stage);
  int* cnt = reinterpret_cast<int*>(smem + L.cnt);
  int* off = reinterpret_cast<int*>(smem + L.off);

  const int64_t n = blockIdx.x;
  const int NG = K / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint16_t* wrow = w + n * (int64_t)K;

  for (int j = tid; j < K; j += kQuantThreads) {
    ex_s[j] = ex[j];
    code[j] = 0;
  }
  for (int i = tid; i < kCPT * kQuantWarps * 16; i += kQuantThreads) cnt[i] = 0;

  // Eq. 1-2: one warp per group; min and max are exact, so their order is free.
  for (int g = warp; g < NG; g += kQuantWarps) {
    float mn = bf16_canon(wrow[g * G + lane]);
    float mx = mn;
    for (int j = g * G + 32 + lane; j < (g + 1) * G; j += 32) {
      const float v = bf16_canon(wrow[j]);
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(kFullMask, mn, s));
      mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, s));
    }
    if (lane == 0) {
      const uint16_t a = f32_to_bf16_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)(NQ - 1)));
      const uint16_t b = (uint16_t)(__float_as_uint(mn) >> 16);   // mn is a bf16 value
      scale[n * NG + g] = a;
      offset[n * NG + g] = b;
      alpha_s[g] = __uint_as_float((uint32_t)a << 16);
      beta_s[g] = mn;
    }
  }
  __syncthreads();

  // Initial table: quantiles of the sorted w_S (+inf pads the sort to P).
  const int P = (int)pow2_at_least(K);
  for (int j = tid; j < P; j += kQuantThreads)
    xs[j] = j < K ? scaled_weight(bf16_canon(wrow[j]), alpha_s[j / G], beta_s[j / G])
                  : __longlong_as_double(0x7ff0000000000000LL);
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < P; i += kQuantThreads) {
        const int l = i ^ jj;
        if (l > i) {
          const double a = xs[i], b = xs[l];
          if ((i & k) == 0 ? (a > b) : (a < b)) {
            xs[i] = b;
            xs[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid < NQ) cent[tid] = xs[(int)(((int64_t)tid * (K - 1)) / (NQ - 1))];
  __syncthreads();
  for (int j = tid; j < K; j += kQuantThreads)
    xs[j] = scaled_weight(bf16_canon(wrow[j]), alpha_s[j / G], beta_s[j / G]);
  __syncthreads();

  estep<NQ, kQuantThreads>(xs, K, cent, code);
  int it = 0;
  while (it < max_iter) {
    {
      // Eq. 23.  Cluster q's numerator sum(u_j * w_S_j) and denominator
      // sum(u_j) over ascending j, added by lane q of warp 0.  The columns go
      // one block-wide batch at a time (thread t: columns b0 + r T + t,
      // r < kCPT, T threads; chunk r W + w is warp w's r-th set of 32):
      //  1. each thread forms its column's two terms; within its warp (32
      //     consecutive columns) __match_any_sync gives the lanes of the same
      //     cluster, hence the thread's rank among them, and the first of
      //     them stores the warp's count for that cluster;
      //  2. lane q of warp 0 turns the counts into offsets (warps in order),
      //     the clusters' list bases by a scan over the lanes, and clears the
      //     counts for the next batch;
      //  3. each thread stores its terms at base[q] + offset[warp][q] + rank:
      //     the batch sorted by cluster, ascending column within a cluster;
      //  4. lane q of warp 0 adds its list front to back, the loads issued
      //     ahead of the adds, while the other warps start the next batch.
      // The adds are the sequential ones, in the same order.
      double acc_n = 0.0, acc_d = 0.0;
      int lbeg = 0, lend = 0;  // lane q < NQ of warp 0: its list in `stage`
      constexpr int kBatch = kCPT * kQuantThreads;
      for (int b0 = 0; b0 < K; b0 += kBatch) {
        int q[kCPT], rank[kCPT];
        double2 term[kCPT];
#pragma unroll
        for (int r = 0; r < kCPT; ++r) {
          const int jb = b0 + r * kQuantThreads + tid;  // chunk r * warps + warp
          q[r] = 0; rank[r] = 0; term[r] = make_double2(0.0, 0.0);
          if (jb < K) {  // whole warps: K % 32 == 0
            q[r] = code[jb];
            const double u = __dmul_rn((double)alpha_s[jb / G], (double)ex_s[jb]);
            term[r] = make_double2(__dmul_rn(u, xs[jb]), u);
            const uint32_t m = __match_any_sync(kFullMask, q[r]);
            rank[r] = __popc(m & ((1u << lane) - 1u));
            if (rank[r] == 0) cnt[(r * kQuantWarps + warp) * 16 + q[r]] = __popc(m);
          }
        }
        __syncthreads();
        if (warp == 0) {
          int run = 0;
          if (lane < NQ) {
            for (int c = 0; c < kCPT * kQuantWarps; ++c) {
              const int v = cnt[c * 16 + lane];
              off[c * 16 + lane] = run;
              cnt[c * 16 + lane] = 0;
              run += v;
            }
          }
          int base = run;
#pragma unroll
          for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(kFullMask, base, d);
            if (lane >= d) base += y;
          }
          base -= run;
          if (lane < NQ) {
            for (int c = 0; c < kCPT * kQuantWarps; ++c) off[c * 16 + lane] += base;
          }
          lbeg = base;
          lend = base + run;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kCPT; ++r) {
          const int jb = b0 + r * kQuantThreads + tid;
          if (jb < K) stage[off[(r * kQuantWarps + warp) * 16 + q[r]] + rank[r]] = term[r];
        }
        __syncthreads();
        if (warp == 0 && lane < NQ) {
          int i = lbeg;
          for (; i + 4 <= lend; i += 4) {
            const double2 v0 = stage[i], v1 = stage[i + 1], v2 = stage[i + 2], v3 = stage[i + 3];
            acc_n = __dadd_rn(__dadd_rn(__dadd_rn(__dadd_rn(acc_n, v0.x), v1.x), v2.x), v3.x);
            acc_d = __dadd_rn(__dadd_rn(__dadd_rn(__dadd_rn(acc_d, v0.y), v1.y), v2.y), v3.y);
          }
          for (; i < lend; ++i) {
            const double2 v = stage[i];
            acc_n = __dadd_rn(acc_n, v.x);
            acc_d = __dadd_rn(acc_d, v.y);
          }
        }
      }
      if (warp == 0 && lane < NQ && acc_d > 0.0) cent[lane] = __ddiv_rn(acc_n, acc_d);
    }
    __syncthreads();
    ++it;
    if (!estep<NQ, kQuantThreads>(xs, K, cent, code)) break;
  }

  if (tid < NQ) {
    const uint16_t b = f32_to_bf16_rn(__double2float_rn(cent[tid]));
    lut[n * NQ + tid] = b;
    table[tid] = (double)__uint_as_float((uint32_t)b << 16);
  }
  if (tid == 0 && iters) iters[n] = it;
  __syncthreads();
  estep<NQ, kQuantThreads>(xs, K, table, code);

  // Pack 32 codes (BITS words) per thread step; K % 32 == 0.
  constexpr int BITS = NQ == 16 ? 4 : (NQ == 8 ? 3 : 2);
  uint32_t* prow = reinterpret_cast<uint32_t*>(packed + n * (int64_t)(K / 8 * BITS));
  for (int c = tid; c < K / 32; c += kQuantThreads) {
    uint32_t v[BITS];
#pragma unroll
    for (int b = 0; b < BITS; ++b) v[b] = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint32_t cd = code[c * 32 + k];
      const int bit = BITS * k, w = bit >> 5, off = bit & 31;
      v[w] |= cd << off;
      if (off + BITS > 32) v[w + 1] |= cd >> (32 - off);
    }
    if constexpr (BITS == 4) {
      reinterpret_cast<uint4*>(prow)[c] = make_uint4(v[0], v[1], v[2], v[3]);
    } else if constexpr (BITS == 2) {
      reinterpret_cast<uint2*>(prow)[c] = make_uint2(v[0], v[1]);
    } else {
#pragma unroll
      for (int b = 0; b < BITS; ++b) prow[c * BITS + b] = v[b];
    }
  }
}

template <int NQ, int kCPT>
any4_status launch_quantize_cpt(const uint16_t* w, const float* ex, int64_t N, int64_t K,
                                int64_t G, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                                uint16_t* scale, uint16_t* offset, int32_t* iters, size_t smem,
                                cudaStream_t stream) {
  // long rows: one block fits per SM, give it 512 threads; else 256 threads
  // and several blocks (rows) per SM
  const bool wide = 2 * (smem + 1024) > (size_t)228 * 1024;
  const void* kern = wide ? reinterpret_cast<const void*>(quantize_kernel<NQ, 512, kCPT>)
                          : reinterpret_cast<const void*>(quantize_kernel<NQ, 256, kCPT>);
  if (ensure_dynamic_smem(kern, smem) != ANY4_OK) return ANY4_ERR_CUDA;
  if (wide)
    quantize_kernel<NQ, 512, kCPT><<<(unsigned)N, 512, smem, stream>>>(
        w, ex, (int)K, (int)G, (int)max_iter, packed, lut, scale, offset, iters);
  else
    quantize_kernel<NQ, 256, kCPT><<<(unsigned)N, 256, smem, stream>>>(
        w, ex, (int)K, (int)G, (int)max_iter, packed, lut, scale, offset, iters);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

// two M-step columns per thread and batch (half the batches and block
// barriers) where the row's shared memory leaves room, else one (and one for
// 2-bit codes, whose two-column form does not fit the 512-thread register
// budget without spills)
template <int NQ>
any4_status launch_quantize_nq(const uint16_t* w, const float* ex, int64_t N, int64_t K,
                               int64_t G, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                               uint16_t* scale, uint16_t* offset, int32_t* iters,
                               cudaStream_t stream, const DeviceInfo& dev) {
  const size_t smem2 = quant_smem_layout(K, G, 2).total;
  if (NQ >= 8 && smem2 <= dev.smem_optin)
    return launch_quantize_cpt<NQ, NQ >= 8 ? 2 : 1>(w, ex, N, K, G, max_iter, packed, lut, scale, offset,
                                      iters, smem2, stream);
  return launch_quantize_cpt<NQ, 1>(w, ex, N, K, G, max_iter, packed, lut, scale, offset, iters,
                                    quant_smem_layout(K, G, 1).total, stream);
}

}  // namespace

size_t quantize_smem_bytes(int64_t K, int64_t G) { return quant_smem_layout(K, G, 1).total; }

any4_status launch_quantize(const uint16_t* w, const float* ex, int64_t N, int64_t K, int64_t G,
                            int bits, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                            uint16_t* scale, uint16_t* offset, int32_t* iters,
                            cudaStream_t stream, const DeviceInfo& dev) {
  const size_t smem = quantize_smem_bytes(K, G);
  if (smem > dev.smem_optin) return ANY4_ERR_SHAPE;
  switch (bits) {
    case 4:
      return launch_quantize_nq<16>(w, ex, N, K, G, max_iter, packed, lut, scale, offset, iters,
                                    stream, dev);
    case 3:
      return launch_quantize_nq<8>(w, ex, N, K, G, max_iter, packed, lut, scale, offset, iters,
                                   stream, dev);
    case 2:
      return launch_quantize_nq<4>(w, ex, N, K, G, max_iter, packed, lut, scale, offset, iters,
                                   stream, dev);
    default:
      return ANY4_ERR_SHAPE;
  }
}

}  // namespace any4
