// Skinny any4 matmul, 2 <= M <= 16: y[m][n] = sum_k x[m][k] * W[n][k].
//
// Paper "any4: Learned 4-bit Numeric Representation for LLMs", §4.1 Eq. 8,
// §2.5.2 (dequant), §4.2 (weights dequantised on the fly, memory-bound at
// small batch).  W' = LUT[c] * scale + offset rounded once to bf16 (bf16x2
// fused multiply-add), fp32 accumulation, bf16 output.
//
// Once M > 1 the decode kernels' diagonal tensor-core mapping needs one MMA
// per row of x, so this kernel uses the plain m16n8k16 mapping instead, with
// the dequantised weights as the B operand: A = x (up to 16 rows of x per
// MMA), B = W^T (8 weight rows x 16 columns).  Every lane owns one weight row
// of an 8-row group (lane / 4) and 32 consecutive codes of it per 128-column
// chunk (lane % 4 picks the 32); the MMA's k positions are mapped onto those
// columns (position 2q + j <-> column 4s + j of lane q's 32, position
// 2q + 8 + j <-> column 4s + 2 + j, for step s), and x is laid out the same
// way, so the contraction is unchanged.  Each lane holds its row's 16-entry
// table in registers as byte planes and looks codes up with byte permutes
// (lookup8), so the dequantisation cost per weight does not depend on M.
//
// Work split: a block owns a contiguous range of 8-row groups (balanced over
// the grid); its warps split K into slices of 128 * KC columns; each warp
// keeps x for its slice in registers, walks the row groups (loads of the next
// group in flight while the current one is computed) and adds its partial
// sums into shared memory; the block then sums the warps' partials in a fixed
// order and writes y.  No atomics: bitwise deterministic.
#include <algorithm>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kSkWarps = 8;

__device__ __forceinline__ void mma_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kSkStages = 4;  // ring stages per warp (8-row groups in flight)

// Asynchronous global -> shared copies (16 or 4 bytes); src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src),
               "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src),
               "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

// One ring stage (one 8-row group of a warp's slice), in shared memory:
//   codes  [KC][32 lanes][16 bytes]   each lane's 32 codes of each chunk
//   table  [8 rows][4 lanes][16 bytes]  the rows' 16-entry tables (the
//                                     first two 16-byte slots of a row)
//   so     [8 rows][KC][4 lanes][2][4 bytes]  per lane and chunk: the aligned
//                                     4-byte words holding the scale, then the
//                                     offset, of the lane's group
template <int KC>
struct SkStage {
  static constexpr int kCodes = 0;
  static constexpr int kTable = KC * 512;
  static constexpr int kSo = kTable + 512;
  static constexpr int kBytes = kSo + 8 * KC * 4 * 8;
};

// MT: rows of x covered (8 or 16; HI = whether the upper 8 rows of the MMA's
// 16 are used); KC: 128-column chunks per slice.
template <int MT, int KC>
__global__ void __launch_bounds__(kSkWarps * 32, 2) skinny_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride, const uint16_t* __restrict__ scale,
    const uint16_t* __restrict__ offset, uint16_t* __restrict__ y, int M, int N, int K, int G,
    int groups8, int nslices, int rows_max) {
  constexpr int MB = MT > 16 ? 2 : 1;
  constexpr int NA = MB == 1 ? 4 : 2;
  constexpr bool HI = MT > 8;
  // dynamic shared memory: [nwarps][kSkStages] ring stages, then the partial
  // sums [nwarps][rows_max][M]
  extern __shared__ __align__(16) uint8_t sk_smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int nw_used = nwarps < nslices ? nwarps : nslices;
  const int g0 = (int)((int64_t)groups8 * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)groups8 * (blockIdx.x + 1) / gridDim.x);
  const int q = lane & 3;        // which 32 columns of a chunk
  const int r = lane >> 2;       // weight row within the group; x row within a 16-row block
  const int64_t row_bytes = K / 2;
  const int groups = K / G;
  const int64_t so_elems = (int64_t)N * groups;  // elements of scale (and of offset)
  constexpr int kSliceCols = 128 * KC;
  const bool shared_lut = lut_row_stride == 0;
  const int ring_bytes = kSkStages * SkStage<KC>::kBytes;
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(sk_smem) + (uint32_t)(warp * ring_bytes);
  const uint8_t* ring_g = sk_smem + warp * ring_bytes;
  float* s_part = reinterpret_cast<float*>(sk_smem + nwarps * ring_bytes);

  uint32_t tls[4] = {0u, 0u, 0u, 0u}, ths[4] = {0u, 0u, 0u, 0u};
  if (shared_lut) table_planes(ldg_nc_v4(lut), ldg_nc_v4(lut + 8), tls, ths);

  if (warp >= nslices) {  // no slice for this warp (not reached: nwarps <= nslices)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  bool first_slice = true;
  for (int s = warp; s < nslices; s += nwarps) {
    // Per-slice constants of this lane: its column in each chunk, whether it
    // lies inside K, and its group index along the row.
    int colq[KC], gq[KC];
    bool inq[KC], lastq[KC];
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      colq[c] = s * kSliceCols + c * 128 + 32 * q;
      inq[c] = colq[c] < K;
      gq[c] = inq[c] ? colq[c] / G : 0;
      // the row's last group at an even flat index ends the scale/offset
      // tensors when N * groups is odd (checked per row below)
      lastq[c] = inq[c] && gq[c] == groups - 1 && (so_elems & 1);
    }

    // Issue the copies of group g into ring stage st: lane (r, q) copies its
    // codes of each chunk, its half (q < 2) of row r's table (lanes q >= 2
    // zero-fill spare slots, so that the instruction is uniform), and the
    // aligned 4-byte words holding its groups' scale and offset.
    auto issue_group = [&](int g, int st) {
      const uint32_t sb = ring + (uint32_t)(st * SkStage<KC>::kBytes);
      const int n = g * 8 + r;
      const bool rin = n < N;
      const int nc = rin ? n : 0;
      const uint8_t* prow = packed + (int64_t)nc * row_bytes;
      const int64_t srow = (int64_t)nc * groups;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const bool in = rin && inq[c];
        cp_async16(sb + SkStage<KC>::kCodes + (uint32_t)((c * 32 + lane) * 16),
                   prow + (in ? colq[c] / 2 : 0), in ? 16u : 0u);
      }
      if (!shared_lut)
        cp_async16(sb + SkStage<KC>::kTable + (uint32_t)(lane * 16),
                   lut + (int64_t)nc * lut_row_stride + 8 * (q & 1), (rin && q < 2) ? 16u : 0u);
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const bool in = rin && inq[c];
        const int64_t gi = srow + gq[c];
        const uint32_t dst = sb + SkStage<KC>::kSo + (uint32_t)(((r * KC + c) * 4 + q) * 8);
        if (lastq[c] && n == N - 1) {
          // the aligned pair would run past the tensors' end: the last group
          // (even flat index, low half) by plain loads instead
          const uint32_t sv = ldg_u16(scale + gi), ov = ldg_u16(offset + gi);
          asm volatile("st.shared.v2.u32 [%0], {%1, %2};" :: "r"(dst), "r"(sv), "r"(ov) : "memory");
        } else {
          cp_async4(dst, scale + (gi & ~(int64_t)1), in ? 4u : 0u);
          cp_async4(dst + 4, offset + (gi & ~(int64_t)1), in ? 4u : 0u);
        }
      }
    };

    // prologue: the first kSkStages - 1 groups in flight (empty commit groups
    // past the end keep the group count uniform)
#pragma unroll
    for (int i = 0; i < kSkStages - 1; ++i) {
      if (g0 + i < g1) issue_group(g0 + i, i);
      cp_async_commit();
    }
    if (first_slice) {
      // x (and y) may belong to the kernel before this one on the stream
      // (programmatic dependent launch); the weight copies above may run ahead
      asm volatile("griddepcontrol.wait;" ::: "memory");
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    // x for this slice: rows 16 mb + r and 16 mb + r + 8, the lane's 32
    // columns of each chunk, as bf16 pairs
    uint32_t xa[MB][KC][16], xb[MB][KC][16];  // xb: rows + 8 (zero unless HI)
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const int col = s * kSliceCols + c * 128 + 32 * q;
        const int ma = 16 * mb + r, mbr = ma + 8;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 a = (ma < M && col < K) ? ldg_nc_v4(x + (int64_t)ma * K + col + 8 * v)
                                              : make_uint4(0u, 0u, 0u, 0u);
          const uint4 b = (HI && mbr < M && col < K)
                              ? ldg_nc_v4(x + (int64_t)mbr * K + col + 8 * v)
                              : make_uint4(0u, 0u, 0u, 0u);
          xa[mb][c][4 * v] = a.x; xa[mb][c][4 * v + 1] = a.y;
          xa[mb][c][4 * v + 2] = a.z; xa[mb][c][4 * v + 3] = a.w;
          xb[mb][c][4 * v] = b.x; xb[mb][c][4 * v + 1] = b.y;
          xb[mb][c][4 * v + 2] = b.z; xb[mb][c][4 * v + 3] = b.w;
        }
      }
    }

    int st = 0, st_issue = kSkStages - 1;
    for (int g = g0; g < g1; ++g) {
      if (g + kSkStages - 1 < g1) issue_group(g + kSkStages - 1, st_issue);
      cp_async_commit();
      st_issue = st_issue + 1 == kSkStages ? 0 : st_issue + 1;
      cp_async_wait<kSkStages - 1>();
      __syncwarp();  // every lane's copies of group g have landed
      const uint8_t* sp = ring_g + st * SkStage<KC>::kBytes;
      st = st + 1 == kSkStages ? 0 : st + 1;
      // parity of the row's first flat scale index (which half of a copied word)
      const int n_row = g * 8 + r;
      const int par_row = (n_row & groups) & 1;
      uint32_t tl[4], th[4];
      if (shared_lut) {
#pragma unroll
        for (int i = 0; i < 4; ++i) { tl[i] = tls[i]; th[i] = ths[i]; }
      } else {
        const uint4* e = reinterpret_cast<const uint4*>(sp + SkStage<KC>::kTable + r * 64);
        table_planes(e[0], e[1], tl, th);
      }
      // NA independent accumulator sets (steps taken in turn), so that the
      // dependent-MMA chain of a group is NA times shorter
      float d[NA][MB][4];
#pragma unroll
      for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) d[a][mb][0] = d[a][mb][1] = d[a][mb][2] = d[a][mb][3] = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        // this chunk's group: its scale and offset sit in the half of the
        // copied 4-byte words given by the flat index's parity
        const uint2 sow =
            *reinterpret_cast<const uint2*>(sp + SkStage<KC>::kSo + ((r * KC + c) * 4 + q) * 8);
        const uint32_t sh = (uint32_t)((par_row ^ gq[c]) & 1) * 16u;
        const uint32_t s2 = ((sow.x >> sh) & 0xFFFFu) * 0x10001u;
        const uint32_t o2 = ((sow.y >> sh) & 0xFFFFu) * 0x10001u;
        const uint4 qv = *reinterpret_cast<const uint4*>(sp + SkStage<KC>::kCodes + (c * 32 + lane) * 16);
        const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          // codes 8t .. 8t + 7 of the lane's 32: W' pairs (8t, 8t+1) .. (8t+6, 8t+7)
          uint32_t w[4];
          lookup8(words[t], tl, th, w);
#pragma unroll
          for (int p = 0; p < 4; ++p) w[p] = hfma2_bf16(w[p], s2, o2);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int stp = 2 * t + h;  // mma step: columns 4 stp .. 4 stp + 3 of the lane's 32
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
              mma_m16n8k16(d[(c * 8 + stp) % NA][mb], xa[mb][c][2 * stp], xb[mb][c][2 * stp],
                           xa[mb][c][2 * stp + 1], xb[mb][c][2 * stp + 1], w[2 * h], w[2 * h + 1]);
          }
        }
      }
      __syncwarp();  // stage st may be refilled by the next iteration's copies
#pragma unroll
      for (int a = 1; a < NA; ++a)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
          for (int i = 0; i < 4; ++i) d[0][mb][i] += d[a][mb][i];
      // d[mb]: D[x row 16 mb + r (+8)][weight row 2q, 2q+1 of the group]
      {
        const int row0 = (g - g0) * 8 + 2 * q;
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
          const int ma = 16 * mb + r, mbr = ma + 8;
          float* base = s_part + (size_t)warp * rows_max * M;
          if (ma < M) {
            float* p0 = base + (size_t)row0 * M + ma;
            float* p1 = base + (size_t)(row0 + 1) * M + ma;
            *p0 = first_slice ? d[0][mb][0] : *p0 + d[0][mb][0];
            *p1 = first_slice ? d[0][mb][1] : *p1 + d[0][mb][1];
          }
          if (HI && mbr < M) {
            float* p0 = base + (size_t)row0 * M + mbr;
            float* p1 = base + (size_t)(row0 + 1) * M + mbr;
            *p0 = first_slice ? d[0][mb][2] : *p0 + d[0][mb][2];
            *p1 = first_slice ? d[0][mb][3] : *p1 + d[0][mb][3];
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncwarp();
    first_slice = false;
  }
  __syncthreads();
  // fixed-order sum over the warps' slices; y written row-contiguously per m
  const int rows = (g1 - g0) * 8;
  const int n0 = g0 * 8;
  for (int i = threadIdx.x; i < rows * M; i += blockDim.x) {
    const int m = i / rows, row = i - m * rows;
    if (n0 + row >= N) continue;
    float tot = 0.f;
    for (int w = 0; w < nw_used; ++w) tot += s_part[((size_t)w * rows_max + row) * M + m];
    y[(int64_t)m * N + n0 + row] = f32_to_bf16_rn(tot);
  }
}

template <int MT, int KC>
any4_status run_skinny(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                       int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                       uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t G, bool overlap,
                       cudaStream_t stream, const DeviceInfo& dev) {
  auto kern = skinny_kernel<MT, KC>;
  const int nslices = (int)((K + 128 * KC - 1) / (128 * KC));
  const int nwarps = std::min(kSkWarps, nslices);
  const int threads = nwarps * 32;
  const int64_t groups8 = (N + 7) / 8;
  // rows of partial sums that fit the shared memory beside the rings (a multiple of 8)
  const size_t smem_max = std::min<size_t>(dev.smem_optin, 227 * 1024);
  const size_t ring_total = (size_t)nwarps * kSkStages * SkStage<KC>::kBytes;
  if (ring_total >= smem_max) return ANY4_ERR_UNSUPPORTED;
  const int64_t rows_cap = std::min<int64_t>(
      512, (int64_t)((smem_max - ring_total) / ((size_t)nwarps * M * sizeof(float))) / 8 * 8);
  if (rows_cap < 8) return ANY4_ERR_UNSUPPORTED;
  int per_sm = 0;
  static bool attr_done = false;  // one per template instance
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) !=
        cudaSuccess)
      return ANY4_ERR_CUDA;
    attr_done = true;
  }
  // balanced 8-row-group ranges, one resident wave
  int64_t grid = 0, rows_max = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t slots = (int64_t)dev.sm_count * std::max(per_sm, 1);
    grid = std::min<int64_t>(groups8, slots);
    rows_max = ((groups8 + grid - 1) / grid) * 8;
    if (rows_max > rows_cap) {
      grid = (groups8 + rows_cap / 8 - 1) / (rows_cap / 8);
      rows_max = ((groups8 + grid - 1) / grid) * 8;
    }
    const size_t smem = ring_total + (size_t)nwarps * rows_max * M * sizeof(float);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess ||
        occ < 1)
      occ = 1;
    if (occ == per_sm) break;
    per_sm = occ;
  }
  const size_t smem = ring_total + (size_t)nwarps * rows_max * M * sizeof(float);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, x, packed, lut, lut_row_stride, scale,
                                             offset, y, (int)M, (int)N, (int)K, (int)G,
                                             (int)groups8, nslices, (int)rows_max);
  return err == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

any4_status launch_skinny(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t G, bool overlap,
                          cudaStream_t stream, const DeviceInfo& dev) {
  if (M < 1 || M > 16 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return ANY4_ERR_UNSUPPORTED;
  if (M <= 8)
    return run_skinny<8, 2>(x, packed, lut, lut_row_stride, scale, offset, y, M, N, K, G, overlap,
                            stream, dev);
  return run_skinny<16, 1>(x, packed, lut, lut_row_stride, scale, offset, y, M, N, K, G, overlap,
                           stream, dev);
}

}  // namespace any4
