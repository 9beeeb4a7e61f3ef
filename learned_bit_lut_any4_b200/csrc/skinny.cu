// Skinny any4 matmul, 2 <= M <= 16: y[m][n] = sum_k x[m][k] * W[n][k].
//
// Paper "any4: Learned 4-bit Numeric Representation for LLMs", §4.1 Eq. 8,
// §2.5.2 (dequant), §4.2 (weights dequantised on the fly, memory-bound at
// small batch).  W' = LUT[c] * scale + offset rounded once to bf16 (bf16x2
// fused multiply-add), fp32 accumulation, bf16 output.
//
// Once M > 1 the decode kernels' diagonal tensor-core mapping needs one MMA
// per row of x, so this kernel uses the plain m16n8k16 mapping: A = a 16-row
// tile of dequantised weights, B = x^T (up to 8 rows of x per MMA; two MMAs for
// M <= 16), so each weight is dequantised once for all rows of x.  Lane l owns
// weight rows l/4 and l/4 + 8 of the tile and 32 consecutive codes of each per
// 128-column chunk (q = l % 4 picks the 32); the MMA's k positions are mapped
// onto those columns (position 2q + j <-> column 4s + j of lane q's 32,
// position 2q + 8 + j <-> column 4s + 2 + j, for step s) and x is read with the
// same map, so the contraction is unchanged.  The two rows' dequantised pairs
// form the A operand directly and x's pairs the B operand, so no operand has
// to be moved into place.  Each lane holds its two rows' 16-entry tables as
// byte planes in registers and looks codes up with byte permutes (lookup8).
//
// Work split: a block owns a contiguous range of 8-row groups (balanced over
// the grid), processed as 16-row tiles (the last may be half empty); its warps
// split K into slices of 128 * KC columns; each warp keeps x for its slice in
// registers, streams the tiles' codes, tables and scales through a per-warp
// ring of asynchronous copies, and adds its partial sums into shared memory;
// the block then sums the warps' partials in a fixed order and writes y.  No
// atomics: bitwise deterministic.
#include <algorithm>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kSkWarps = 8;
constexpr int kSkStages = 3;  // ring stages per warp (16-row tiles in flight)

__device__ __forceinline__ void mma_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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

// One ring stage (one 16-row tile of a warp's slice), in shared memory:
//   codes  [KC][2 halves][32 lanes][16 bytes]  each lane's 32 codes of rows
//                                     l/4 (half 0) and l/4 + 8 (half 1) per chunk
//   table  [16 rows][32 bytes]        the tile rows' 16-entry tables
//   so     [KC][2 halves][32 lanes][2][4 bytes]  per lane, chunk and row: the
//                                     aligned 4-byte words holding the scale,
//                                     then the offset, of the lane's group; or,
//                                     when the slice's groups fit one aligned
//                                     8-group window, [16 rows][2][16 bytes]:
//                                     that window of each row's scales, offsets
template <int KC>
struct SkStage {
  static constexpr int kCodes = 0;
  static constexpr int kTable = KC * 1024;
  static constexpr int kSo = kTable + 512;
  static constexpr int kBytes = kSo + KC * 512;
};

// MT: rows of x covered (8 or 16: one or two MMAs per step); KC: 128-column
// chunks per slice.
template <int MT, int KC>
__global__ void __launch_bounds__(kSkWarps * 32, 2) skinny_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride, const uint16_t* __restrict__ scale,
    const uint16_t* __restrict__ offset, uint16_t* __restrict__ y, float* __restrict__ y32,
    int M, int N, int K, int G, int groups8, int nslices, int rows_max) {
  constexpr int MB = MT / 8;  // 8-row blocks of x (one MMA each per step)
  constexpr int NA = 2;       // accumulator sets (even / odd steps)
  // dynamic shared memory: [nwarps][kSkStages] ring stages, then the partial
  // sums [nwarps][rows_max][M]
  extern __shared__ __align__(16) uint8_t sk_smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int nw_used = nwarps < nslices ? nwarps : nslices;
  const int g0 = (int)((int64_t)groups8 * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)groups8 * (blockIdx.x + 1) / gridDim.x);
  const int ngroups = g1 - g0;            // 8-row groups of this block
  const int ntiles = (ngroups + 1) / 2;   // 16-row tiles (the last may be half empty)
  const int n_base = g0 * 8;
  const int q = lane & 3;   // which 32 columns of a chunk
  const int r = lane >> 2;  // weight rows r and r + 8 of a tile; x row of the B operand
  const int64_t row_bytes = K / 2;
  const int groups = K / G;
  const int64_t so_elems = (int64_t)N * groups;  // elements of scale (and of offset)
  const bool so_vec = (groups & 7) == 0 && (G & (G - 1)) == 0;
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
    // The slice's groups lie in one aligned window of 8 groups (16 bytes of a
    // scale or offset row) when G is a power of two and every row holds a
    // multiple of 8 groups: then a tile's scales and offsets are 32 such
    // windows, one 16-byte copy per lane.
    const int win = ((s * kSliceCols) / G) & ~7;
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

    // Issue the copies of tile t into ring stage st: lane (r, q) copies its
    // codes of rows r and r + 8 for each chunk, one 16-byte half of one row's
    // table (q < 2: row r, else row r + 8), and the aligned 4-byte words
    // holding its groups' scale and offset.
    auto issue_tile = [&](int t, int st) {
      const uint32_t sb = ring + (uint32_t)(st * SkStage<KC>::kBytes);
      const bool upper = 2 * t + 1 < ngroups;  // rows r + 8 belong to this block
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n_base + 16 * t + r + 8 * h;
        const bool rin = n < N && (h == 0 || upper);
        const int nc = rin ? n : 0;
        const uint8_t* prow = packed + (int64_t)nc * row_bytes;
        const int64_t srow = (int64_t)nc * groups;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          const bool in = rin && inq[c];
          cp_async16(sb + SkStage<KC>::kCodes + (uint32_t)(((c * 2 + h) * 32 + lane) * 16),
                     prow + (in ? colq[c] / 2 : 0), in ? 16u : 0u);
          if (so_vec) continue;  // scales and offsets come as whole windows below
          const int64_t gi = srow + gq[c];
          const uint32_t dst = sb + SkStage<KC>::kSo + (uint32_t)(((c * 2 + h) * 32 + lane) * 8);
          if (lastq[c] && n == N - 1) {
            // the aligned pair would run past the tensors' end: the last group
            // (even flat index, low half) by plain loads instead
            const uint32_t sv = ldg_u16(scale + gi), ov = ldg_u16(offset + gi);
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" :: "r"(dst), "r"(sv), "r"(ov)
                         : "memory");
          } else {
            cp_async4(dst, scale + (gi & ~(int64_t)1), in ? 4u : 0u);
            cp_async4(dst + 4, offset + (gi & ~(int64_t)1), in ? 4u : 0u);
          }
        }
      }
      if (so_vec) {
        // lane l: the 16-byte window (8 groups from `win`) of row l & 15 of the
        // scales (l < 16) or the offsets (l >= 16)
        const int i = lane & 15, tsr = lane >> 4;
        const int n = n_base + 16 * t + i;
        const bool rin = n < N && (i < 8 || upper);
        cp_async16(sb + SkStage<KC>::kSo + (uint32_t)((i * 2 + tsr) * 16),
                   (tsr ? offset : scale) + (int64_t)(rin ? n : 0) * groups + win, rin ? 16u : 0u);
      }
      if (!shared_lut) {
        const int trow = (q < 2 ? r : r + 8);
        const int n = n_base + 16 * t + trow;
        const bool rin = n < N && (q < 2 || upper);
        cp_async16(sb + SkStage<KC>::kTable + (uint32_t)(trow * 32 + (q & 1) * 16),
                   lut + (int64_t)(rin ? n : 0) * lut_row_stride + 8 * (q & 1), rin ? 16u : 0u);
      }
    };

    // prologue: the first kSkStages - 1 tiles in flight (empty commit groups
    // past the end keep the group count uniform)
#pragma unroll
    for (int i = 0; i < kSkStages - 1; ++i) {
      if (i < ntiles) issue_tile(i, i);
      cp_async_commit();
    }
    if (first_slice) {
      // x (and y) may belong to the kernel before this one on the stream
      // (programmatic dependent launch); the weight copies above may run ahead
      asm volatile("griddepcontrol.wait;" ::: "memory");
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    // x for this slice as the B operand: rows 8 mb + r, the lane's 32 columns
    // of each chunk, as bf16 pairs
    uint32_t xw[MB][KC][16];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
      const int m = 8 * mb + r;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 a = (m < M && inq[c]) ? ldg_nc_v4(x + (int64_t)m * K + colq[c] + 8 * v)
                                            : make_uint4(0u, 0u, 0u, 0u);
          xw[mb][c][4 * v] = a.x; xw[mb][c][4 * v + 1] = a.y;
          xw[mb][c][4 * v + 2] = a.z; xw[mb][c][4 * v + 3] = a.w;
        }
      }
    }

    int st = 0, st_issue = kSkStages - 1;
    for (int t = 0; t < ntiles; ++t) {
      if (t + kSkStages - 1 < ntiles) issue_tile(t + kSkStages - 1, st_issue);
      cp_async_commit();
      st_issue = st_issue + 1 == kSkStages ? 0 : st_issue + 1;
      cp_async_wait<kSkStages - 1>();
      __syncwarp();  // every lane's copies of tile t have landed
      const uint8_t* sp = ring_g + st * SkStage<KC>::kBytes;
      st = st + 1 == kSkStages ? 0 : st + 1;
      const bool upper = 2 * t + 1 < ngroups;  // warp-uniform
      // parity of each row's first flat scale index (which half of a copied word)
      const int nA = n_base + 16 * t + r;
      const int parA = (nA & groups) & 1, parB = ((nA + 8) & groups) & 1;
      uint32_t tlA[4], thA[4], tlB[4], thB[4];
      if (shared_lut) {
#pragma unroll
        for (int i = 0; i < 4; ++i) { tlA[i] = tlB[i] = tls[i]; thA[i] = thB[i] = ths[i]; }
      } else {
        const uint4* ea = reinterpret_cast<const uint4*>(sp + SkStage<KC>::kTable + r * 32);
        const uint4* eb = reinterpret_cast<const uint4*>(sp + SkStage<KC>::kTable + (r + 8) * 32);
        table_planes(ea[0], ea[1], tlA, thA);
        table_planes(eb[0], eb[1], tlB, thB);
      }
      float d[NA][MB][4];
#pragma unroll
      for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) d[a][mb][0] = d[a][mb][1] = d[a][mb][2] = d[a][mb][3] = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        // the rows' group scale and offset sit in the half of the copied
        // 4-byte words given by the flat index's parity
        uint32_t sA, oA, sB, oB;
        if (so_vec) {
          const uint16_t* wv = reinterpret_cast<const uint16_t*>(sp + SkStage<KC>::kSo);
          const int gw = inq[c] ? gq[c] - win : 0;  // group within the window
          sA = (uint32_t)wv[(r * 2 + 0) * 8 + gw] * 0x10001u;
          oA = (uint32_t)wv[(r * 2 + 1) * 8 + gw] * 0x10001u;
          sB = (uint32_t)wv[((r + 8) * 2 + 0) * 8 + gw] * 0x10001u;
          oB = (uint32_t)wv[((r + 8) * 2 + 1) * 8 + gw] * 0x10001u;
        } else {
          const uint2 swA = *reinterpret_cast<const uint2*>(
              sp + SkStage<KC>::kSo + ((c * 2 + 0) * 32 + lane) * 8);
          const uint2 swB = *reinterpret_cast<const uint2*>(
              sp + SkStage<KC>::kSo + ((c * 2 + 1) * 32 + lane) * 8);
          const uint32_t shA = (uint32_t)((parA ^ gq[c]) & 1) * 16u;
          const uint32_t shB = (uint32_t)((parB ^ gq[c]) & 1) * 16u;
          sA = ((swA.x >> shA) & 0xFFFFu) * 0x10001u;
          oA = ((swA.y >> shA) & 0xFFFFu) * 0x10001u;
          sB = ((swB.x >> shB) & 0xFFFFu) * 0x10001u;
          oB = ((swB.y >> shB) & 0xFFFFu) * 0x10001u;
        }
        const uint4 qa =
            *reinterpret_cast<const uint4*>(sp + SkStage<KC>::kCodes + ((c * 2 + 0) * 32 + lane) * 16);
        const uint4 qb =
            *reinterpret_cast<const uint4*>(sp + SkStage<KC>::kCodes + ((c * 2 + 1) * 32 + lane) * 16);
        const uint32_t wa4[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb4[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          // codes 8w .. 8w + 7 of the lane's 32, both rows: W' pairs
          // (8w, 8w+1) .. (8w+6, 8w+7)
          uint32_t pa[4], pb[4] = {0u, 0u, 0u, 0u};
          lookup8(wa4[w], tlA, thA, pa);
#pragma unroll
          for (int p = 0; p < 4; ++p) pa[p] = hfma2_bf16(pa[p], sA, oA);
          if (upper) {
            lookup8(wb4[w], tlB, thB, pb);
#pragma unroll
            for (int p = 0; p < 4; ++p) pb[p] = hfma2_bf16(pb[p], sB, oB);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int stp = 2 * w + h;  // mma step: columns 4 stp .. 4 stp + 3 of the lane's 32
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
              mma_m16n8k16(d[h][mb], pa[2 * h], pb[2 * h], pa[2 * h + 1], pb[2 * h + 1],
                           xw[mb][c][2 * stp], xw[mb][c][2 * stp + 1]);
          }
        }
      }
      __syncwarp();  // stage may be refilled by the next iteration's copies
      // d[.][mb]: D[weight row r (+8)][x row 8 mb + 2q, 2q + 1]
      const int rowA = 16 * t + r, rowB = rowA + 8;
      float* base = s_part + (size_t)warp * rows_max * M;
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const float v[4] = {d[0][mb][0] + d[1][mb][0], d[0][mb][1] + d[1][mb][1],
                            d[0][mb][2] + d[1][mb][2], d[0][mb][3] + d[1][mb][3]};
        const int m0 = 8 * mb + 2 * q;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = m0 + (i & 1);
          const int row = (i < 2) ? rowA : rowB;
          if (m < M && (i < 2 || upper)) {
            float* p = base + (size_t)row * M + m;
            *p = first_slice ? v[i] : *p + v[i];
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
  const int rows = ngroups * 8;
  for (int i = threadIdx.x; i < rows * M; i += blockDim.x) {
    const int m = i / rows, row = i - m * rows;
    if (n_base + row >= N) continue;
    float tot = 0.f;
    for (int w = 0; w < nw_used; ++w) tot += s_part[((size_t)w * rows_max + row) * M + m];
    if (y32 != nullptr)
      y32[(int64_t)m * N + n_base + row] = tot;
    else
      y[(int64_t)m * N + n_base + row] = f32_to_bf16_rn(tot);
  }
}

template <int MT, int KC>
any4_status run_skinny(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                       int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                       uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                       bool overlap, cudaStream_t stream, const DeviceInfo& dev) {
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
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem_max) != ANY4_OK)
    return ANY4_ERR_CUDA;
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
    int occ = cached_occupancy(reinterpret_cast<const void*>(kern), threads, smem);
    if (occ < 1) occ = 1;
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
                                             offset, y, y32, (int)M, (int)N, (int)K, (int)G,
                                             (int)groups8, nslices, (int)rows_max);
  return err == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

any4_status launch_skinny(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                          int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                          uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                          bool overlap, cudaStream_t stream, const DeviceInfo& dev) {
  if (M < 1 || M > 16 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return ANY4_ERR_UNSUPPORTED;
  if (M <= 8)
    return run_skinny<8, 2>(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                            overlap, stream, dev);
  return run_skinny<16, 1>(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                           overlap, stream, dev);
}

}  // namespace any4
