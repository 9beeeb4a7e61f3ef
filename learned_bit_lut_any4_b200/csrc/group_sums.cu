// any4_group_sums: the per-group activation sums (sm_100a)
//
//   xsum[m][g] = sum of x[m][k] over the columns k = g*G .. g*G+G-1
//
// the factor that multiplies the group offset beta when the product of Eq. 8
// (paper §4.1) is taken with the group-affine weights alpha*LUT[c] + beta of
// §2.5.2:  sum_k x (alpha LUT + beta) = alpha sum_k x LUT + beta xsum.
//
// HBM-bound (reads 2 M K bytes, writes 4 M K / G).  A warp owns a "unit": a
// run of whole groups of one row (at most 32, one per lane), up to 2048
// columns (8 KiB of loads in flight per warp: 8 x 16-byte loads per lane, 512 coalesced bytes per warp
// instruction).  Fixed summation order, so results are deterministic:
//   1. each 16-byte chunk (8 columns) is summed left to right in fp32;
//   2. a group's chunk partials are summed left to right in fp32 by one lane.
// Any order of G fp32 additions is within gamma_{G-1} * sum |x| of the exact
// sum (gamma_n = n u / (1 - n u), u = 2^-24), the bound the tests hold it to.
#include "common.cuh"

namespace any4 {
namespace {

constexpr int kGsWarps = 8;
constexpr int kGsThreads = kGsWarps * 32;
constexpr int kGsChunksPerLane = 8;                        // 16-byte chunks per lane per pass
constexpr int kGsPassChunks = 32 * kGsChunksPerLane;       // 256 chunks = 2048 columns
constexpr int kGsPassCols = kGsPassChunks * 8;

__device__ __forceinline__ float sum8_bf16(uint4 v) {
  // columns in ascending order: low half of .x first
  float s = bf16_lo_to_f32(v.x);
  s += bf16_lo_to_f32(v.x >> 16);
  s += bf16_lo_to_f32(v.y);
  s += bf16_lo_to_f32(v.y >> 16);
  s += bf16_lo_to_f32(v.z);
  s += bf16_lo_to_f32(v.z >> 16);
  s += bf16_lo_to_f32(v.w);
  s += bf16_lo_to_f32(v.w >> 16);
  return s;
}

// Groups per unit: as many whole groups as fit in one pass, at most one per
// lane (at least one; a group wider than a pass is walked in passes).
__host__ __device__ inline int64_t groups_per_unit(int64_t G) {
  return G >= kGsPassCols ? 1 : (kGsPassCols / G < 32 ? kGsPassCols / G : 32);
}

__global__ void __launch_bounds__(kGsThreads) group_sums_kernel(
    const uint16_t* __restrict__ x, float* __restrict__ xsum, int64_t M, int64_t K, int64_t G) {
  __shared__ float s_part[kGsWarps][kGsPassChunks];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t groups = K / G;
  const int64_t gpu_ = groups_per_unit(G);
  const int64_t units_per_row = (groups + gpu_ - 1) / gpu_;
  const int64_t units = M * units_per_row;
  const int chunks_per_group = (int)(G / 8);
  float* part = s_part[warp];
  for (int64_t u = (int64_t)blockIdx.x * kGsWarps + warp; u < units;
       u += (int64_t)gridDim.x * kGsWarps) {
    const int64_t m = u / units_per_row;
    const int64_t g0 = (u - m * units_per_row) * gpu_;
    const int ng = (int)(gpu_ < groups - g0 ? gpu_ : groups - g0);  // groups in this unit
    const uint16_t* row = x + m * K + g0 * G;
    const int64_t unit_chunks = (int64_t)ng * chunks_per_group;
    float acc = 0.f;                                         // lane j: group j's running sum
    for (int64_t c0 = 0; c0 < unit_chunks; c0 += kGsPassChunks) {
      const int64_t left = unit_chunks - c0;
      const int pass_chunks = left < kGsPassChunks ? (int)left : kGsPassChunks;
      uint4 v[kGsChunksPerLane];
#pragma unroll
      for (int i = 0; i < kGsChunksPerLane; ++i) {
        const int c = lane + 32 * i;
        v[i] = c < pass_chunks ? ldg_stream_v4(row + (c0 + c) * 8) : make_uint4(0, 0, 0, 0);
      }
      __syncwarp();  // the previous pass's partials have been read
#pragma unroll
      for (int i = 0; i < kGsChunksPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c < pass_chunks) part[c] = sum8_bf16(v[i]);
      }
      __syncwarp();
      // lane j adds the chunks of group j that lie in this pass, in order
      if (G >= kGsPassCols) {
        if (lane == 0)
          for (int c = 0; c < pass_chunks; ++c) acc += part[c];
      } else if (lane < ng) {
        const float* p = part + lane * chunks_per_group;
        for (int c = 0; c < chunks_per_group; ++c) acc += p[c];
      }
    }
    if (lane < ng) xsum[m * groups + g0 + lane] = acc;
  }
}

}  // namespace

any4_status launch_group_sums(const uint16_t* x, float* xsum, int64_t M, int64_t K, int64_t G,
                              cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t groups = K / G;
  const int64_t gpu_ = groups_per_unit(G);
  const int64_t units = M * ((groups + gpu_ - 1) / gpu_);
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(group_sums_kernel), kGsThreads, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t want = (units + kGsWarps - 1) / kGsWarps;
  const int64_t cap = (int64_t)dev.sm_count * per_sm;
  const int grid = (int)(want < cap ? want : cap);
  group_sums_kernel<<<grid, kGsThreads, 0, stream>>>(x, xsum, M, K, G);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
