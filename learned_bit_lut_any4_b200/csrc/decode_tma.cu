// Decode-path any4 matmul at M = 1 with TMA-fed weight streaming.
//
// Paper "any4: Learned 4-bit Numeric Representation for LLMs", §4.1 Eq. 8,
// §2.5.2, §4.2: bf16 W = LUT[c] * scale + offset rounded once to bf16, table
// lookup by warp shuffle, fp32 accumulation.  Two kernels share the streaming
// design below: for G = 128 and 4-bit codes the table is folded with the
// group's scale and offset and the products go through packed fp32 FMAs
// (decode_tma_ffma_kernel); every other group size and code width forms
// W' per weight (one bf16x2 fused multiply-add per pair) and sums on the
// tensor core through the diagonal m16n8k16 mapping (decode_tma_kernel).
//
// What differs is how the weights reach the warps.  Each warp owns one
// 1024-column slice of K for the rows of its block and streams them through a
// private ring of S shared-memory stages; one lane issues, per stage of P rows,
// four cp.async.bulk.tensor.2d loads (packed codes viewed as u32 [N][K/8] with a
// 128 x P box = 512 bytes a row, the rows' tables [N][16], scales and offsets
// [N][K/G]), completed on an mbarrier.  The loads run as far ahead as the ring
// allows without holding registers, so the memory system always has
// S * P rows queued per warp while the lanes compute, and the block's register
// footprint stays small enough for several blocks per SM.  Rows past N and
// columns past K come back as zeros from the tensor loads.
//
// Waits on the ring are bounded (about 2 s of %globaltimer); on expiry the
// kernel sets ANY4_ERR_TIMEOUT in dev_status and every warp stops after
// waiting (bounded) for the copies it has in flight.
#include <cuda.h>

#include <algorithm>
#include <type_traits>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kTmaMaxWarps = 8;
constexpr int kTmaMaxGroup = ANY4_GROUP_MAX;
constexpr int kTmaRows = 8;      // P: rows per stage
constexpr int kTmaStages = 2;    // S: stages per warp (2 keeps two blocks per SM)

constexpr unsigned long long kTmaWaitNs = 2000000000ull;
constexpr unsigned long long kTmaTestWaitNs = 1000000ull;  // the test-stall mode's limit

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init_(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_test_(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit) {
  if (mbar_test_(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_test_(bar, parity)) return true;
    if ((i & 63u) == 0u && gtimer() - t0 > limit) return false;
  }
}
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                      uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(bar) : "memory");
}

struct TmaMaps {
  CUtensorMap codes;   // u32 [N][K/8], box {128, P}
  CUtensorMap codes_head;  // the same, box {128, head_rows}
  CUtensorMap lut;     // bf16 [N][16], box {16, P}
  CUtensorMap scale;   // bf16 [N][K/G], box {1024/G, P}
  CUtensorMap offset;  // bf16 [N][K/G], box {1024/G, P}
};

// Up to kTmaMaxGroup matrices that multiply the same x (the q, k, v or gate,
// up projections of a layer) in one launch: their row blocks are numbered one
// after the other, block b of the launch belongs to the first matrix i with
// b < blk_end[i].  All share K and G.
struct TmaGroup {
  TmaMaps maps[kTmaMaxGroup];
  uint16_t* y[kTmaMaxGroup];
  float* y32[kTmaMaxGroup];
  const uint16_t* lut_shared[kTmaMaxGroup];  // one table for the matrix, or NULL
  int N[kTmaMaxGroup];
  int64_t blk_end[kTmaMaxGroup];
  int count;
  int head_rows;  // rows of a slice's first stage (folded-table kernel), 1..P
};

// D += A * B, m16n8k16 bf16 -> fp32 (legacy warp-level tensor-core MMA).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two weights of one row from the table held in the lanes (lane l: entry
// l & 15 as bf16 bits): both entries fetched by shuffle, paired into one
// bf16x2 (first code in the low half) and turned into W' = LUT * s + o by one
// bf16x2 fused multiply-add: the exact value rounded once to bf16, which is
// bf16(fmaf(LUT, s, o)) unless that fp32 fmaf is inexact and lands on a bf16
// rounding tie.  The shuffle reads only the low 5 bits of the code word.
__device__ __forceinline__ uint32_t dq_pair(uint32_t lut_lane, uint32_t c_lo, uint32_t c_hi,
                                           uint32_t s2, uint32_t o2) {
  uint32_t a, b, w;
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=r"(a) : "r"(lut_lane), "r"(c_lo));
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=r"(b) : "r"(lut_lane), "r"(c_hi));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(w) : "r"(__byte_perm(a, b, 0x5410)), "r"(s2), "r"(o2));
  return w;
}

// a bf16 value (bits) in both halves of a bf16x2
__device__ __forceinline__ uint32_t dup2(uint16_t h) { return (uint32_t)h * 0x10001u; }

// Sum 8 per-lane values over the warp; value i's total ends in the lanes
// whose bits 4, 3, 2 spell i (lanes 4i .. 4i+3 after the bit reversal below).
__device__ __forceinline__ float reduce8(float (&v)[8], int lane) {
  int n = 8;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (lane & off) != 0;
      const int half = n / 2;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
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

// The stage layout of one warp's ring: P rows of codes (BITS * 128 bytes a
// row: 1024 codes), the rows' tables (2^BITS bf16 each), scales, offsets.
template <int GPS, int BITS>
struct TmaStage {
  static constexpr int P = kTmaRows;
  static constexpr int kEntries = 1 << BITS;
  static constexpr int kCodeBytes = P * 128 * BITS;
  static constexpr int kLutBytes = P * kEntries * 2;
  static constexpr int kLutSlot = ((kLutBytes + 127) / 128) * 128;
  static constexpr int kGrpBytes = ((P * GPS * 2 + 127) / 128) * 128;
  static constexpr int kBytes = kCodeBytes + kLutSlot + 2 * kGrpBytes;
  static constexpr uint32_t kTx = kCodeBytes + kLutBytes + 2 * P * GPS * 2;
  static_assert(kBytes % 128 == 0, "stage alignment");
};

__device__ __forceinline__ void tma1d(uint32_t dst, const CUtensorMap* map, int c0, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2}], [%3];"
      :: "r"(dst), "l"(map), "r"(c0), "r"(bar) : "memory");
}

// Code j (0..31) of a lane's 32 codes held in BITS words (a little-endian
// bit stream), in the low bits of the result; the bits above it are the
// following codes, which the table shuffle ignores.
template <int BITS>
__device__ __forceinline__ uint32_t code_word(const uint32_t (&w)[BITS], int j) {
  const int bit = BITS * j, wi = bit >> 5, off = bit & 31;
  if (wi + 1 < BITS) return __funnelshift_r(w[wi], w[wi + 1], off);
  return w[wi] >> off;
}

template <int GPS, int BITS>  // groups per 1024-column slice (1024 / G), code width
__global__ void __maxnreg__(96) decode_tma_kernel(
    const __grid_constant__ TmaGroup grp, const uint16_t* __restrict__ x, int K, int nslices,
    int rows_per_block, int32_t* dev_status, int test_stall) {
  // test_stall: warp 0 of block 0 stops its weight stream after one stage,
  // so its next wait runs out (1 ms limit) and the kernel ends cleanly
  const unsigned long long wait_ns = test_stall ? kTmaTestWaitNs : kTmaWaitNs;
  using St = TmaStage<GPS, BITS>;
  constexpr int P = St::P;
  constexpr int S = kTmaStages;
  constexpr int NE = St::kEntries;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int RT = rows_per_block;
  const int RTP = ((RT + P - 1) / P) * P;
  // layout: [rings: nwarps * S * St::kBytes][bars: nwarps * S * 8][partials]
  const uint32_t base = (smem_addr(smem_raw) + 127u) & ~127u;
  uint8_t* gbase = smem_raw + (base - smem_addr(smem_raw));
  const uint32_t ring = base + (uint32_t)(warp * S * St::kBytes);
  const uint8_t* gring = gbase + warp * S * St::kBytes;
  const uint32_t bars = base + (uint32_t)(nwarps * S * St::kBytes) + (uint32_t)(warp * S * 8);
  float* s_part =
      reinterpret_cast<float*>(gbase + nwarps * S * St::kBytes + nwarps * S * 8 + 16);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + nwarps * S * St::kBytes +
                                                          nwarps * S * 8);
  if (threadIdx.x == 0) *s_abort = 0;

  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init_(bars + 8u * st, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // barriers and the abort flag are initialised

  const int64_t nblocks = grp.blk_end[grp.count - 1];
  uint32_t it_issue = 0, it_use = 0;  // ring positions (issue and consumption order)
  bool waited = false, ok = true;
  const int gsub = (lane * 32) / (1024 / GPS);  // this lane's group within the slice

  // Every warp runs the same block loop and reaches the same __syncthreads;
  // a warp whose wait gave up only stops computing (ok = false) and raises
  // the block-wide flag so that no result of the block is written.
  for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    int mi = 0;  // the matrix of this row block
    while (mi + 1 < grp.count && blk >= grp.blk_end[mi]) ++mi;
    const TmaMaps& maps = grp.maps[mi];
    const int N = grp.N[mi];
    const uint16_t* lut_shared = grp.lut_shared[mi];
    const int row0 = (int)((blk - (mi > 0 ? grp.blk_end[mi - 1] : 0)) * RT);
    const int nrows = (N - row0) < RT ? (N - row0) : RT;
    const int nstages = (nrows + P - 1) / P;
    bool first_slice = true;
    for (int s = warp; s < nslices && ok; s += nwarps) {
      // producer: the first S stages of this slice
      // (every lane counts the issues; lane 0 issues the tensor loads)
      auto issue = [&](int stage_idx) {
        if (test_stall && blockIdx.x == 0 && warp == 0 && it_issue >= 1) return;
        if (lane != 0) {
          ++it_issue;
          return;
        }
        const int st = (int)(it_issue % S);
        const uint32_t dst = ring + (uint32_t)(st * St::kBytes);
        const uint32_t bar = bars + 8u * st;
        const int r = row0 + stage_idx * P;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     :: "r"(bar), "r"(St::kTx) : "memory");
        tma2d(dst, &maps.codes, s * 32 * BITS, r, bar);
        if constexpr (BITS == 2)
          tma1d(dst + St::kCodeBytes, &maps.lut, r * NE, bar);
        else
          tma2d(dst + St::kCodeBytes, &maps.lut, 0, r, bar);
        tma2d(dst + St::kCodeBytes + St::kLutSlot, &maps.scale, s * GPS, r, bar);
        tma2d(dst + St::kCodeBytes + St::kLutSlot + St::kGrpBytes, &maps.offset, s * GPS, r,
              bar);
        ++it_issue;
      };
      for (int q = 0; q < S && q < nstages; ++q) issue(q);
      if (!waited) {  // x (and y) may belong to the preceding kernel
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        waited = true;
      }
      const int k0 = s * 1024 + lane * 32;
      const bool kin = k0 < K;
      uint32_t xw[16];
      if (kin) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 q = ldg_nc_v4(x + k0 + 8 * v);
          xw[4 * v] = q.x; xw[4 * v + 1] = q.y; xw[4 * v + 2] = q.z; xw[4 * v + 3] = q.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xw[i] = 0u;
      }
      const uint32_t lv_shared =
          lut_shared ? (uint32_t)ldg_u16(lut_shared + (lane & (NE - 1))) : 0u;

      for (int si = 0; si < nstages; ++si) {
        const int st = (int)(it_use % S);
        const uint32_t parity = (it_use / S) & 1u;
        if (!mbar_wait_bounded(bars + 8u * st, parity, wait_ns)) {
          if (lane == 0) report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
          ok = false;
          *s_abort = 1;
          break;
        }
        const uint8_t* sp = gring + st * St::kBytes;
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(sp);
        const uint16_t* lt = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes);
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes + St::kLutSlot);
        const uint16_t* of = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes + St::kLutSlot +
                                                               St::kGrpBytes);
        // The stage's rows a pair at a time (rows 2pp, 2pp+1 share the tensor-core
        // steps), the pair loop unrolled so that the pairs' work interleaves and
        // the per-pair slots of part[] are fixed registers; each pair
        // accumulates in two chains (even and odd steps) to halve the
        // dependent-MMA latency.  A stage's rows past the matrix come back as
        // zeros from the tensor loads, and rows past the block's last are
        // computed and dropped, so the code loads need no row test.
        constexpr int NP = P / 2;
        float part[P];
#pragma unroll
        for (int j = 0; j < P; ++j) part[j] = 0.f;
        const int qd = lane >> 2;
        const bool diag = (lane & 3) == (qd >> 1);
        // row pairs holding at least one row of the matrix (the last stage of
        // a block may be partly past its rows)
        const int rows_left = nrows - si * P;
        const int npairs = rows_left >= P ? NP : (rows_left + 1) / 2;
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          if (pp >= npairs) break;
          const int ja = 2 * pp, jb = 2 * pp + 1;
          // the lane's 32 codes of each row: BITS consecutive words
          uint32_t wa[BITS], wb[BITS];
          if constexpr (BITS == 4) {
            const uint4 qa = reinterpret_cast<const uint4*>(codes)[ja * 32 + lane];
            const uint4 qb = reinterpret_cast<const uint4*>(codes)[jb * 32 + lane];
            wa[0] = qa.x; wa[1] = qa.y; wa[2] = qa.z; wa[3] = qa.w;
            wb[0] = qb.x; wb[1] = qb.y; wb[2] = qb.z; wb[3] = qb.w;
          } else if constexpr (BITS == 2) {
            const uint2 qa = reinterpret_cast<const uint2*>(codes)[ja * 32 + lane];
            const uint2 qb = reinterpret_cast<const uint2*>(codes)[jb * 32 + lane];
            wa[0] = qa.x; wa[1] = qa.y;
            wb[0] = qb.x; wb[1] = qb.y;
          } else {
#pragma unroll
            for (int b = 0; b < BITS; ++b) {
              wa[b] = codes[(ja * 32 + lane) * BITS + b];
              wb[b] = codes[(jb * 32 + lane) * BITS + b];
            }
          }
          const uint32_t la = lut_shared ? lv_shared : (uint32_t)lt[ja * NE + (lane & (NE - 1))];
          const uint32_t lb = lut_shared ? lv_shared : (uint32_t)lt[jb * NE + (lane & (NE - 1))];
          const uint32_t sa = dup2(sc[ja * GPS + gsub]), oa = dup2(of[ja * GPS + gsub]);
          const uint32_t sb = dup2(sc[jb * GPS + gsub]), ob = dup2(of[jb * GPS + gsub]);
          float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
          // codes 8t .. 8t + 7 of the lane's 32, two mma steps of 4 codes:
          // A rows 0-7 = row ja, rows 8-15 = row jb, B = x at the same four
          // columns; the diagonals C[q][q], C[q+8][q] are the two rows'
          // partial sums
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            uint32_t A[4], B[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int j = 8 * t + 2 * p;
              A[p] = dq_pair(la, code_word<BITS>(wa, j), code_word<BITS>(wa, j + 1), sa, oa);
              B[p] = dq_pair(lb, code_word<BITS>(wb, j), code_word<BITS>(wb, j + 1), sb, ob);
            }
            mma16816(c0, A[0], B[0], A[1], B[1], xw[4 * t], xw[4 * t + 1]);
            mma16816(c1, A[2], B[2], A[3], B[3], xw[4 * t + 2], xw[4 * t + 3]);
          }
          const float da = (qd & 1) ? c0[1] + c1[1] : c0[0] + c1[0];
          const float db = (qd & 1) ? c0[3] + c1[3] : c0[2] + c1[2];
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            if (k == pp) {
              part[2 * k] = diag ? da : 0.f;
              part[2 * k + 1] = diag ? db : 0.f;
            }
          }
        }
        ++it_use;
        // stage st is consumed: let the tensor loads overwrite it
        __syncwarp();
        if (si + S < nstages) {
          if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(si + S);
        }
        const float tot = reduce8(part, lane);
        if ((lane & 3) == 0) {
          const int idx = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
          float* dst = s_part + (size_t)warp * RTP + si * P + idx;
          *dst = first_slice ? tot : *dst + tot;
        }
      }
      first_slice = false;
    }
    __syncthreads();
    if (*s_abort == 0) {
      const int nw_used = nwarps < nslices ? nwarps : nslices;
      for (int t = threadIdx.x; t < nrows; t += blockDim.x) {
        float tot = 0.f;
        for (int w = 0; w < nw_used; ++w) tot += s_part[(size_t)w * RTP + t];
        if (grp.y32[mi] != nullptr)
          grp.y32[mi][row0 + t] = tot;
        else
          grp.y[mi][row0 + t] = f32_to_bf16_rn(tot);
      }
    }
    __syncthreads();
  }
  if (!waited) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  // before leaving, make sure no tensor load of this warp is still writing its ring
  if (!ok) {
    while (it_use < it_issue) {
      const int st = (int)(it_use % S);
      if (!mbar_wait_bounded(bars + 8u * st, (it_use / S) & 1u, wait_ns)) break;
      ++it_use;
    }
  }
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// G = 128 with 4-bit codes: the scale and offset folded into the shuffle
// table, and the products summed on the FMA pipe.
//
// A half-warp covers one group of a row at a time (16 lanes x 8 codes = 128
// columns), so the 16 lanes that hold a table can hold it already
// dequantised for that group: for row j, source lane e of half h computes
//   (W'(e, 4h), W'(e, 4h + 1)) and (W'(e, 4h + 2), W'(e, 4h + 3)),
//   W'(e, g) = bf16(LUT_j[e] * s_jg + o_jg)   (one bf16x2 fused multiply-add,
// the rounding the per-weight kernel applies), and keeps each widened to an
// fp32 (exact) in one register per step.  A lookup is then one shuffle inside
// the half-warp (segment mask 16) that returns the weight itself.  Step t
// (0..3) of a lane in half h reads code word 16 (4h + (t ^ h)) + (lane & 15)
// of the row, so the two halves read different 16-bank ranges; the lane's x
// columns follow the same map and are widened to fp32 once per slice.  Two
// weights and their two x values go into one packed fp32 fused multiply-add
// (__ffma2_rn); each lane keeps two accumulator pairs per row, and the rows'
// lane sums are added over the warp at the end of a stage.
//
// Measured on B200 against the same kernel shape with the products on the
// tensor core (mma.sync m16n8k16, one useful diagonal in eight): 42.0
// against 48.8 us on 8192 -> 28672; the legacy warp-level MMA, not the
// lookups, bounded that form.
__device__ __forceinline__ float fold_fetch(uint32_t tab, uint32_t code) {
  uint32_t v;
  asm("shfl.sync.idx.b32 %0, %1, %2, 0x101f, 0xffffffff;" : "=r"(v) : "r"(tab), "r"(code));
  return __uint_as_float(v);
}

// kDecodeLayout: the codes are in any4_repack's layout, where the four words
// a lane reads in a row's 1024-column slice sit together (one 16-byte load)
template <bool kDecodeLayout>
__global__ void __maxnreg__(128) decode_tma_ffma_kernel(
    const __grid_constant__ TmaGroup grp, const uint16_t* __restrict__ x, int K, int nslices,
    int rows_per_block, int32_t* dev_status, int test_stall) {
  constexpr int GPS = 8, BITS = 4;
  const unsigned long long wait_ns = test_stall ? kTmaTestWaitNs : kTmaWaitNs;
  using St = TmaStage<GPS, BITS>;
  constexpr int P = St::P;
  constexpr int S = kTmaStages;
  constexpr int NE = St::kEntries;
  constexpr int kRowWords = 32 * BITS;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int RT = rows_per_block;
  // A slice's stages: head_rows rows (the block's rows modulo P, or P),
  // then P rows each, so that a block's one short stage comes first and
  // every later stage is full.
  const int H = grp.head_rows;
  const int RTP = RT <= H ? H : H + ((RT - H + P - 1) / P) * P;
  auto stage_row = [H](int si) { return si == 0 ? 0 : H + (si - 1) * P; };
  const uint32_t base = (smem_addr(smem_raw) + 127u) & ~127u;
  uint8_t* gbase = smem_raw + (base - smem_addr(smem_raw));
  const uint32_t ring = base + (uint32_t)(warp * S * St::kBytes);
  const uint8_t* gring = gbase + warp * S * St::kBytes;
  const uint32_t bars = base + (uint32_t)(nwarps * S * St::kBytes) + (uint32_t)(warp * S * 8);
  float* s_part =
      reinterpret_cast<float*>(gbase + nwarps * S * St::kBytes + nwarps * S * 8 + 16);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + nwarps * S * St::kBytes +
                                                          nwarps * S * 8);
  if (threadIdx.x == 0) *s_abort = 0;

  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init_(bars + 8u * st, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const int64_t nblocks = grp.blk_end[grp.count - 1];
  uint32_t it_issue = 0, it_use = 0;
  bool waited = false, ok = true;

  const int h = lane >> 4, e = lane & 15;
  const int wofs0 = 80 * h + e, wofs1 = 48 * h + 16 + e;
  // W' of the lane's step-t group into the high half of an fp32 (the low
  // half zero): steps whose group sits in the low bf16 half use sel_lo
  const uint32_t sel_lo = 0x1044u, sel_hi = 0x3244u;
  const uint32_t sel_even = h ? sel_hi : sel_lo, sel_odd = h ? sel_lo : sel_hi;

  for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    int mi = 0;
    while (mi + 1 < grp.count && blk >= grp.blk_end[mi]) ++mi;
    const TmaMaps& maps = grp.maps[mi];
    const int N = grp.N[mi];
    const uint16_t* lut_shared = grp.lut_shared[mi];
    const int row0 = (int)((blk - (mi > 0 ? grp.blk_end[mi - 1] : 0)) * RT);
    const int nrows = (N - row0) < RT ? (N - row0) : RT;
    const int nstages = nrows <= H ? 1 : 1 + (nrows - H + P - 1) / P;
    bool first_slice = true;
    for (int s = warp; s < nslices && ok; s += nwarps) {
      auto issue = [&](int stage_idx) {
        if (test_stall && blockIdx.x == 0 && warp == 0 && it_issue >= 1) return;
        if (lane != 0) {
          ++it_issue;
          return;
        }
        const int st = (int)(it_issue % S);
        const uint32_t dst = ring + (uint32_t)(st * St::kBytes);
        const uint32_t bar = bars + 8u * st;
        const int r = row0 + stage_row(stage_idx);
        const uint32_t tx = stage_idx == 0 ? St::kTx - (uint32_t)((P - H) * kRowWords * 4) : St::kTx;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     :: "r"(bar), "r"(tx) : "memory");
        tma2d(dst, stage_idx == 0 ? &maps.codes_head : &maps.codes, s * kRowWords, r, bar);
        tma2d(dst + St::kCodeBytes, &maps.lut, 0, r, bar);
        tma2d(dst + St::kCodeBytes + St::kLutSlot, &maps.scale, s * GPS, r, bar);
        tma2d(dst + St::kCodeBytes + St::kLutSlot + St::kGrpBytes, &maps.offset, s * GPS, r,
              bar);
        ++it_issue;
      };
      for (int q = 0; q < S && q < nstages; ++q) issue(q);
      if (!waited) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        waited = true;
      }
      // x at this lane's columns of the four steps, widened to fp32 pairs
      float2 xf[4][4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 q = ldg_nc_v4(x + s * 1024 + 128 * (4 * h + (t ^ h)) + 8 * e);
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int m = 0; m < 4; ++m)
          xf[t][m] = make_float2(__uint_as_float(qw[m] << 16),
                                 __uint_as_float(qw[m] & 0xffff0000u));
      }
      const uint32_t lv_shared = lut_shared ? dup2(ldg_u16(lut_shared + e)) : 0u;

      for (int si = 0; si < nstages; ++si) {
        const int st = (int)(it_use % S);
        const uint32_t parity = (it_use / S) & 1u;
        if (!mbar_wait_bounded(bars + 8u * st, parity, wait_ns)) {
          if (lane == 0) report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
          ok = false;
          *s_abort = 1;
          break;
        }
        const uint8_t* sp = gring + st * St::kBytes;
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(sp);
        const uint16_t* lt = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes);
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes + St::kLutSlot);
        const uint16_t* of = reinterpret_cast<const uint16_t*>(sp + St::kCodeBytes + St::kLutSlot +
                                                               St::kGrpBytes);
        // one row of the stage: the lane's sum over its 32 columns (shared:
        // the matrix has one table, held in lv_shared; the choice is made
        // once per stage, outside the unrolled rows)
        auto row = [&](int j, auto shared) -> float {
          uint32_t w[4];
          if constexpr (kDecodeLayout) {
            const uint4 q4 = reinterpret_cast<const uint4*>(codes + j * kRowWords)[lane];
            w[0] = q4.x; w[1] = q4.y; w[2] = q4.z; w[3] = q4.w;
          } else {
            w[0] = codes[j * kRowWords + wofs0];
            w[1] = codes[j * kRowWords + wofs1];
            w[2] = codes[j * kRowWords + wofs0 + 32];
            w[3] = codes[j * kRowWords + wofs1 + 32];
          }
          uint32_t l2;
          if constexpr (decltype(shared)::value)
            l2 = lv_shared;
          else
            l2 = dup2(lt[j * NE + e]);
          const uint2 s4 = *reinterpret_cast<const uint2*>(sc + j * GPS + 4 * h);
          const uint2 o4 = *reinterpret_cast<const uint2*>(of + j * GPS + 4 * h);
          const uint32_t t01 = hfma2_bits(l2, s4.x, o4.x), t23 = hfma2_bits(l2, s4.y, o4.y);
          const uint32_t tab[4] = {__byte_perm(t01, 0u, sel_even), __byte_perm(t01, 0u, sel_odd),
                                   __byte_perm(t23, 0u, sel_even), __byte_perm(t23, 0u, sel_odd)};
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float2 wv = make_float2(fold_fetch(tab[t], w[t] >> (8 * m)),
                                            fold_fetch(tab[t], w[t] >> (8 * m + 4)));
              if (m & 1)
                a1 = __ffma2_rn(wv, xf[t][m], a1);
              else
                a0 = __ffma2_rn(wv, xf[t][m], a0);
            }
          }
          return (a0.x + a0.y) + (a1.x + a1.y);
        };
        float part[P];
        const int rows_left = si == 0 ? (nrows < H ? nrows : H) : nrows - stage_row(si);
        auto rows = [&](auto shared) {
          if (rows_left >= P) {
#pragma unroll
            for (int j = 0; j < P; ++j) part[j] = row(j, shared);
          } else {
#pragma unroll
            for (int j = 0; j < P; ++j) part[j] = j < rows_left ? row(j, shared) : 0.f;
          }
        };
        if (lut_shared)
          rows(std::true_type{});
        else
          rows(std::false_type{});
        ++it_use;
        __syncwarp();
        if (si + S < nstages) {
          if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(si + S);
        }
        const float tot = reduce8(part, lane);
        const int idx = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
        if ((lane & 3) == 0 && idx < (si == 0 ? H : P)) {
          float* dst = s_part + (size_t)warp * RTP + stage_row(si) + idx;
          *dst = first_slice ? tot : *dst + tot;
        }
      }
      first_slice = false;
    }
    __syncthreads();
    if (*s_abort == 0) {
      const int nw_used = nwarps < nslices ? nwarps : nslices;
      for (int t = threadIdx.x; t < nrows; t += blockDim.x) {
        float tot = 0.f;
        for (int w = 0; w < nw_used; ++w) tot += s_part[(size_t)w * RTP + t];
        if (grp.y32[mi] != nullptr)
          grp.y32[mi][row0 + t] = tot;
        else
          grp.y[mi][row0 + t] = f32_to_bf16_rn(tot);
      }
    }
    __syncthreads();
  }
  if (!waited) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  if (!ok) {
    while (it_use < it_issue) {
      const int st = (int)(it_use % S);
      if (!mbar_wait_bounded(bars + 8u * st, (it_use / S) & 1u, wait_ns)) break;
      ++it_use;
    }
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// Encoded maps, kept on the host: a decode loop calls the same matrices over
// and over, and a map depends only on the arguments in MapKey (address,
// sizes, box, element type; not the device), so each distinct map is encoded
// once.  Keys are zero-filled before use, so padding compares equal.
struct MapKey {
  const void* ptr;
  uint64_t dims[2];
  uint64_t stride;
  uint32_t box[2];
  int32_t dtype;
  int32_t rank;
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
    uint64_t h = 1469598103934665603ull;  // FNV-1a
    for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ b[i]) * 1099511628211ull;
    return (size_t)h;
  }
};
struct MapKeyEq {
  bool operator()(const MapKey& a, const MapKey& b) const {
    return memcmp(&a, &b, sizeof(MapKey)) == 0;
  }
};
constexpr size_t kMapCacheMax = 8192;  // cleared when full

bool cached_encode(EncodeFn enc, CUtensorMap* m, const MapKey& key) {
  static std::mutex mu;
  static auto* cache = new std::unordered_map<MapKey, CUtensorMap, MapKeyHash, MapKeyEq>();
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache->find(key);
    if (it != cache->end()) {
      *m = it->second;
      return true;
    }
  }
  const cuuint64_t dims[2] = {key.dims[0], key.dims[1]};
  // a rank-1 map has no stride, but the encoder rejects a NULL stride array
  const cuuint64_t strides[1] = {key.stride};
  const cuuint32_t box[2] = {key.box[0], key.box[1]};
  const cuuint32_t es[2] = {1, 1};
  if (enc(m, (CUtensorMapDataType)key.dtype, (cuuint32_t)key.rank, const_cast<void*>(key.ptr),
          dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache->size() >= kMapCacheMax) cache->clear();
  cache->emplace(key, *m);
  return true;
}

bool encode2d(EncodeFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* ptr,
              uint64_t inner, uint64_t rows, uint64_t row_bytes, uint32_t box_inner,
              uint32_t box_rows) {
  MapKey k;
  memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = inner;
  k.dims[1] = rows;
  k.stride = row_bytes;
  k.box[0] = box_inner;
  k.box[1] = box_rows;
  k.dtype = (int32_t)dt;
  k.rank = 2;
  return cached_encode(enc, m, k);
}

// 1-D map over n u16 values (the 2-bit tables: 8 bytes a row, below the
// 16-byte row stride a 2-D map needs), box of box_n values
bool encode1d(EncodeFn enc, CUtensorMap* m, const void* ptr, uint64_t n, uint32_t box_n) {
  MapKey k;
  memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = n;
  k.stride = ((n * 2 + 15) / 16) * 16;
  k.box[0] = box_n;
  k.dtype = (int32_t)CU_TENSOR_MAP_DATA_TYPE_UINT16;
  k.rank = 1;
  return cached_encode(enc, m, k);
}

bool encode_weights(EncodeFn enc, TmaMaps* maps, const DecodeWeights& w, int64_t K, int64_t G,
                    int GPS, int bits, int head_rows) {
  constexpr int P = kTmaRows;
  const uint64_t N = (uint64_t)w.N;
  const uint32_t ne = 1u << bits;
  // codes as u32 [N][K bits / 32]: 1024 codes of a row = 32 * bits words
  if (!encode2d(enc, &maps->codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, w.packed,
                (uint64_t)K * bits / 32, N, (uint64_t)K * bits / 8, 32 * bits, P) ||
      !encode2d(enc, &maps->codes_head, CU_TENSOR_MAP_DATA_TYPE_UINT32, w.packed,
                (uint64_t)K * bits / 32, N, (uint64_t)K * bits / 8, 32 * bits, head_rows) ||
      !encode2d(enc, &maps->scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scale, (uint64_t)(K / G), N,
                (uint64_t)(K / G) * 2, GPS, P) ||
      !encode2d(enc, &maps->offset, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.offset, (uint64_t)(K / G),
                N, (uint64_t)(K / G) * 2, GPS, P))
    return false;
  // One table for the matrix (lut_row_stride 0) is read directly by the
  // kernel; the per-stage tensor load of the table slot still runs (rows past
  // the first come back as zeros) so that every stage carries the same bytes.
  const uint64_t lut_rows = w.lut_row_stride != 0 ? N : 1;
  if (bits == 2) return encode1d(enc, &maps->lut, w.lut, lut_rows * ne, P * ne);
  return encode2d(enc, &maps->lut, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.lut, ne, lut_rows, ne * 2,
                  ne, P);
}

template <int GPS, int BITS>
any4_status run_tma(const uint16_t* x, const DecodeWeights* w, int count, int64_t K, int64_t G,
                    bool overlap, int32_t* dev_status, bool test_stall, bool decode_layout,
                    cudaStream_t stream, const DeviceInfo& dev) {
  using St = TmaStage<GPS, BITS>;
  constexpr int P = St::P;
  constexpr int S = kTmaStages;
  if (count < 1 || count > kTmaMaxGroup) return ANY4_ERR_UNSUPPORTED;
  EncodeFn enc = get_encode();
  if (!enc) return ANY4_ERR_UNSUPPORTED;
  TmaGroup grp;
  memset(&grp, 0, sizeof(grp));
  int64_t total_rows = 0;
  for (int i = 0; i < count; ++i) total_rows += w[i].N;
  const int nslices = (int)((K + 1023) / 1024);
  const int per_warp = (nslices + kTmaMaxWarps - 1) / kTmaMaxWarps;
  const int nwarps = (nslices + per_warp - 1) / per_warp;
  const int threads = nwarps * 32;

  // G = 128 with 4-bit codes: the folded-table kernel; every other shape:
  // the per-weight multiply-add kernel
  constexpr bool kFold = GPS == 8 && BITS == 4;
  if (decode_layout && (!kFold || K % 1024 != 0)) return ANY4_ERR_UNSUPPORTED;
  auto kern = kFold ? (decode_layout ? decode_tma_ffma_kernel<true> : decode_tma_ffma_kernel<false>)
                    : decode_tma_kernel<GPS, BITS>;
  const size_t ring_bytes = (size_t)nwarps * S * St::kBytes + (size_t)nwarps * S * 8 + 16 + 128;
  const int kMaxRT = 512;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern),
                          std::min<size_t>(dev.smem_optin, 227 * 1024)) != ANY4_OK)
    return ANY4_ERR_CUDA;
  // rows per block (one value for every matrix of the group) from the blocks
  // that fit per SM, which depends (through the partial sums) on the rows per
  // block: settle it in two passes
  int per_sm = 2;
  int64_t rt = 0, rtp = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t wave = (int64_t)dev.sm_count * per_sm;
    rt = std::min<int64_t>((total_rows + wave - 1) / wave, kMaxRT);
    rtp = ((rt + P - 1) / P) * P;
    const size_t smem_try = ring_bytes + (size_t)nwarps * rtp * sizeof(float);
    int occ = cached_occupancy(reinterpret_cast<const void*>(kern), threads, smem_try);
    if (occ < 1) occ = 1;
    if (occ == per_sm) break;
    per_sm = occ;
  }
  const int64_t wave = (int64_t)dev.sm_count * per_sm;
  rt = std::min<int64_t>((total_rows + wave - 1) / wave, kMaxRT);
  // at least 4 rows a block: below that a block's fixed costs (barriers, its
  // x loads, the partial-sum pass) outweigh its rows (1024-row matrices ran
  // 25 % faster with 4 rows a block than with the 2 that one wave gives)
  rt = std::max<int64_t>(rt, 4);
  // 2-bit tables come by a 1-D tensor load at element 4 r of the table
  // array: its byte offset 8 r must be a multiple of 16, so every stage's
  // first row r (row0 + a multiple of P) must be even, hence rt even
  if (BITS == 2 && (rt & 1)) ++rt;
  rtp = ((rt + P - 1) / P) * P;
  // the folded-table kernel's first stage per slice: rt mod P rows (or P)
  const int head_rows = kFold && rt % P != 0 ? (int)(rt % P) : P;
  for (int i = 0; i < count; ++i) {
    if (!encode_weights(enc, &grp.maps[i], w[i], K, G, GPS, BITS, head_rows))
      return ANY4_ERR_CUDA;
    grp.y[i] = w[i].y;
    grp.y32[i] = w[i].y32;
    grp.lut_shared[i] = w[i].lut_row_stride == 0 ? w[i].lut : nullptr;
    grp.N[i] = (int)w[i].N;
  }
  grp.count = count;
  grp.head_rows = head_rows;
  int64_t nblocks = 0;
  for (int i = 0; i < count; ++i) {
    nblocks += (w[i].N + rt - 1) / rt;
    grp.blk_end[i] = nblocks;
  }
  const int grid = (int)std::min<int64_t>(nblocks, wave);
  const size_t smem = ring_bytes + (size_t)nwarps * rtp * sizeof(float);

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
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, grp, x, (int)K, nslices, (int)rt,
                                             dev_status, test_stall ? 1 : 0);
  return err == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

template <int BITS>
any4_status run_tma_bits(const uint16_t* x, const DecodeWeights* w, int count, int64_t K,
                         int64_t G, bool overlap, int32_t* dev_status, bool test_stall,
                         bool decode_layout, cudaStream_t stream, const DeviceInfo& dev) {
  switch (G) {
    case 128:
      return run_tma<8, BITS>(x, w, count, K, G, overlap, dev_status, test_stall, decode_layout,
                              stream, dev);
    case 64:
      return run_tma<16, BITS>(x, w, count, K, G, overlap, dev_status, test_stall,
                               decode_layout, stream, dev);
    case 32:
      return run_tma<32, BITS>(x, w, count, K, G, overlap, dev_status, test_stall,
                               decode_layout, stream, dev);
    default:
      return ANY4_ERR_UNSUPPORTED;
  }
}

}  // namespace

bool decode_tma_supported(int64_t M, int64_t N, int64_t K, int64_t G, int bits) {
  if (M != 1) return false;
  if (bits < 2 || bits > 4) return false;
  if (G != 32 && G != 64 && G != 128) return false;
  if ((K / G) % 8 != 0) return false;           // 16-byte row stride of scale/offset
  if ((K * bits) % 128 != 0) return false;      // 16-byte row stride of the codes
  if (N > INT32_MAX / 2 || K > INT32_MAX / 2) return false;
  return true;
}

any4_status launch_decode_tma_group(const uint16_t* x, const DecodeWeights* w, int count,
                                    int64_t K, int64_t G, int bits, bool overlap,
                                    int32_t* dev_status, bool test_stall, cudaStream_t stream,
                                    const DeviceInfo& dev, bool decode_layout) {
  switch (bits) {
    case 4:
      return run_tma_bits<4>(x, w, count, K, G, overlap, dev_status, test_stall, decode_layout,
                             stream, dev);
    case 3:
      return run_tma_bits<3>(x, w, count, K, G, overlap, dev_status, test_stall, decode_layout,
                             stream, dev);
    case 2:
      return run_tma_bits<2>(x, w, count, K, G, overlap, dev_status, test_stall, decode_layout,
                             stream, dev);
    default:
      return ANY4_ERR_UNSUPPORTED;
  }
}

any4_status launch_decode_tma(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                              int64_t lut_row_stride, const uint16_t* scale,
                              const uint16_t* offset, uint16_t* y, float* y32, int64_t N,
                              int64_t K, int64_t G, bool overlap, int32_t* dev_status,
                              bool test_stall, cudaStream_t stream, const DeviceInfo& dev,
                              bool decode_layout) {
  const DecodeWeights w = {packed, lut, lut_row_stride, scale, offset, y, y32, N};
  return launch_decode_tma_group(x, &w, 1, K, G, 4, overlap, dev_status, test_stall, stream,
                                 dev, decode_layout);
}

bool decode_layout_supported(int64_t M, int64_t N, int64_t K, int64_t G) {
  return M == 1 && G == 128 && K % 1024 == 0 && decode_tma_supported(M, N, K, G);
}

}  // namespace any4
