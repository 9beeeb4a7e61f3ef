// Prefill-path any4 matmul (large M) on the 5th-generation tensor cores.
//
//   y[m][n] = sum_k x[m][k] * W[n][k],   W[n][k] = bf16(fmaf(LUT[n][c], s, o))
//
// Paper: "any4: Learned 4-bit Numeric Representation for LLMs", §4.1 Eq. 8,
// §2.5.2 (dequant), §4.2 (y = x W^T; weights are dequantised on the fly
// before the tensor-core multiply).  At large M the product is a dense
// contraction, so it runs on tcgen05.mma with fp32 accumulators in TMEM.
//
// One persistent CTA per SM (the smem footprint allows one), tile = 256 rows
// of x by 256 weight rows, K in 64-column stages:
//   warp 0      TMA loads of the two 128 x 64 bf16 x tiles of a stage
//               (SWIZZLE_128B, no multicast)
//   warp 1      TMEM allocation (512 columns = two 128 x 256 fp32
//               accumulators) and, from one thread, the tcgen05.mma issue
//               (M = 128, N = 256, K = 16; both operands K-major in smem)
//   warps 2..17 the dequant stage: two lanes per weight row of the tile, each
//               owning 32 of the stage's 64 codes; codes, scale and offset are
//               fetched from global memory three stages ahead into registers,
//               each code is looked up in the row's table held in registers
//               (byte permutes, no memory traffic), scaled and offset by a
//               bf16x2 fused multiply-add (the exact LUT*scale+offset rounded
//               once to bf16: the dequant definition's bf16(fmaf(...)) whenever
//               the fp32 fmaf is exact, at most one bf16 ulp away otherwise)
//               and stored into the row of the B tile in
//               the 128-byte-swizzled layout the MMA reads.  After the last
//               stage of a tile the same warps drain TMEM (tcgen05.ld), round
//               to bf16 and write y.
// Shared-memory bandwidth is the scarce resource here (the MMA reads both
// operands from it, TMA and the dequant warps write them), which is why the
// table lookups are done in registers.  Each weight tile is dequantised once
// per 256 rows of x.
//
// Synchronisation: mbarriers per stage (x landed / W written / stage free),
// one for "accumulators ready" and one for "accumulators drained".  Every
// wait is bounded (about 2 s of %globaltimer); on expiry the kernel sets
// ANY4_ERR_TIMEOUT in dev_status, every role leaves its loop, and TMEM is
// released before the CTA exits.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kBM = 128;                        // x rows per accumulator (MMA M)
constexpr int kNAcc = 2;                        // accumulators per CTA -> 256 rows of x
constexpr int kBN = 256;                        // weight rows per tile (MMA N)
constexpr int kBK = 64;                         // K per stage: one 128-byte swizzle row
constexpr int kStages = 3;
constexpr int kATileBytes = kBM * kBK * 2;      // 16 KB
constexpr int kBTileBytes = kBN * kBK * 2;      // 32 KB
constexpr int kStageBytes = kNAcc * kATileBytes + kBTileBytes;  // 64 KB
constexpr int kXformWarps = 2 * kBN / 32;       // 16: two lanes per weight row
constexpr int kThreads = 64 + kXformWarps * 32; // 576
constexpr int kTmemCols = kNAcc * kBN;          // 512
// layout of the dynamic shared memory (offsets from a 1 KB-aligned base)
constexpr int kStageOff = 0;                    // 1024-byte aligned stages
constexpr int kBarOff = kStageOff + kStages * kStageBytes;
constexpr int kNumBars = 3 * kStages + 2;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kSmemUsed = kMiscOff + 32;
constexpr int kSmemAlloc = kSmemUsed + 1024;    // slack to align the base to 1 KB
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// Every wait on a barrier or a flag gives up after this long (about 2 s of
// %globaltimer), or after 1 ms in the test mode that stops one block's x
// stream on purpose.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr unsigned long long kTestWaitLimitNs = 1000000ull;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.  Returns
// false (after flagging the error and the CTA-wide abort) if it does not
// complete within the limit or another role has aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* dev_status, unsigned long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// mbar_wait by every lane of a warp, with one outcome for the whole warp (so
// that no lane is left alone in a later warp-synchronous instruction).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, int32_t* dev_status,
                                               unsigned long long limit) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, dev_status, limit)) != 0;
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Tensor load with an L2 eviction policy (from createpolicy): x tiles are
// read by every block that works on their rows, so they are kept in L2
// (evict_last) while the weight stream, read once, goes first (evict_first).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(bar), "l"(policy) : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, rows of 128 bytes,
// 128-byte swizzle, 8-row groups 1024 bytes apart (SBO), base 1024-aligned.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);   // start address, 16-byte units
  d |= (uint64_t)1 << 16;                    // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                    // SWIZZLE_128B
  return d;
}
// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

// Phase alignment of the stream-K schedule (two-pass mode): block b starts at
// unit U b / grid, mostly inside a tile, so without care the blocks sweep K at
// offsets spread over the whole of it and every x and W panel is wanted at
// many different times (the down shape re-read x about 9 times from DRAM).
// Each tile's stages are therefore taken in a rotated order, starting at
// stage rot(tile), chosen so that the block that finishes the tile reads
// stage t of K at step t of its own range; the other blocks then run at most
// one block range (mod the tile's stages) ahead, so at any moment all blocks
// read a narrow band of K and each x and W panel is fetched from DRAM about
// once.  Only the TMA coordinates change: the MMA consumes stages in issue
// order, and a tile's partial sums still meet in block order.
__device__ __forceinline__ int kb_rotation(int tile, int nkb, int64_t U, int64_t grid) {
  const int64_t v = (int64_t)(tile + 1) * nkb;              // one past the tile's last unit
  const int64_t b = (v * grid + U - 1) / U - 1;             // the block holding unit v - 1
  const int64_t ub = U * b / grid;                          // where that block starts
  int64_t r = ((int64_t)tile * nkb - ub) % nkb;
  if (r < 0) r += nkb;
  return (int)r;
}

// Walks a block's range [u, ue) of (tile, stage) units as segments: the
// stages kb0 .. kb1-1 of one tile.
struct SegIter {
  int64_t u, ue;
  int nkb;
  __device__ __forceinline__ bool next(int& tile, int& kb0, int& kb1) {
    if (u >= ue) return false;
    tile = (int)(u / nkb);
    kb0 = (int)(u - (int64_t)tile * nkb);
    const int64_t rem = ue - u;
    kb1 = (int)((int64_t)kb0 + rem < nkb ? (int64_t)kb0 + rem : nkb);
    u += kb1 - kb0;
    return true;
  }
};

// Stream-K partial sums of one block: 256 x 256 fp32, stored in the order the
// epilogue threads hold them (block, dequant warp, 16-column chunk, float4 of
// the chunk, lane) so that every warp-wide store and load is contiguous.  The
// layout is private to this kernel: the same thread mapping writes and reads it.
__device__ __forceinline__ size_t partial_index(int blk, int tw, int chunk, int lane) {
  return ((((size_t)blk * kXformWarps + tw) * (kBN / 32) + chunk) * 4) * 32 + lane;
}

// ---------------------------------------------------------------- the kernel
// kWTma = false: the dequant warps build each W tile from the packed codes
// (one pass).  kWTma = true: W was dequantised to bf16 beforehand (any4_dequant
// into the workspace) and warp 0 loads its tiles with TMA like the x tiles;
// the dequant warps only run the epilogue (two passes, for large M).
template <bool kWTma>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
    const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ y, float* __restrict__ y32, int M, int N, int K, int G, int vec_store,
    int32_t* dev_status, float* __restrict__ ws_partial, uint32_t* __restrict__ ws_flags,
    int test_stall) {
  // test_stall: block 0's x stream stops after its first stage, so a wait of
  // the MMA issuer runs out (1 ms limit); the kernel must end cleanly
  const unsigned long long wait_ns = test_stall ? kTestWaitLimitNs : kWaitLimitNs;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  auto stage_a = [&](int s, int h) { return base + kStageOff + s * kStageBytes + h * kATileBytes; };
  auto stage_b = [&](int s) { return base + kStageOff + s * kStageBytes + kNAcc * kATileBytes; };
  const uint32_t bars = base + kBarOff;
  auto full_a = [&](int s) { return bars + 8u * s; };
  auto full_b = [&](int s) { return bars + 8u * (kStages + s); };
  auto empty = [&](int s) { return bars + 8u * (2 * kStages + s); };
  const uint32_t accum_full = bars + 8u * (3 * kStages);
  const uint32_t accum_empty = bars + 8u * (3 * kStages + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
  int* partial_done = reinterpret_cast<int*>(smem + kMiscOff + 8);
  // stages of x (and W) the producer issued and the MMA issuer saw complete:
  // on an abort, the copies between the two are drained before the exit
  volatile uint32_t* n_issued = reinterpret_cast<volatile uint32_t*>(smem + kMiscOff + 12);
  volatile uint32_t* n_landed = reinterpret_cast<volatile uint32_t*>(smem + kMiscOff + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_a(s), 1);
      mbar_init(full_b(s), kWTma ? 1 : kXformWarps);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum_full, 1);
    mbar_init(accum_empty, kXformWarps);
    *abort_flag = 0;
    *partial_done = 0;
    *n_issued = 0;
    *n_landed = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_mtiles = (M + kNAcc * kBM - 1) / (kNAcc * kBM);
  const int n_ntiles = (N + kBN - 1) / kBN;
  const int ntiles = n_mtiles * n_ntiles;
  const int nkb = (K + kBK - 1) / kBK;
  // Stream-K split: the (tile, stage) units are divided evenly over the
  // blocks; this block owns units [ub, ue).
  const int64_t U = (int64_t)ntiles * nkb;
  const int64_t ub = U * blockIdx.x / gridDim.x;
  const int64_t ue = U * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------ x tiles via TMA
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last(), pol_w = l2_policy_evict_first();
      uint32_t it = 0;
      SegIter seg{ub, ue, nkb};
      int tile, kb0, kb1;
      while (seg.next(tile, kb0, kb1)) {
        const int mt = tile % n_mtiles;
        const int rot = kWTma ? kb_rotation(tile, nkb, U, gridDim.x) : 0;
        for (int kbl = kb0; kbl < kb1; ++kbl, ++it) {
          const int kb = kbl + rot < nkb ? kbl + rot : kbl + rot - nkb;
          const int s = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (test_stall && blockIdx.x == 0 && it >= 1) goto done;  // the stream stops here
          if (!mbar_wait(empty(s), ph ^ 1u, abort_flag, dev_status, wait_ns)) goto done;
          *n_issued = it + 1;
          mbar_arrive_expect_tx(full_a(s), kNAcc * kATileBytes);
          for (int h = 0; h < kNAcc; ++h)
            tma_load_2d(stage_a(s, h), &tmap_x, kb * kBK, mt * kNAcc * kBM + h * kBM, full_a(s),
                        pol_x);
          if (kWTma) {
            // the bf16 W tile: 256 weight rows x 64 columns, same swizzled layout
            mbar_arrive_expect_tx(full_b(s), kBTileBytes);
            tma_load_2d(stage_b(s), &tmap_w, kb * kBK, (tile / n_mtiles) * kBN, full_b(s),
                        pol_w);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue (one thread)
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      SegIter seg{ub, ue, nkb};
      int tile, kb0, kb1;
      for (; seg.next(tile, kb0, kb1); ++tcount) {
        if (tcount > 0 && !mbar_wait(accum_empty, (tcount - 1) & 1u, abort_flag, dev_status, wait_ns))
          goto done;
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(full_a(s), ph, abort_flag, dev_status, wait_ns)) goto done;
          if (!mbar_wait(full_b(s), ph, abort_flag, dev_status, wait_ns)) goto done;
          *n_landed = it + 1;
          tc_fence_after();
          const uint64_t db = smem_desc_sw128(stage_b(s));
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j) {
#pragma unroll
            for (int h = 0; h < kNAcc; ++h) {
              const uint64_t da = smem_desc_sw128(stage_a(s, h));
              // advance 16 columns = 32 bytes = 2 descriptor units
              tc_mma(tmem + (uint32_t)(h * kBN), da + 2u * j, db + 2u * j, kIdesc,
                     (kb > kb0 || j > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty(s));  // stage s free once these MMAs have read it
        }
        tc_commit(accum_full);  // accumulators of this segment complete
      }
    }
  } else {
    // ------------------------------------------------ dequant + epilogue
    const int tw = warp - 2;                         // 0 .. 15
    // Lanes 2i and 2i+1 of warp tw share weight row tw * 16 + i: lane parity
    // `half` picks which 32 of a stage's 64 codes the lane converts, so the
    // pair's code loads fall in one 32-byte sector.
    const int half = lane & 1;
    const int rloc = tw * 16 + (lane >> 1);          // weight row within the tile
    const int64_t row_bytes = K / 2;
    const int groups = K / G;
    // scale/offset rows are read 8 groups (16 bytes) at a time when every
    // row starts on a 16-byte boundary
    const bool oct_vec = (groups & 7) == 0;
    uint32_t it = 0, tcount = 0;
    SegIter seg{ub, ue, nkb};
    int tile, kb0, kb1;
    for (; seg.next(tile, kb0, kb1); ++tcount) {
      const int mt = tile % n_mtiles;
      const int nt = tile / n_mtiles;
      const int n = nt * kBN + rloc;
      const bool rin = n < N;
      if constexpr (!kWTma) {
        // The row's 16-entry table in registers, split into byte planes:
        // tl[i] = low bytes of entries 4i..4i+3, th[i] = their high bytes.
        uint32_t tl[4], th[4];
        {
          const uint16_t* lrow = lut + (int64_t)(rin ? n : 0) * lut_row_stride;
          const uint4 e0 = rin ? ldg_nc_v4(lrow) : make_uint4(0u, 0u, 0u, 0u);
          const uint4 e1 = rin ? ldg_nc_v4(lrow + 8) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
  #pragma unroll
          for (int i = 0; i < 4; ++i) {
            tl[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x6420);
            th[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x7531);
          }
        }
        const uint8_t* prow = packed + (int64_t)(rin ? n : 0) * row_bytes;
        // the even lane of a pair holds its row's scales, the odd lane its
        // offsets, 8 groups per register quad
        const uint16_t* grow = (half ? offset : scale) + (int64_t)(rin ? n : 0) * groups;
        auto fetch_octet = [&](int o8) -> uint4 {
          if (!rin || 8 * o8 >= groups) return make_uint4(0u, 0u, 0u, 0u);
          if (oct_vec) return ldg_nc_v4(grow + 8 * o8);
          uint32_t w[4];
  #pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int g0 = 8 * o8 + 2 * i;
            const uint32_t lo = g0 < groups ? ldg_u16(grow + g0) : 0u;
            const uint32_t hi = g0 + 1 < groups ? ldg_u16(grow + g0 + 1) : 0u;
            w[i] = lo | (hi << 16);
          }
          return make_uint4(w[0], w[1], w[2], w[3]);
        };
        // bf16 bits of group slot j (0..7) of an octet
        auto pick = [](const uint4& v, int j) -> uint32_t {
          const uint32_t w = (j & 4) ? ((j & 2) ? v.w : v.z) : ((j & 2) ? v.y : v.x);
          return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
        };

        // This lane's 16 bytes of codes of a stage, fetched three stages ahead.
        auto fetch = [&](int kb) -> uint4 {
          const int k = kb * kBK + 32 * half;
          return (rin && k < K) ? ldg_stream_v4(prow + k / 2) : make_uint4(0u, 0u, 0u, 0u);
        };
        int cur8 = (kb0 * kBK) / G >> 3;
        uint4 oct_cur = fetch_octet(cur8), oct_nxt = fetch_octet(cur8 + 1);
        // Dequantise this lane's half of one stage of its row into the B tile.
        auto xform = [&](int kb, const uint4& q) -> bool {
          const int s = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          ++it;
          // this lane's group and its partner's (the other half of the row)
          const int g = (kb * kBK + 32 * half) / G;
          const int gp = (kb * kBK + 32 * (half ^ 1)) / G;
          if ((g >> 3) != cur8) {  // both lanes of a pair enter a new octet together
            cur8 = g >> 3;
            oct_cur = oct_nxt;
            oct_nxt = fetch_octet(cur8 + 1);
          }
          const uint32_t mine = pick(oct_cur, g & 7);
          const uint32_t other = __shfl_xor_sync(0xffffffffu, pick(oct_cur, gp & 7), 1);
          // scale and offset as bf16 pairs (both columns of a pair share a group)
          const uint32_t s2 = (half ? other : mine) * 0x10001u;
          const uint32_t o2 = (half ? mine : other) * 0x10001u;
          if (!mbar_wait_warp(empty(s), ph ^ 1u, abort_flag, dev_status, wait_ns)) return false;
          const uint32_t brow = stage_b(s) + (uint32_t)rloc * 128u;
          const uint32_t words[4] = {q.x, q.y, q.z, q.w};
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            // the 8 codes of word j (columns k + 8j .. k + 8j + 7), looked up 4 at a time
            uint32_t lut_pair[4];
            lookup8(words[j], tl, th, lut_pair);
            uint32_t out[4];
  #pragma unroll
            for (int p = 0; p < 4; ++p) {
              // W' = LUT * scale + offset for both codes of the pair with one bf16x2
              // fused multiply-add (the exact value rounded once to bf16)
              asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(out[p]) : "r"(lut_pair[p]), "r"(s2), "r"(o2));
            }
            // 16-byte chunk (4 half + j) of the 128-byte row, 128-byte swizzle
            const uint32_t chunk = (uint32_t)((4 * half + j) ^ (rloc & 7));
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};"
                         :: "r"(brow + chunk * 16u), "r"(out[0]), "r"(out[1]), "r"(out[2]),
                            "r"(out[3]) : "memory");
          }
          fence_proxy_async_smem();  // make the generic-proxy stores visible to the MMA
          __syncwarp();
          if (lane == 0) mbar_arrive(full_b(s));
          return true;
        };

        uint4 pa = fetch(kb0), pb = make_uint4(0u, 0u, 0u, 0u), pc = pb;
        if (kb0 + 1 < kb1) pb = fetch(kb0 + 1);
        if (kb0 + 2 < kb1) pc = fetch(kb0 + 2);
        bool alive = true;
        for (int kb = kb0; kb < kb1 && alive; kb += 3) {
          alive = xform(kb, pa);
          if (alive && kb + 3 < kb1) pa = fetch(kb + 3);
          if (alive && kb + 1 < kb1) {
            alive = xform(kb + 1, pb);
            if (alive && kb + 4 < kb1) pb = fetch(kb + 4);
          }
          if (alive && kb + 2 < kb1) {
            alive = xform(kb + 2, pc);
            if (alive && kb + 5 < kb1) pc = fetch(kb + 5);
          }
        }
        if (!alive) goto done;
      }

      // epilogue: TMEM -> registers; then either this segment's fp32 partial
      // sums go to the workspace (a segment that does not start the tile), or
      // the partials of the tile's later segments are added (in block order)
      // and the bf16 result is written to y.
      if (!mbar_wait_warp(accum_full, tcount & 1u, abort_flag, dev_status, wait_ns)) goto done;
      tc_fence_after();
      {
        const int quad = warp & 3;       // TMEM lanes 32*quad .. 32*quad+31
        const int hacc = (tw >> 2) & 1;  // which accumulator
        const int cpart = tw >> 3;       // which half of the 256 columns
        const int mloc = hacc * kBM + quad * 32 + lane;  // row within the 256-row tile
        const int m = mt * kNAcc * kBM + mloc;
        const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(hacc * kBN);
        const bool first = kb0 == 0;
        const bool last = kb1 == nkb;
        // blocks holding the later segments of this tile (stream-K), waited for
        // once each; they do not depend on this block, so the waits end
        int c_end = (int)blockIdx.x + 1;
        if (first && !last) {
          const int64_t tile_end = (int64_t)(tile + 1) * nkb;
          while (c_end < (int)gridDim.x && U * c_end / gridDim.x < tile_end) {
            if (lane == 0) {
              const unsigned long long t0 = globaltimer();
              uint32_t f = 0;
              for (uint32_t i = 0;; ++i) {
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                             : "=r"(f) : "l"(ws_flags + c_end) : "memory");
                if (f != 0u) break;
                if ((i & 63u) == 0u && (*abort_flag || globaltimer() - t0 > wait_ns)) {
                  *abort_flag = 1;
                  report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
                  break;
                }
              }
            }
            __syncwarp();
            ++c_end;
          }
          if (__any_sync(0xffffffffu, *abort_flag != 0)) goto done;
          __threadfence();  // the partials below are read after their flags
        }
        // 16 columns at a time: this warp's 32 rows x 128 columns
        for (int cc = cpart * (kBN / 32); cc < (cpart + 1) * (kBN / 32); ++cc) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(tbase + (uint32_t)(cc * 16), r);
          tmem_wait_ld();
          if (!first) {
            float4* dst = reinterpret_cast<float4*>(ws_partial) +
                          partial_index(blockIdx.x, tw, cc - cpart * (kBN / 32), lane);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[32 * v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            continue;
          }
          float acc[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = __uint_as_float(r[i]);
          for (int c = (int)blockIdx.x + 1; c < c_end; ++c) {
            const float4* src = reinterpret_cast<const float4*>(ws_partial) +
                                partial_index(c, tw, cc - cpart * (kBN / 32), lane);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 q = __ldcg(src + 32 * v);  // written by another SM: read through L2
              acc[4 * v] += q.x; acc[4 * v + 1] += q.y; acc[4 * v + 2] += q.z; acc[4 * v + 3] += q.w;
            }
          }
          const int n0 = nt * kBN + cc * 16;
          if (m < M && y32 != nullptr) {
            // the unrounded fp32 sums
            float* yr = y32 + (int64_t)m * N;
            for (int i = 0; i < 16; ++i)
              if (n0 + i < N) yr[n0 + i] = acc[i];
          } else if (m < M) {
            uint16_t* yr = y + (int64_t)m * N;
            if (vec_store && n0 + 16 <= N) {
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                const uint4 w = make_uint4(pack_bf16x2_rn(acc[8 * v + 0], acc[8 * v + 1]),
                                           pack_bf16x2_rn(acc[8 * v + 2], acc[8 * v + 3]),
                                           pack_bf16x2_rn(acc[8 * v + 4], acc[8 * v + 5]),
                                           pack_bf16x2_rn(acc[8 * v + 6], acc[8 * v + 7]));
                *reinterpret_cast<uint4*>(yr + n0 + 8 * v) = w;
              }
            } else {
              for (int i = 0; i < 16; ++i)
                if (n0 + i < N) yr[n0 + i] = f32_to_bf16_rn(acc[i]);
            }
          }
        }
        if (!first) {
          // this block's partial is complete once all dequant warps have stored
          // their part: the last one to finish publishes the flag
          __threadfence();
          __syncwarp();
          if (lane == 0 && atomicAdd(partial_done, 1) == kXformWarps - 1) {
            __threadfence();
            asm volatile("st.release.gpu.global.u32 [%0], %1;"
                         :: "l"(ws_flags + blockIdx.x), "r"(1u) : "memory");
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accum_empty);
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // tensor loads issued but never seen complete may still be writing the
    // stages: wait for them (bounded) before the block's shared memory is freed
    for (uint32_t it = *n_landed; it < *n_issued; ++it) {
      const int s = (int)(it % kStages);
      const uint32_t ph = (it / kStages) & 1u;
      const unsigned long long t0 = globaltimer();
      while (!(mbar_try_wait(full_a(s), ph) && (!kWTma || mbar_try_wait(full_b(s), ph))))
        if (globaltimer() - t0 > kWaitLimitNs) break;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// Workspace: one fp32 256 x 256 partial tile per block (stream-K) followed by
// one flag word per block.
int prefill_slots() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
    return sms;
  return 160;
}

size_t prefill_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G) {
  (void)M; (void)N; (void)K; (void)G;
  const size_t slots = (size_t)prefill_slots();
  return slots * (size_t)(kNAcc * kBM) * kBN * sizeof(float) + ((slots * 4 + 255) / 256) * 256;
}

namespace {

// Shared launcher of both kernel modes; w_bf16 is the dequantised weight
// matrix (kWTma) or unused.
template <bool kWTma>
any4_status launch_prefill_impl(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                                int64_t lut_row_stride, const uint16_t* scale,
                                const uint16_t* offset, const uint16_t* w_bf16, uint16_t* y,
                                float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                bool test_stall, cudaStream_t stream, const DeviceInfo& dev) {
  if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return ANY4_ERR_SHAPE;
  if (dev.smem_optin < (size_t)kSmemAlloc) return ANY4_ERR_UNSUPPORTED;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return ANY4_ERR_UNSUPPORTED;

  // x [M][K] in 128 x 64 boxes; W [N][K] (bf16, two-pass mode) in 256 x 64
  // boxes; both 128-byte swizzled, the layout the MMA descriptors read
  CUtensorMap map, map_w;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ANY4_ERR_CUDA;
  }
  map_w = map;
  if (kWTma) {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
    if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(w_bf16), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ANY4_ERR_CUDA;
  }

  if (ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_kernel<kWTma>), kSmemAlloc) !=
      ANY4_OK)
    return ANY4_ERR_CUDA;

  const int64_t tiles = ((M + kNAcc * kBM - 1) / (kNAcc * kBM)) * ((N + kBN - 1) / kBN);
  const int64_t units = tiles * ((K + kBK - 1) / kBK);
  // every block keeps at least 4 stages of work
  const int64_t slots = prefill_slots();
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>({units / 4, (int64_t)dev.sm_count,
                                                                slots}));
  const size_t partial_bytes = (size_t)slots * (kNAcc * kBM) * kBN * sizeof(float);
  if (workspace_bytes < prefill_workspace_size(M, N, K, G) || workspace == nullptr)
    return ANY4_ERR_WORKSPACE;
  float* ws_partial = static_cast<float*>(workspace);
  uint32_t* ws_flags = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + partial_bytes);
  if (cudaMemsetAsync(ws_flags, 0, (size_t)grid * sizeof(uint32_t), stream) != cudaSuccess)
    return ANY4_ERR_CUDA;
  const int vec_store = (N % 8 == 0) ? 1 : 0;
  // Blocks wait on blocks with larger indices for their partial sums: all
  // blocks must be resident at once, which the cooperative launch guarantees
  // (one block fits per SM and the grid is at most the SM count).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, prefill_kernel<kWTma>, map, map_w, packed, lut, lut_row_stride,
                         scale, offset, y, y32, (int)M, (int)N, (int)K, (int)G, vec_store,
                         dev_status,
                         ws_partial, ws_flags, test_stall ? 1 : 0) != cudaSuccess)
    return ANY4_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

any4_status launch_prefill(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                           int64_t N, int64_t K, int64_t G, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, bool test_stall,
                           cudaStream_t stream, const DeviceInfo& dev) {
  return launch_prefill_impl<false>(x, packed, lut, lut_row_stride, scale, offset, nullptr, y,
                                    y32, M, N, K, G, workspace, workspace_bytes, dev_status,
                                    test_stall, stream, dev);
}

// Two passes for large M: the weights are dequantised once into the
// workspace (bf16, bit-exact with any4_dequant) and the tensor-core kernel
// streams them with TMA, so every weight is dequantised once instead of once
// per 256 rows of x.
bool prefill_use_two_pass(int64_t M, int64_t N, int64_t K) {
  (void)N; (void)K;
  return M >= 1024;
}

size_t prefill_two_pass_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G) {
  return prefill_workspace_size(M, N, K, G) + (((size_t)N * K * 2 + 255) / 256) * 256;
}

any4_status launch_prefill_two_pass(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                                    int64_t lut_row_stride, const uint16_t* scale,
                                    const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                                    int64_t N, int64_t K, int64_t G, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, bool test_stall,
                                    cudaStream_t stream, const DeviceInfo& dev) {
  if (workspace == nullptr || workspace_bytes < prefill_two_pass_workspace_size(M, N, K, G))
    return ANY4_ERR_WORKSPACE;
  const size_t fused = prefill_workspace_size(M, N, K, G);
  uint16_t* w = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + fused);
  // plain write-back stores: the GEMM pass reads W next, and what of it
  // stays in L2 is not read from DRAM again
  any4_status st = launch_dequant(packed, lut, lut_row_stride, scale, offset, w, N, K, G, stream,
                                  dev, /*streaming=*/false);
  if (st != ANY4_OK) return st;
  return launch_prefill_impl<true>(x, packed, lut, lut_row_stride, scale, offset, w, y, y32, M, N,
                                   K, G, workspace, fused, dev_status, test_stall, stream, dev);
}

// The same two passes for codes of 2 or 3 bits: the n-bit dequant kernel
// fills the workspace with bf16 weights, then the same tensor-core pass.
any4_status launch_prefill_two_pass_bits(const uint16_t* x, const uint8_t* packed,
                                         const uint16_t* lut, int64_t lut_row_stride,
                                         const uint16_t* scale, const uint16_t* offset,
                                         uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K,
                                         int64_t G, int bits, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status,
                                         bool test_stall, cudaStream_t stream,
                                         const DeviceInfo& dev) {
  if (workspace == nullptr || workspace_bytes < prefill_two_pass_workspace_size(M, N, K, G))
    return ANY4_ERR_WORKSPACE;
  const size_t fused = prefill_workspace_size(M, N, K, G);
  uint16_t* w = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + fused);
  any4_status st = launch_dequant_bits(packed, lut, lut_row_stride, scale, offset, w, N, K, G,
                                       bits, stream, dev);
  if (st != ANY4_OK) return st;
  return launch_prefill_impl<true>(x, packed, lut, lut_row_stride, scale, offset, w, y, y32, M, N,
                                   K, G, workspace, fused, dev_status, test_stall, stream, dev);
}

}  // namespace any4
