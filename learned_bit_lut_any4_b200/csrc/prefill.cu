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
//               packed fp32x2 fused multiply-add, rounded to bf16 (exactly the
//               dequant definition) and stored into the row of the B tile in
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
constexpr int kSmemUsed = kMiscOff + 16;
constexpr int kSmemAlloc = kSmemUsed + 1024;    // slack to align the base to 1 KB
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr unsigned long long kWaitLimitNs = 2000000000ull;

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
                                          int32_t* dev_status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(bar) : "memory");
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
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// The 4-bit code at bit `pos` of w, moved to bits 10..13 (a byte offset of
// code * 1024 into the transposed table); pos is a compile-time constant.
__device__ __forceinline__ uint32_t code_at_bit10(uint32_t w, int pos) {
  return (pos <= 10 ? (w << (10 - pos)) : (w >> (pos - 10))) & 0x3C00u;
}

// Table lookup in registers, no memory traffic: tl/th are the low/high byte
// planes of a 16-entry bf16 table (tl[i] holds the low bytes of entries
// 4i..4i+3).  For the 8 codes of w (code i at bits 4i..4i+3) returns the 8
// entries as 4 bf16 pairs, pair p = (entry of code 2p) | (entry of code 2p+1) << 16.
// Per 4 codes: byte permutes pick each byte from entries 0..7 and 8..15 by the
// code's low 3 bits, a sign-replicating permute turns each code's bit 3 into a
// byte mask, and a bitwise select keeps the right half-table's byte.
__device__ __forceinline__ void lookup8(uint32_t w, const uint32_t (&tl)[4],
                                        const uint32_t (&th)[4], uint32_t (&pair)[4]) {
  const uint32_t u = w << 4;  // bit 3 of codes 0, 2, 4, 6 into byte sign bits
#pragma unroll
  for (int hv = 0; hv < 2; ++hv) {
    const uint32_t sel = (hv ? (w >> 16) : w) & 0x7777u;
    // prmt's default mode: a selector nibble with bit 3 set replicates the
    // sign bit of the chosen byte (the __byte_perm intrinsic ignores bit 3)
    uint32_t m;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(u), "r"(w), "r"(hv ? 0xFBEAu : 0xD9C8u));
    const uint32_t x0 = __byte_perm(tl[0], tl[1], sel), x1 = __byte_perm(tl[2], tl[3], sel);
    const uint32_t y0 = __byte_perm(th[0], th[1], sel), y1 = __byte_perm(th[2], th[3], sel);
    const uint32_t lo = (x0 & ~m) | (x1 & m);
    const uint32_t hi = (y0 & ~m) | (y1 & m);
    pair[2 * hv] = __byte_perm(lo, hi, 0x5140u);
    pair[2 * hv + 1] = __byte_perm(lo, hi, 0x7362u);
  }
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

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ lut, int64_t lut_row_stride,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ y, int M, int N, int K, int G, int vec_store, int32_t* dev_status) {
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

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_a(s), 1);
      mbar_init(full_b(s), kXformWarps);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum_full, 1);
    mbar_init(accum_empty, kXformWarps);
    *abort_flag = 0;
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

  if (warp == 0) {
    // ------------------------------------------------ x tiles via TMA
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int mt = tile % n_mtiles;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(empty(s), ph ^ 1u, abort_flag, dev_status)) goto done;
          mbar_arrive_expect_tx(full_a(s), kNAcc * kATileBytes);
          for (int h = 0; h < kNAcc; ++h)
            tma_load_2d(stage_a(s, h), &tmap_x, kb * kBK, mt * kNAcc * kBM + h * kBM, full_a(s));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue (one thread)
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
        if (tcount > 0 && !mbar_wait(accum_empty, (tcount - 1) & 1u, abort_flag, dev_status))
          goto done;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(full_a(s), ph, abort_flag, dev_status)) goto done;
          if (!mbar_wait(full_b(s), ph, abort_flag, dev_status)) goto done;
          tc_fence_after();
          const uint64_t db = smem_desc_sw128(stage_b(s));
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j) {
#pragma unroll
            for (int h = 0; h < kNAcc; ++h) {
              const uint64_t da = smem_desc_sw128(stage_a(s, h));
              // advance 16 columns = 32 bytes = 2 descriptor units
              tc_mma(tmem + (uint32_t)(h * kBN), da + 2u * j, db + 2u * j, kIdesc,
                     (kb > 0 || j > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty(s));  // stage s free once these MMAs have read it
        }
        tc_commit(accum_full);  // accumulators of this tile complete
      }
    }
  } else {
    // ------------------------------------------------ dequant + epilogue
    const int tw = warp - 2;                         // 0 .. 15
    const int half = tw >> 3;                        // which 32 codes of a stage
    const int rloc = (tw & 7) * 32 + lane;           // weight row within the tile
    const int64_t row_bytes = K / 2;
    const int groups = K / G;
    uint32_t it = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
      const int mt = tile % n_mtiles;
      const int nt = tile / n_mtiles;
      const int n = nt * kBN + rloc;
      const bool rin = n < N;
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
      const uint16_t* srow = scale + (int64_t)(rin ? n : 0) * groups;
      const uint16_t* orow = offset + (int64_t)(rin ? n : 0) * groups;

      // This lane's 32 codes of a stage and their group's scale/offset,
      // fetched three stages ahead.
      struct Payload {
        uint4 q;
        float s, o;
      };
      auto fetch = [&](int kb, Payload& pl) {
        const int k = kb * kBK + 32 * half;
        const bool kin = rin && k < K;
        pl.q = kin ? ldg_stream_v4(prow + k / 2) : make_uint4(0u, 0u, 0u, 0u);
        pl.s = kin ? bf16_lo_to_f32(ldg_u16(srow + k / G)) : 0.f;
        pl.o = kin ? bf16_lo_to_f32(ldg_u16(orow + k / G)) : 0.f;
      };
      // Dequantise this lane's half of one stage of its row into the B tile.
      auto xform = [&](int kb, const Payload& pl) -> bool {
        const int s = (int)(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        ++it;
        if (!mbar_wait(empty(s), ph ^ 1u, abort_flag, dev_status)) return false;
        const uint32_t brow = stage_b(s) + (uint32_t)rloc * 128u;
        const uint32_t words[4] = {pl.q.x, pl.q.y, pl.q.z, pl.q.w};
        unsigned long long s2, o2;
        asm("mov.b64 %0, {%1, %1};" : "=l"(s2) : "f"(pl.s));
        asm("mov.b64 %0, {%1, %1};" : "=l"(o2) : "f"(pl.o));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // the 8 codes of word j (columns k + 8j .. k + 8j + 7), looked up 4 at a time
          uint32_t lut_pair[4];
          lookup8(words[j], tl, th, lut_pair);
          uint32_t out[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            // W' = bf16(fmaf(LUT, s, o)) for both codes of the pair, one packed fp32x2 FMA
            const float l0 = bf16_lo_to_f32(lut_pair[p]);
            const float l1 = bf16_hi_to_f32(lut_pair[p]);
            unsigned long long vv, r;
            asm("mov.b64 %0, {%1, %2};" : "=l"(vv) : "f"(l0), "f"(l1));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(vv), "l"(s2), "l"(o2));
            float r0, r1;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
            out[p] = pack_bf16x2_rn(r0, r1);  // zeros past K (codes 0, scale 0, offset 0)
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

      Payload pa, pb, pc;
      fetch(0, pa);
      if (nkb > 1) fetch(1, pb);
      if (nkb > 2) fetch(2, pc);
      bool alive = true;
      for (int kb = 0; kb < nkb && alive; kb += 3) {
        alive = xform(kb, pa);
        if (alive && kb + 3 < nkb) fetch(kb + 3, pa);
        if (alive && kb + 1 < nkb) {
          alive = xform(kb + 1, pb);
          if (alive && kb + 4 < nkb) fetch(kb + 4, pb);
        }
        if (alive && kb + 2 < nkb) {
          alive = xform(kb + 2, pc);
          if (alive && kb + 5 < nkb) fetch(kb + 5, pc);
        }
      }
      if (!alive) goto done;

      // epilogue: TMEM -> registers -> bf16 -> y
      if (!mbar_wait(accum_full, tcount & 1u, abort_flag, dev_status)) goto done;
      tc_fence_after();
      {
        const int quad = warp & 3;       // TMEM lanes 32*quad .. 32*quad+31
        const int hacc = (tw >> 2) & 1;  // which accumulator
        const int cpart = tw >> 3;       // which half of the 256 columns
        const int m = mt * kNAcc * kBM + hacc * kBM + quad * 32 + lane;
        const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(hacc * kBN);
        for (int cc = cpart * (kBN / 64); cc < (cpart + 1) * (kBN / 64); ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + (uint32_t)(cc * 32), r);
          tmem_wait_ld();
          const int n0 = nt * kBN + cc * 32;
          if (m < M) {
            uint16_t* yr = y + (int64_t)m * N;
            if (vec_store && n0 + 32 <= N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const uint4 w = make_uint4(
                    pack_bf16x2_rn(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1])),
                    pack_bf16x2_rn(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                    pack_bf16x2_rn(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                    pack_bf16x2_rn(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
                *reinterpret_cast<uint4*>(yr + n0 + 8 * v) = w;
              }
            } else {
              for (int i = 0; i < 32; ++i)
                if (n0 + i < N) yr[n0 + i] = f32_to_bf16_rn(__uint_as_float(r[i]));
            }
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

size_t prefill_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G) {
  (void)M; (void)N; (void)K; (void)G;
  return 0;
}

any4_status launch_prefill(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                           int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, cudaStream_t stream, const DeviceInfo& dev) {
  (void)workspace; (void)workspace_bytes;
  if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return ANY4_ERR_SHAPE;
  if (dev.smem_optin < (size_t)kSmemAlloc) return ANY4_ERR_UNSUPPORTED;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return ANY4_ERR_UNSUPPORTED;

  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return ANY4_ERR_CUDA;

  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmemAlloc);
  });
  if (attr_err != cudaSuccess) return ANY4_ERR_CUDA;

  const int64_t tiles = ((M + kNAcc * kBM - 1) / (kNAcc * kBM)) * ((N + kBN - 1) / kBN);
  const int grid = (int)std::min<int64_t>(tiles, dev.sm_count);
  const int vec_store = (N % 8 == 0) ? 1 : 0;
  prefill_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(map, packed, lut, lut_row_stride, scale,
                                                         offset, y, (int)M, (int)N, (int)K,
                                                         (int)G, vec_store, dev_status);
  return cudaGetLastError() == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace any4
