// Decode-path any4 matmul for M <= 2 with pair-table lookups.
//
// Paper "any4: Learned 4-bit Numeric Representation for LLMs": §4.1 Eq. 8
// (y_i = sum_j dequant(w_Q[i,j]) x_j), §2.5.2 (dequant = alpha * w_Q + beta,
// here with the per-row table of §2.4.1), §4.2 (y = x w^T with x M x K and
// w N x K; two 4-bit codes per byte; memory bound at small M).
//
// The paper's kernel keeps a row's 16-entry table in a register and reads it
// with one warp shuffle per code.  On B200 a shuffle returns 32 values per
// clock per SM, below the ~33 weights per clock per SM that 80 % of the HBM
// bandwidth needs at 0.54 bytes per weight.  This kernel looks up two codes
// at once instead: a byte of packed codes (the even column in its low nibble)
// indexes a 256-entry table of bf16 PAIRS (LUT[c_even], LUT[c_odd]) built per
// row in shared memory, so one 32-bit shared-memory load serves two weights.
// Measured on B200 it beats the skinny kernel at M = 2 (17.5 against 21.9 us
// on 4096 -> 14336), which is where the decode path uses it; at M = 1 the
// weight-streaming shuffle kernel stays faster on every shape measured (the
// table builds and the cross-block exchange cost more than the halved lookup
// count saves), so M = 1 runs this kernel only on request.
//
//  * Row sets: a block works on 64 weight rows at a time; lane l of every warp
//    owns rows l and 32 + l of the set (row slots h = 0, 1).  The pair tables
//    are private to a lane: entry e of lane l, slot h sits at byte
//    (e << 8) | (h << 7) | (l << 2) of a 64 KiB-aligned table, so the lanes
//    of a warp always read 32 different banks (no conflicts, whatever the
//    codes) and the address is one byte permute of the code word.  The 8
//    warps of the block share the table (same lane, same rows) and split the
//    set's columns; the table is rebuilt when the block moves to the next set
//    (64 x 256 entries, each one byte permute and one store).
//  * Dequantisation: the pair (LUT[c0], LUT[c1]) times (s, s) plus (o, o) in
//    one bf16x2 fused multiply-add: LUT * s + o rounded once to bf16, which
//    equals bf16(fmaf(LUT, s, o)) unless that fp32 fmaf is inexact and lands
//    on a bf16 rounding tie.
//  * Products on the tensor core: mma.sync m16n8k16 with A rows g = lane's
//    row slot 0 and g + 8 = row slot 1 (four consecutive columns each), and
//    B holding x only at the k positions of lane (g, t) in column t (lanes
//    with g == t), so C[g][t] and C[g+8][t] are that lane's two rows' partial
//    sums; 256 weights per MMA, fp32 accumulation.  With M = 2 the second
//    row of x sits in columns 4..7 (lanes with g == t + 4).
//  * Weights stream through a per-warp ring of 4 stages filled by
//    cp.async.bulk.tensor (codes [64 rows][64 B] with the 64-byte swizzle, so
//    each lane's 16-byte reads are conflict free; x [M][128]).  The warps of
//    a block split a set's chunks into contiguous ranges.  A lane loads its
//    two rows' scales and offsets for the chunk itself (a few bytes, shared
//    with its neighbouring chunks through L1), one chunk ahead of their use.
//  * Work split (stream-K): the (row set, 128-column chunk) units are divided
//    evenly over the blocks (one per SM).  A block whose range starts inside
//    a row set publishes its 64 x M partial sums in the workspace and then
//    sets its flag to a fixed 64-bit marker; the block holding the set's
//    first chunk waits (bounded) for those markers, adds the partials in
//    block order (so the sums are deterministic) and puts each flag it
//    consumed back to 0.  A flag therefore holds the marker only between a
//    publication and its consumption within one launch, whatever the
//    workspace held before (any other value reads as "not yet"), and the
//    workspace needs no clearing.  (The launch's %gridid cannot serve as
//    the marker: replays of a CUDA graph reuse it.)  All other sets are
//    summed over the block's warps in shared memory in a fixed order.
//
// Every wait is bounded (about 2 s of %globaltimer); on expiry the kernel sets
// ANY4_ERR_TIMEOUT in dev_status, stops computing, and waits (bounded) for its
// own copies in flight before returning.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"

namespace any4 {
namespace {

constexpr int kPWarps = 8;
constexpr int kPThreads = kPWarps * 32;
constexpr int kPRows = 64;                          // rows of a set: two per lane
constexpr int kPChunk = 128;                        // columns per ring stage
constexpr int kPStages = 4;
constexpr int kPCodeBytes = kPRows * kPChunk / 2;   // 4096
constexpr int kPLutBytes = kPRows * 32;             // the set's 64 tables
constexpr uint32_t kPTableBytes = 65536;
constexpr unsigned long long kPWaitNs = 2000000000ull;
constexpr unsigned long long kPTestWaitNs = 1000000ull;  // the test-stall mode's limit
// a block's partial sums are published (any other flag value: not published)
constexpr unsigned long long kPPublished = 0x616E7934F1A65E7Dull;

template <int MT>
struct PLayout {
  static constexpr int kStage = ((kPCodeBytes + MT * kPChunk * 2 + 511) / 512) * 512;
  static constexpr uint32_t kTxCodes = kPCodeBytes;
  static constexpr uint32_t kTxX = MT * kPChunk * 2;
};

// Unit ranges of the blocks (block b: units ub[b] .. ub[b + 1] - 1), worked
// out on the host so that the kernel needs no 64-bit division.
constexpr int kPMaxGrid = 160;
struct PSched {
  int ub[kPMaxGrid + 1];
};

struct PMaps {
  CUtensorMap codes;   // u8 [N][K/2], box {64, 64}, 64-byte swizzle
  CUtensorMap x;       // bf16 [M][K], box {128, MT}
  CUtensorMap lut;     // bf16 [N][16], box {16, 64} (a table per row)
};

__device__ __forceinline__ uint32_t sa(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtime() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          unsigned long long limit) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtime();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63u) == 0u && gtime() - t0 > limit) return false;
  }
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(tx)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(tx)
               : "memory");
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                       uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// bf16 scale or offset pairs (s, s) of the 32-column sub-blocks of a chunk:
// one group for G = 128 (GS = 4), two for G = 64, four for G = 32.  The raw
// 2, 4 or 8 bytes of a row's groups of the chunk sit in `raw` (2 words).
template <int GS>
__device__ __forceinline__ uint32_t group_dup(const uint2& raw, int sub) {
  const int q = sub / GS;  // group of the sub-block within the chunk
  const uint32_t w = (q & 2) ? raw.y : raw.x;
  return prmt(w, 0u, (q & 1) ? 0x3232u : 0x1010u);
}
template <int GS>
__device__ __forceinline__ uint2 load_groups(const uint16_t* p) {
  if constexpr (GS == 4) return make_uint2((uint32_t)ldg_u16(p), 0u);
  if constexpr (GS == 2) return make_uint2(__ldg(reinterpret_cast<const uint32_t*>(p)), 0u);
  return __ldg(reinterpret_cast<const uint2*>(p));
}

// The block's units [u0, u1) of the flattened (row set, chunk) space and the
// chunks of row set r that warp w handles: an eighth of the block's chunks
// of the set, contiguous (each warp streams long runs of its rows).
struct PRange {
  int u0, u1;  // units of the block (fewer than 2^31: N K / 8192 <= 2^27)
  int KC;
  __device__ void warp_chunks(int r, int w, int& lo, int& hi) const {
    const int base = r * KC;
    const int cl = (u0 > base ? u0 : base) - base;
    const int n = (u1 < base + KC ? u1 : base + KC) - base - cl;
    lo = cl + (n * w) / kPWarps;
    hi = cl + (n * (w + 1)) / kPWarps;
  }
};

// The sequence of (row set, chunk) items of one warp, in consumption order.
struct PIter {
  PRange rg;
  int warp;
  int r, r_last;
  int c, c_hi;
  __device__ void start(const PRange& range, int w) {
    rg = range;
    warp = w;
    r = range.u0 / range.KC;
    r_last = (range.u1 - 1) / range.KC;
    range.warp_chunks(r, w, c, c_hi);
    skip();
  }
  __device__ void skip() {
    while (r <= r_last && c >= c_hi) {
      ++r;
      if (r <= r_last) rg.warp_chunks(r, warp, c, c_hi);
    }
  }
  __device__ bool valid() const { return r <= r_last; }
  __device__ void next() {
    ++c;
    skip();
  }
};

template <int MT, int GS>  // rows of x (1, 2); G / 32 (1, 2, 4)
__global__ void __launch_bounds__(kPThreads, 1) decode_pair_kernel(
    const __grid_constant__ PMaps maps, const uint16_t* __restrict__ lut_shared,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
    uint16_t* __restrict__ y, float* __restrict__ y32, int N, int K, int KC,
    const __grid_constant__ PSched sched,
    float* __restrict__ ws_part, unsigned long long* __restrict__ ws_flag, int dyn_bytes,
    int32_t* dev_status, int test_stall) {
  using L = PLayout<MT>;
  constexpr int kGPC = 4 / GS;  // groups per 128-column chunk
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // test_stall: warp 0 of block 0 stops its weight stream after one item, so
  // its next wait runs out (1 ms limit) and the kernel ends cleanly
  const unsigned long long wait_ns = test_stall ? kPTestWaitNs : kPWaitNs;
  const bool stalled = test_stall && blockIdx.x == 0 && warp == 0;
  if (threadIdx.x == 0) {
    // fetch the tensor-map descriptors now rather than at each first use
    asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.codes) : "memory");
    asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.x) : "memory");
    if (lut_shared == nullptr)
      asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.lut) : "memory");
  }

  // ---- shared-memory layout: the 64 KiB-aligned pair table, then everything
  // else first-fit in the space below and above it
  const uint32_t base = sa(smem);
  const uint32_t end = base + (uint32_t)dyn_bytes;
  const uint32_t tab = (base + 0xFFFFu) & ~0xFFFFu;
  uint32_t lo_ptr = base, hi_ptr = tab + kPTableBytes;
  bool fits = tab + kPTableBytes <= end;
  auto alloc = [&](uint32_t bytes, uint32_t align) -> uint32_t {
    uint32_t a = (lo_ptr + align - 1) & ~(align - 1);
    if (a + bytes <= tab) { lo_ptr = a + bytes; return a; }
    a = (hi_ptr + align - 1) & ~(align - 1);
    if (a + bytes <= end) { hi_ptr = a + bytes; return a; }
    fits = false;
    return 0u;
  };
  uint32_t my_stage0 = 0;
  for (int w = 0; w < kPWarps; ++w) {  // per warp: kPStages stages of L::kStage bytes
    const uint32_t a = alloc(kPStages * L::kStage, 512);
    if (w == warp) my_stage0 = a;
  }
  const uint32_t lutbuf = alloc(2 * kPLutBytes, 128);
  const uint32_t part = alloc(kPWarps * MT * kPRows * 4, 16);
  const uint32_t bars = alloc((kPWarps * kPStages + 2) * 8, 8);
  const uint32_t flags = alloc(16, 16);
  if (!fits) {  // cannot happen with the launch's dynamic size; checked, not assumed
    if (threadIdx.x == 0) report_status(dev_status, (int32_t)ANY4_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* const gsm = smem - base;  // generic pointer of shared address a: gsm + a
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + flags);
  volatile int* late_flag = reinterpret_cast<volatile int*>(gsm + flags + 4);
  float* const s_part = reinterpret_cast<float*>(gsm + part);
  const uint32_t my_bars = bars + 8u * (uint32_t)(warp * kPStages);
  const uint32_t lut_bars = bars + 8u * (uint32_t)(kPWarps * kPStages);

  if (threadIdx.x == 0) *abort_flag = 0;
  if (lane == 0) {
    for (int s = 0; s < kPStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(my_bars + 8u * s) : "memory");
    if (warp == 0)
      for (int s = 0; s < 2; ++s)
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(lut_bars + 8u * s)
                     : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  PRange rg;
  rg.KC = KC;
  rg.u0 = sched.ub[blockIdx.x];
  rg.u1 = sched.ub[blockIdx.x + 1];
  const int r_first = rg.u0 / KC, r_last = (rg.u1 - 1) / KC;
  const int nsets = (int)(r_last - r_first + 1);

  // ---- producer state (lane 0 of each warp): items issued ahead of use
  PIter pit;
  pit.start(rg, warp);
  int issued = 0;
  auto issue = [&](int consumed, bool with_x) {
    while (pit.valid() && issued < consumed + kPStages && !(stalled && issued >= 1)) {
      const int st = issued % kPStages;
      const uint32_t dst = my_stage0 + (uint32_t)(st * L::kStage);
      const uint32_t bar = my_bars + 8u * st;
      const uint32_t tx = L::kTxCodes + L::kTxX;
      if (with_x) {
        mbar_arrive_expect(bar, tx);
      } else {
        mbar_expect(bar, tx);  // the arrival comes once x is issued too
      }
      tma_2d(dst, &maps.codes, pit.c * (kPChunk / 2), (int)(pit.r * kPRows), bar);
      if (with_x) tma_2d(dst + kPCodeBytes, &maps.x, pit.c * kPChunk, 0, bar);
      ++issued;
      pit.next();
    }
  };
  // table loads (warp 0, lane 0): the LUT box of set s goes to slot s & 1
  auto issue_lut = [&](int s) {
    if (lut_shared != nullptr || s >= nsets) return;
    const uint32_t bar = lut_bars + 8u * (uint32_t)(s & 1);
    mbar_arrive_expect(bar, (uint32_t)kPLutBytes);
    tma_2d(lutbuf + (uint32_t)((s & 1) * kPLutBytes), &maps.lut, 0, (int)((r_first + s) * kPRows),
           bar);
  };

  // weights (codes, tables) may stream before the preceding kernel finishes;
  // x is read and y written only after griddepcontrol.wait
  int early = 0;
  if (lane == 0) {
    if (warp == 0) {
      issue_lut(0);
      issue_lut(1);
    }
    issue(0, false);
    early = issued;
  }
  // the scales and offsets of a lane's two rows for one item: rows
  // r * 64 + lane and r * 64 + 32 + lane, the chunk's groups (zeros past N)
  const int groups = K / (32 * GS);
  auto load_so = [&](int r, int c, uint2 (&so)[4]) {
    const int ra = r * kPRows + lane, rb = ra + 32;
    const int g0 = c * kGPC;
#pragma unroll
    for (int i = 0; i < 4; ++i) so[i] = make_uint2(0u, 0u);
    if (ra < N) {
      so[0] = load_groups<GS>(scale + (int64_t)ra * groups + g0);
      so[1] = load_groups<GS>(offset + (int64_t)ra * groups + g0);
    }
    if (rb < N) {
      so[2] = load_groups<GS>(scale + (int64_t)rb * groups + g0);
      so[3] = load_groups<GS>(offset + (int64_t)rb * groups + g0);
    }
  };
  PIter cit;  // the consumer's copy of the item sequence (all lanes)
  cit.start(rg, warp);
  uint2 so_next[4];
  if (cit.valid()) load_so(cit.r, cit.c, so_next);

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (lane == 0) {
    PIter it;  // the early items again, for their chunk index
    it.start(rg, warp);
    for (int i = 0; i < early; ++i, it.next()) {
      const int st = i % kPStages;
      tma_2d(my_stage0 + (uint32_t)(st * L::kStage) + kPCodeBytes, &maps.x, it.c * kPChunk, 0,
             my_bars + 8u * st);
      mbar_arrive(my_bars + 8u * st);
    }
  }

  const int g = lane >> 2, t = lane & 3;
  // lanes that carry x in the B operand: x row m = g >> 2 in column t
  const bool xlane = (g & 3) == t && (g >> 2) < MT;
  const uint32_t xoff = (uint32_t)((g >> 2) * kPChunk * 2);
  const uint32_t lb0 = tab | (uint32_t)(lane << 2);
  const uint32_t lb1 = tab | 128u | (uint32_t)(lane << 2);
  // 16-byte unit j of a lane's code row sits at unit j ^ swz (64-byte swizzle);
  // both of its rows (lane, 32 + lane) share it
  const uint32_t swz = (uint32_t)((lane >> 1) & 3);

  bool ok = true;
  int item = 0;

  for (int s = 0; s < nsets; ++s) {
    const int r = r_first + s;
    // ---- the pair tables of this set: warp w builds entries 32w .. 32w+31
    {
      uint32_t la[8], lb[8], lwa, lwb;
      if (lut_shared != nullptr) {
        const uint4 e0 = ldg_nc_v4(lut_shared), e1 = ldg_nc_v4(lut_shared + 8);
        la[0] = e0.x; la[1] = e0.y; la[2] = e0.z; la[3] = e0.w;
        la[4] = e1.x; la[5] = e1.y; la[6] = e1.z; la[7] = e1.w;
#pragma unroll
        for (int i = 0; i < 8; ++i) lb[i] = la[i];
        lwa = lwb = la[0];
#pragma unroll
        for (int i = 1; i < 8; ++i)
          if (i == warp) lwa = lwb = la[i];
      } else {
        const uint32_t bar = lut_bars + 8u * (uint32_t)(s & 1);
        if (!mbar_wait(bar, (uint32_t)((s >> 1) & 1), wait_ns)) {
          if (lane == 0) report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        }
        const uint32_t lt = lutbuf + (uint32_t)((s & 1) * kPLutBytes);
        const uint4 a0 = lds128(lt + (uint32_t)(lane * 32)), a1 = lds128(lt + (uint32_t)(lane * 32 + 16));
        const uint4 b0 = lds128(lt + (uint32_t)((32 + lane) * 32));
        const uint4 b1 = lds128(lt + (uint32_t)((32 + lane) * 32 + 16));
        la[0] = a0.x; la[1] = a0.y; la[2] = a0.z; la[3] = a0.w;
        la[4] = a1.x; la[5] = a1.y; la[6] = a1.z; la[7] = a1.w;
        lb[0] = b0.x; lb[1] = b0.y; lb[2] = b0.z; lb[3] = b0.w;
        lb[4] = b1.x; lb[5] = b1.y; lb[6] = b1.z; lb[7] = b1.w;
        lwa = lds32(lt + (uint32_t)(lane * 32 + warp * 4));
        lwb = lds32(lt + (uint32_t)((32 + lane) * 32 + warp * 4));
      }
      // entry e = 32 warp + j: low half LUT[e & 15], high half LUT[e >> 4]
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint32_t sel = ((j >> 4) ? 0x7600u : 0x5400u) | ((j & 1) ? 0x32u : 0x10u);
        const uint32_t e = (uint32_t)(32 * warp + j);
        sts32(lb0 | (e << 8), prmt(la[(j & 15) >> 1], lwa, sel));
        sts32(lb1 | (e << 8), prmt(lb[(j & 15) >> 1], lwb, sel));
      }
    }
    __syncthreads();  // the table is complete; the LUT slot of set s is free
    if (threadIdx.x == 0) issue_lut(s + 2);

    // ---- this warp's chunks of the set
    float acc[MT == 1 ? 4 : 2][4];
#pragma unroll
    for (int q = 0; q < (MT == 1 ? 4 : 2); ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[q][i] = 0.f;
    while (cit.valid() && cit.r == r) {
      const int c = cit.c;
      uint2 so[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) so[i] = so_next[i];
      cit.next();  // the next item's scales and offsets, one item ahead
      if (cit.valid()) load_so(cit.r, cit.c, so_next);
      // after an abort the remaining items are skipped, not consumed: the
      // drain at the end waits for the copies of those already issued
      if (*abort_flag != 0) ok = false;
      if (!ok) continue;
      const int st = item % kPStages;
      if (!mbar_wait(my_bars + 8u * st, (uint32_t)((item / kPStages) & 1), wait_ns)) {
        if (lane == 0) report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
        *abort_flag = 1;
        ok = false;
        continue;
      }
      const uint32_t sp = my_stage0 + (uint32_t)(st * L::kStage);
      const uint32_t rowa = sp + (uint32_t)(lane * 64), rowb = rowa + 32u * 64u;
      const int nsub = min(4, (K - c * kPChunk) / 32);  // K % 32 == 0
#pragma unroll 1
      for (int sub = 0; sub < nsub; ++sub) {
        const uint32_t sa2 = group_dup<GS>(so[0], sub), oa2 = group_dup<GS>(so[1], sub);
        const uint32_t sb2 = group_dup<GS>(so[2], sub), ob2 = group_dup<GS>(so[3], sub);
        // codes of the lane's two rows, columns 32 sub .. 32 sub + 31
        const uint32_t ju = ((uint32_t)sub ^ swz) << 4;
        const uint4 qa = lds128(rowa + ju);
        const uint4 qb = lds128(rowb + ju);
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint4 xv = make_uint4(0u, 0u, 0u, 0u);
          if (xlane) xv = lds128(sp + kPCodeBytes + xoff + (uint32_t)((sub * 32 + wi * 8) * 2));
          uint32_t A[4], B[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint32_t sel = 0x7604u | ((uint32_t)p << 4);
            A[p] = hfma2_bf16(lds32(prmt(wa[wi], lb0, sel)), sa2, oa2);
            B[p] = hfma2_bf16(lds32(prmt(wb[wi], lb1, sel)), sb2, ob2);
          }
          if (MT == 1) {
            mma_bf16(acc[(2 * wi) & 3], A[0], B[0], A[1], B[1], xv.x, xv.y);
            mma_bf16(acc[(2 * wi + 1) & 3], A[2], B[2], A[3], B[3], xv.z, xv.w);
          } else {
            mma_bf16(acc[0], A[0], B[0], A[1], B[1], xv.x, xv.y);
            mma_bf16(acc[1], A[2], B[2], A[3], B[3], xv.z, xv.w);
          }
        }
      }
      ++item;
      // stage consumed: let the tensor loads refill it
      __syncwarp();
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(item, true);
      }
    }
    // ---- partial sums of the 64 rows (x MT) over this warp's chunks
    float tot[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < (MT == 1 ? 4 : 2); ++q) v += acc[q][i];
      tot[i] = v;
    }
    // C[g][2t + j] (j = 0, 1) is row slot 0 of lane 4g + 2(t & 1) + j for x row
    // t >> 1, C[g + 8][..] the same lanes' row slot 1
    if ((t >> 1) < MT) {
      const int m = t >> 1;
      float* dst = s_part + (size_t)(warp * MT + m) * kPRows;
      const int l0 = 4 * g + 2 * (t & 1);
      dst[l0] = tot[0];
      dst[l0 + 1] = tot[1];
      dst[32 + l0] = tot[2];
      dst[32 + l0 + 1] = tot[3];
    }
    // ---- the set's sums: fixed order over warps, then over blocks
    const int set_u0 = r * KC, set_u1 = set_u0 + KC;
    const bool starts = rg.u0 <= set_u0;  // this block holds chunk 0 of the set
    const bool whole = starts && rg.u1 >= set_u1;
    // blocks holding later parts of the set: blockIdx + 1 .. blockIdx + nlater
    int nlater = 0;
    if (starts && !whole)
      while (blockIdx.x + 1 + nlater < gridDim.x && sched.ub[blockIdx.x + 1 + nlater] < set_u1)
        ++nlater;
    if (threadIdx.x == 0) *late_flag = 0;
    __syncthreads();
    if (threadIdx.x < nlater && *abort_flag == 0) {
      // one thread per later block: wait (bounded) for its published partials
      const unsigned long long* fp = ws_flag + blockIdx.x + 1 + threadIdx.x;
      unsigned long long f;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(f) : "l"(fp) : "memory");
      if (f != kPPublished) {
        const unsigned long long t0 = gtime();
        for (uint32_t i = 1;; ++i) {
          asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(f) : "l"(fp) : "memory");
          if (f == kPPublished) break;
          if ((i & 15u) == 0u && gtime() - t0 > wait_ns) break;
        }
      }
      if (f != kPPublished) {
        report_status(dev_status, (int32_t)ANY4_ERR_TIMEOUT);
        *late_flag = 1;
      }
    }
    __syncthreads();
    const bool good = *abort_flag == 0 && *late_flag == 0;
    if (threadIdx.x < MT * kPRows && good) {
      const int m = threadIdx.x / kPRows, slot = threadIdx.x % kPRows;
      float v = 0.f;
      for (int w = 0; w < kPWarps; ++w) v += s_part[(size_t)(w * MT + m) * kPRows + slot];
      const int row = r * kPRows + slot;
      if (!starts) {
        // a later part of the set: hand the partial sums to the set's first block
        __stcg(ws_part + (size_t)blockIdx.x * (MT * kPRows) + threadIdx.x, v);
      } else {
        // add the later blocks' parts in block order (their flags were seen above)
        for (int b = 1; b <= nlater; ++b)
          v += __ldcg(ws_part + (size_t)(blockIdx.x + b) * (MT * kPRows) + threadIdx.x);
        if (row < N) {
          if (y32 != nullptr)
            y32[(int64_t)m * N + row] = v;
          else
            y[(int64_t)m * N + row] = f32_to_bf16_rn(v);
        }
      }
    }
    __syncthreads();  // partial sums read; table and s_part may be rewritten
    if (threadIdx.x == 0 && good) {
      if (!starts) {
        __threadfence();
        asm volatile("st.release.gpu.global.u64 [%0], %1;" :: "l"(ws_flag + blockIdx.x),
                     "l"(kPPublished) : "memory");
      }
    }
    if (threadIdx.x < nlater && good) {
      // the consumed flags go back to "not published" for the next launch
      asm volatile("st.relaxed.gpu.global.u64 [%0], %1;"
                   :: "l"(ws_flag + blockIdx.x + 1 + threadIdx.x), "l"(0ull) : "memory");
    }
  }
  // before leaving, no tensor load of this warp may still be writing its ring
  if (lane == 0) {
    for (; item < issued; ++item) {
      if (!mbar_wait(my_bars + 8u * (item % kPStages), (uint32_t)((item / kPStages) & 1),
                     kPWaitNs))
        break;
    }
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encoder() {
  static EncodeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeFn>(p);
    return static_cast<EncodeFn>(nullptr);
  }();
  return fn;
}

bool map2d(EncodeFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
           uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
           CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kPDynBytes = 227 * 1024;

template <int MT, int GS>
any4_status run_pair(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                     int64_t lut_row_stride, const uint16_t* scale, const uint16_t* offset,
                     uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K, int64_t G,
                     void* workspace, bool overlap, int32_t* dev_status, bool test_stall,
                     cudaStream_t stream, const DeviceInfo& dev) {
  EncodeFn enc = encoder();
  if (!enc) return ANY4_ERR_UNSUPPORTED;
  PMaps maps;
  if (!map2d(enc, &maps.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2,
             (uint64_t)N, (uint64_t)K / 2, kPChunk / 2, kPRows, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !map2d(enc, &maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, (uint64_t)K, (uint64_t)M,
             (uint64_t)K * 2, kPChunk, MT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ANY4_ERR_CUDA;
  if (lut_row_stride == 16) {
    if (!map2d(enc, &maps.lut, CU_TENSOR_MAP_DATA_TYPE_UINT16, lut, 16, (uint64_t)N, 32, 16,
               kPRows, CU_TENSOR_MAP_SWIZZLE_NONE))
      return ANY4_ERR_CUDA;
  } else {
    maps.lut = maps.codes;  // unused: one table for the matrix, read directly
  }
  auto kern = decode_pair_kernel<MT, GS>;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), kPDynBytes) != ANY4_OK)
    return ANY4_ERR_CUDA;
  const int KC = (int)((K + kPChunk - 1) / kPChunk);
  const int64_t sets = (N + kPRows - 1) / kPRows;
  const int64_t units = sets * KC;
  const int grid = (int)std::min<int64_t>({units, (int64_t)dev.sm_count, (int64_t)kPMaxGrid});
  PSched sched;
  for (int b = 0; b <= grid; ++b) sched.ub[b] = (int)(units * b / grid);
  float* ws_part = static_cast<float*>(workspace);
  auto* ws_flag = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(workspace) + (size_t)dev.sm_count * MT * kPRows * sizeof(float));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPDynBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint16_t* lut_shared = lut_row_stride == 0 ? lut : nullptr;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, maps, lut_shared, scale, offset, y, y32,
                                             (int)N, (int)K,
                                             KC, sched, ws_part, ws_flag, kPDynBytes, dev_status,
                                             test_stall ? 1 : 0);
  return err == cudaSuccess ? ANY4_OK : ANY4_ERR_CUDA;
}

}  // namespace

bool decode_pair_supported(int64_t M, int64_t N, int64_t K, int64_t G) {
  if (M < 1 || M > 2) return false;
  if (G != 32 && G != 64 && G != 128) return false;
  // whole 128-column chunks, so that a chunk holds 4 / (G / 32) whole groups
  // and its scales are one aligned 2-, 4- or 8-byte load per row
  if (K % kPChunk != 0) return false;
  // unit, row and column indices in 32 bits
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return false;
  if (((N + kPRows - 1) / kPRows) * (K / kPChunk) > (int64_t(1) << 30)) return false;
  return true;
}

size_t decode_pair_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G,
                                  const DeviceInfo& dev) {
  if (!decode_pair_supported(M, N, K, G)) return 0;
  const size_t part = (size_t)dev.sm_count * (size_t)M * kPRows * sizeof(float);
  return ((part + (size_t)dev.sm_count * 8 + 255) / 256) * 256;
}

any4_status launch_decode_pair(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                               int64_t lut_row_stride, const uint16_t* scale,
                               const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                               int64_t N, int64_t K, int64_t G, void* workspace, bool overlap,
                               int32_t* dev_status, bool test_stall, cudaStream_t stream,
                               const DeviceInfo& dev) {
  if (!decode_pair_supported(M, N, K, G)) return ANY4_ERR_UNSUPPORTED;
#define ANY4_PAIR_CASE(MT_, GS_)                                                               \
  if (M == MT_ && G == 32 * GS_)                                                               \
    return run_pair<MT_, GS_>(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, \
                              G, workspace, overlap, dev_status, test_stall, stream, dev);
  ANY4_PAIR_CASE(1, 4)
  ANY4_PAIR_CASE(1, 2)
  ANY4_PAIR_CASE(1, 1)
  ANY4_PAIR_CASE(2, 4)
  ANY4_PAIR_CASE(2, 2)
  ANY4_PAIR_CASE(2, 1)
#undef ANY4_PAIR_CASE
  return ANY4_ERR_UNSUPPORTED;
}

}  // namespace any4
