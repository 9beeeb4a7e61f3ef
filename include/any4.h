/*
 * any4.h -- C ABI of libany4, the B200 (sm_100a) implementation of the any4
 * weight-only 4-bit matmul.
 *
 * Method: "any4: Learned 4-bit Numeric Representation for LLMs" (Elhoushi &
 * Johnson, arXiv 2507.04610).  Each weight row n owns a learned 16-entry
 * lookup table LUT[n][0..15]; each weight is a 4-bit code c indexing it; each
 * group of G consecutive columns of a row shares one scale and one offset
 * (paper §2.4.1, §2.5.1), and a weight is dequantised as
 *       W[n][k] = LUT[n][c] * scale[n][k/G] + offset[n][k/G]      (§2.5.2)
 * The matmul is y = x W^T with x of size M x K and W of size N x K (§4.2,
 * §4.1 Eq. 8).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - bf16 tensors (x, y, W, LUT, scale, offset) are passed as uint16_t
 *    pointers to their raw bfloat16 bit patterns.
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or any
 *    device-accessible allocation), owned by the caller, row-major and
 *    contiguous.  The library never allocates, frees or keeps them.
 *  - Every pointer must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream).  The return value reports only host-side argument
 *    validation and launch errors; nothing is launched when a call returns
 *    an error.  Errors detected on the device (a code above 15 in any4_pack, a
 *    pipeline wait that ran out in any4_matmul) are OR-ed into `*dev_status`
 *    (int32 in device memory, may be NULL), which the caller zeroes before the
 *    call and reads after synchronising the stream; a non-zero value is one
 *    of the negative any4_status codes below (their bits OR-ed together).
 *  - Shape rules: N >= 1, M >= 1, K >= 32, K % 32 == 0, G % 32 == 0,
 *    K % G == 0.  So every 32-code (16-byte) chunk of a packed row lies in a
 *    single group.
 *  - Outputs must not overlap inputs.
 *  - Results are deterministic: the same inputs, shape and GPU give the same
 *    bits on every run (no atomics in any reduction).
 */
#ifndef ANY4_H
#define ANY4_H

#include <stddef.h>
#include <stdint.h>

/* Every entry point is exported from the shared library (which is built with
 * hidden default visibility). */
#if defined(__GNUC__)
#define ANY4_API __attribute__((visibility("default")))
#else
#define ANY4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum any4_status {
  ANY4_OK = 0,
  ANY4_ERR_NULL = -1,        /* a required pointer is NULL                        */
  ANY4_ERR_SHAPE = -2,       /* a size breaks the shape rules above               */
  ANY4_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned                  */
  ANY4_ERR_RANGE = -4,       /* device: a code above 15 was given to any4_pack    */
  ANY4_ERR_CUDA = -5,        /* a CUDA runtime call or launch failed              */
  ANY4_ERR_TIMEOUT = -6,     /* device: a bounded pipeline wait gave up           */
  ANY4_ERR_UNSUPPORTED = -7, /* no kernel for this request (e.g. not an sm_100 GPU)*/
  ANY4_ERR_WORKSPACE = -8    /* workspace missing or smaller than required        */
} any4_status;

/* Same type as cudaStream_t. */
typedef struct CUstream_st* any4_stream_t;

/* Which kernel family any4_matmul_ex runs. */
typedef enum any4_path {
  ANY4_PATH_AUTO = 0,    /* choose by M (what any4_matmul does)                  */
  ANY4_PATH_DECODE = 1,  /* CUDA-core LUT-in-registers GEMV / skinny GEMM, M<=16 */
  ANY4_PATH_PREFILL = 2  /* tcgen05 tensor-core GEMM with dequantised tiles      */
} any4_path;

/*
 * any4_pack -- nibble-pack 4-bit codes, two per byte (paper §4.2; §2.4.1).
 *   idx     [N][K] uint8, each value 0..15           (input)
 *   packed  [N][K/2] uint8: packed[n][j] = idx[n][2j] | idx[n][2j+1] << 4
 *           (the even column in the LOW nibble)       (output)
 * A value above 15 is packed masked to 4 bits and sets ANY4_ERR_RANGE in
 * *dev_status.  Shape rule: K % 32 == 0 (G plays no part).
 */
ANY4_API any4_status any4_pack(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                      int32_t* dev_status, any4_stream_t stream);

/*
 * any4_quantize -- learn the any4 representation of a bf16 weight matrix: per
 * group scaling (paper §2.5.1 Eq. 1-2), then per row a weighted k-means on the
 * scaled weights (§4.1: E-step Eq. 18, M-step Eq. 23; Appendix A.1 Alg. 1).
 * Its outputs are the inputs of any4_dequant and any4_matmul (one table per
 * row, lut_row_stride 16).
 *   w          [N][K] bf16 weight                                    (input)
 *   ex_abs     [K] fp32, E|x_j|: the mean absolute calibration activation of
 *              input column j; finite and >= 0                       (input)
 *   max_iter   M-steps at most, 0 <= max_iter <= ANY4_QUANTIZE_MAX_ITER
 *   packed     [N][K/2] uint8 codes (layout of any4_pack)            (output)
 *   lut        [N][16] bf16 table                                     (output)
 *   scale      [N][K/G] bf16 alpha                                    (output)
 *   offset     [N][K/G] bf16 beta                                     (output)
 *   iters      [N] int32, M-steps run per row; may be NULL (4-byte aligned)
 * Steps, each floating-point operation correctly rounded, in this order:
 *   alpha = bf16(fp32(max - min) / 15) and beta = min over each group of G
 *   columns (-0 read as +0); w_S = (w - beta) / alpha in fp64 (0 where alpha
 *   is 0); the starting table holds the elements at positions
 *   floor(q (K - 1) / 15), q = 0..15, of the row's sorted w_S; E-step: nearest
 *   entry by |w_S - c_q|, ties to the lowest q; M-step: c_q = sum(u_j w_S_j) /
 *   sum(u_j) over the columns of cluster q in ascending order, fp64, with
 *   u_j = alpha_{g(j)} * E|x_j|; a cluster whose u_j sum to 0 keeps its entry;
 *   stop after max_iter M-steps or when an E-step changes no code;
 *   LUT_q = bf16(fp32(c_q)); the codes are a final E-step against the stored
 *   LUT.  The results are bit-identical on every run and GPU.
 * Shape rules as above, plus K <= ANY4_QUANTIZE_MAX_K (the row and its sort
 * buffer live in one block's shared memory).  NaN or infinite weights or
 * activation statistics give unspecified results.  One thread block per row.
 */
#define ANY4_QUANTIZE_MAX_K 16384
#define ANY4_QUANTIZE_MAX_ITER 100000
ANY4_API any4_status any4_quantize(const uint16_t* w, const float* ex_abs, int64_t N, int64_t K,
                                   int64_t G, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                                   uint16_t* scale, uint16_t* offset, int32_t* iters,
                                   any4_stream_t stream);

/*
 * n-bit variants: any3 and any2 (and any4 again as bits = 4).  The paper states
 * the learned table for any bit width n (§4.1 Eq. 9: 2^n values per row) and
 * evaluates 3 and 2 bits (§5); it gives no storage layout below 4 bits.
 * Layout here: the codes of a row form one little-endian bit stream, code k in
 * bits [n k, n k + n) (bit i of the stream is bit i % 8 of byte i / 8), so a
 * packed row holds n K / 8 bytes; for n = 4 this is any4_pack's layout.  A
 * row's table holds 2^n bf16 entries.  Shape rules and conventions as above;
 * bits is 2, 3 or 4 (4 runs the any4 call of the same name).
 *
 * any4_pack_bits     idx [N][K] uint8 (codes 0 .. 2^n - 1) -> packed
 *                    [N][n K / 8]; a larger code is packed masked to n bits
 *                    and sets ANY4_ERR_RANGE in *dev_status.
 * any4_dequant_bits  W[n][k] = bf16_rne(fmaf(LUT[n][c], scale[n][k/G],
 *                    offset[n][k/G])) for the n-bit code c; lut_row_stride is
 *                    2^n (a table per row) or 0 (one table).  Bit-exact.
 * any4_quantize_bits any4_quantize with 2^n table entries: alpha =
 *                    bf16(fp32(max - min) / (2^n - 1)), the quantile start at
 *                    positions floor(q (K - 1) / (2^n - 1)), lut [N][2^n],
 *                    packed [N][n K / 8]; otherwise the steps of
 *                    any4_quantize.  The results are bit-identical on every
 *                    run and GPU.
 */
ANY4_API any4_status any4_pack_bits(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                                    int32_t bits, int32_t* dev_status, any4_stream_t stream);
ANY4_API any4_status any4_dequant_bits(const uint8_t* packed, const uint16_t* lut,
                                       int64_t lut_row_stride, const uint16_t* scale,
                                       const uint16_t* offset, uint16_t* W, int64_t N, int64_t K,
                                       int64_t G, int32_t bits, any4_stream_t stream);
ANY4_API any4_status any4_quantize_bits(const uint16_t* w, const float* ex_abs, int64_t N,
                                        int64_t K, int64_t G, int32_t bits, int32_t max_iter,
                                        uint8_t* packed, uint16_t* lut, uint16_t* scale,
                                        uint16_t* offset, int32_t* iters, any4_stream_t stream);

/*
 * any4_matmul_bits -- y = x * dequant(W)^T for n-bit codes (n = 2, 3 or 4;
 * the any3 / any2 formats of paper §5, a table of 2^n values per row, §4.1
 * Eq. 9), codes in the layout of any4_pack_bits, lut_row_stride 2^n or 0.
 * n = 4 runs any4_matmul_ex (auto path).  For n = 2, 3:
 *   M = 1, G of 32, 64 or 128, K/G a multiple of 8 and n K a multiple of 128:
 *     the weight-streaming decode kernel reads the n-bit codes directly
 *     (fused lookup, scale and offset; no workspace);
 *   otherwise two passes as any4_matmul's large-M path: the n-bit dequant
 *     into the workspace (bf16 W, bit-exact with any4_dequant_bits), then the
 *     tensor-core GEMM.
 * workspace: at least any4_matmul_bits_workspace_size bytes (0: none).
 * flags: ANY4_FLAG_OVERLAP_PRIOR, _FP32_OUT, _TEST_STALL as for any4_matmul_ex.
 * Tolerance and determinism as any4_matmul.
 */
ANY4_API any4_status any4_matmul_bits(const uint16_t* x, const uint8_t* packed,
                                      const uint16_t* lut, int64_t lut_row_stride,
                                      const uint16_t* scale, const uint16_t* offset, uint16_t* y,
                                      int64_t M, int64_t N, int64_t K, int64_t G, int32_t bits,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, uint32_t flags, any4_stream_t stream);
ANY4_API size_t any4_matmul_bits_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G,
                                                int32_t bits);

/*
 * any4_dequant -- materialise the bf16 weight (paper §2.5.2 dequant with the
 * per-row table of §2.4.1):
 *   W[n][k] = bf16_rne( fmaf( LUT[n][c], scale[n][k/G], offset[n][k/G] ) )
 * computed in fp32 with one rounding for the fused multiply-add, then rounded
 * to nearest-even bf16 (no flush to zero).  Bit-exact.
 *   packed          [N][K/2] uint8 (layout of any4_pack)
 *   lut             table of row n at lut + n * lut_row_stride, 16 bf16 each;
 *                   lut_row_stride = 16 for any4 (a table per row) or 0 for
 *                   one table shared by the whole matrix (the nf4/af4 mode
 *                   the paper's §2.4.1 describes)
 *   scale, offset   [N][K/G] bf16
 *   W               [N][K] bf16 (output)
 */
ANY4_API any4_status any4_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                         const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                         int64_t N, int64_t K, int64_t G, any4_stream_t stream);

/*
 * any4_group_sums -- per-group sums of the activations:
 *   xsum[m][g] = sum over the G columns k = g*G .. g*G+G-1 of x[m][k]
 * The factor of the group offset when the product of paper §4.1 Eq. 8 is
 * expanded with the group-affine weights of §2.5.2 (alpha * LUT[c] + beta):
 *   sum_k x * (alpha * LUT[c] + beta) = alpha * sum_k x * LUT[c] + beta * xsum.
 * For callers that apply the offsets themselves (a matmul on the bare table
 * values, an offset correction, a calibration statistic); any4_matmul does not
 * need it, it applies alpha and beta to every weight.
 *   x      [M][K] bf16 (device, caller-owned, 16-byte aligned)
 *   xsum   [M][K/G] fp32 (device, caller-owned output, 16-byte aligned)
 *   M >= 1; K and G multiples of 32 with K % G == 0.
 * fp32 sums in a fixed order (each 8-column chunk left to right, then the
 * group's chunks left to right), so deterministic; every result is within
 * gamma_{G-1} * sum |x| of the exact sum (gamma_n = n u / (1 - n u),
 * u = 2^-24).  Returns ANY4_ERR_NULL, _SHAPE or _ALIGN without launching
 * when a precondition fails; asynchronous on `stream` otherwise.
 */
ANY4_API any4_status any4_group_sums(const uint16_t* x, float* xsum, int64_t M, int64_t K,
                                     int64_t G, any4_stream_t stream);

/*
 * any4_read_probe -- a read-only stream over a device buffer, the measurement
 * of the read bandwidth that bounds the decode matmuls (they read the packed
 * codes, tables, scales and offsets once and write only y, so their roofline
 * is HBM delivering reads alone, not a copy's mix of reads and writes):
 *   *out = XOR of the 32-bit words buf[0 .. bytes / 4)
 *   buf    device, caller-owned, 16-byte aligned (may be NULL when bytes == 0)
 *   bytes  >= 0, a multiple of 16
 *   out    one uint32 in device memory, caller-owned, 4-byte aligned; zeroed
 *          on `stream` before the kernel runs (0 for an empty buffer)
 * Every byte is read once, with 16-byte loads that skip L1, by a grid of
 * 8 blocks of 256 threads per SM.  The result does not depend on the order of
 * the reads.  Returns ANY4_ERR_NULL, _SHAPE or _ALIGN without launching when a
 * precondition fails; asynchronous on `stream` otherwise.
 */
ANY4_API any4_status any4_read_probe(const void* buf, int64_t bytes, uint32_t* out,
                                     any4_stream_t stream);

/*
 * any4_matmul -- y = x * dequant(W)^T (paper §4.1 Eq. 8, orientation §4.2),
 * dequantisation fused (W is never written to memory on the decode path).
 *   x               [M][K] bf16
 *   packed, lut, lut_row_stride, scale, offset   as for any4_dequant
 *   y               [M][N] bf16 (output): fp32 accumulation, rounded to
 *                   nearest-even bf16
 *   workspace       device scratch of workspace_bytes bytes, at least
 *                   any4_matmul_workspace_size(M, N, K, G); may be NULL when
 *                   that size is 0.  Its contents need not be initialised and
 *                   are undefined afterwards; two calls in flight at the same
 *                   time must not share one.  At M <= 2 the size is that of
 *                   the pair-table decode kernel (tens of KiB); a NULL
 *                   or smaller workspace there runs the slower decode kernels
 *                   that need none.  After a call that reported
 *                   ANY4_ERR_TIMEOUT, zero the workspace (or take another)
 *                   before its next use: the aborted call may have left a
 *                   block's "partial sums published" marker in it.
 *   dev_status      see the conventions above (ANY4_ERR_TIMEOUT)
 * Accuracy: |y - y_ref| <= 1e-2 * rms(y_ref) + ulp_bf16(y_ref) per element,
 * with y_ref the exact dequant-then-matmul.  Inside the kernels each weight is
 * formed as LUT * scale + offset rounded once to bf16 (a bf16x2 fused
 * multiply-add), which equals any4_dequant's W except when the fp32 fmaf is
 * inexact and lands exactly on a bf16 rounding tie.
 * Kernels: M <= 2 the pair-table decode (given its workspace; else M = 1
 * weight-streaming decode), 2 <= M <= 16 skinny, larger M the tensor-core
 * prefill (any4_matmul_choose_path).
 */
ANY4_API any4_status any4_matmul(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                        int64_t lut_row_stride, const uint16_t* scale,
                        const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                        int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, any4_stream_t stream);

/* Flags of any4_matmul_ex. */
typedef enum any4_flags {
  ANY4_FLAG_NONE = 0,
  /* The caller guarantees that no work still running on `stream` when the
   * call is issued writes packed, lut, scale or offset (the usual case for
   * inference weights).  The kernel is then launched as a programmatic
   * dependent of that work: it may start, and begin streaming the weights,
   * while the preceding kernel on the stream finishes; x is read and y is
   * written only after the preceding kernel has completed.  Decode path only;
   * ignored elsewhere. */
  ANY4_FLAG_OVERLAP_PRIOR = 1,
  /* y is an fp32 [M][N] array (still 16-byte aligned) and receives the fp32
   * sums before their rounding to bf16: the kernels' accumulation can then be
   * compared with the exact result on its own.  Every path. */
  ANY4_FLAG_FP32_OUT = 2,
  /* Test hook for the failure handling, not for production calls: block 0 of
   * the kernel stops its weight (or x) stream after the first stage and every
   * bounded wait gives up after 1 ms instead of about 2 s.  The call then ends
   * with ANY4_ERR_TIMEOUT in *dev_status, its y undefined, no memory outside
   * y and the workspace written, the kernel's own copies drained and its
   * tensor memory released, so the device and stream stay usable.  Kernels
   * with bounded waits only: the pair-table and weight-streaming decode
   * kernels and the prefill kernel (others ignore it). */
  ANY4_FLAG_TEST_STALL = 4,
  /* Decode path, M = 1: run the pair-table kernel (the M = 2 default) instead
   * of the weight-streaming kernel that M = 1 takes by default.  Needs the
   * workspace any4_matmul_workspace_size returns for the shape; without it,
   * or where the pair-table kernel does not take the shape, the flag is
   * ignored. */
  ANY4_FLAG_PAIR_TABLE = 8,
  /* packed holds the codes in the decode layout that any4_repack writes, not
   * any4_pack's.  Taken only where the M = 1 weight-streaming kernel with
   * folded tables runs: M = 1, G = 128, K a multiple of 1024, path auto or
   * decode, without ANY4_FLAG_PAIR_TABLE (any4_matmul_ex and
   * any4_matmul_grouped); any other call with this flag returns
   * ANY4_ERR_UNSUPPORTED.  Results are the same bits as the call on
   * any4_pack's layout. */
  ANY4_FLAG_DECODE_LAYOUT = 16
} any4_flags;

/* any4_matmul with an explicit kernel family (ANY4_PATH_DECODE needs M <= 16)
 * and flags (a bitwise OR of any4_flags).  Same arguments and results
 * otherwise; used to test each path at any M and to overlap launches. */
ANY4_API any4_status any4_matmul_ex(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                           int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, any4_path path, uint32_t flags,
                           any4_stream_t stream);

/*
 * any4_matmul_static_scratch -- any4_matmul on the prefill kernel (the
 * tensor-core path, any M) with its scratch taken from a fixed array inside
 * the library instead of a caller-supplied workspace.  The paper has no
 * counterpart: this is an interface variant for callers that cannot allocate
 * device memory at the call site (a step that must not call cudaMalloc or
 * cudaFree, since cudaFree synchronises the whole device; a C caller with no
 * device allocator of its own).  It allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *   arguments       as for any4_matmul, minus the workspace
 *   scratch         a file-scope device array of ANY4_STATIC_SCRATCH_BYTES
 *                   bytes, one per device: 37 MiB + 1 KiB, i.e. one 256 KiB
 *                   fp32 partial tile per block of a 148-SM grid plus the
 *                   per-block flags, which each call clears (an async memset
 *                   on `stream`) before its launch.  The array is reserved on
 *                   every device where the library's module is loaded, in
 *                   every process that loads libany4, whether or not this
 *                   entry point is ever called.  If the device needs more
 *                   (any4_matmul_workspace_size_ex(..., ANY4_PATH_PREFILL)
 *                   above ANY4_STATIC_SCRATCH_BYTES, e.g. a GPU with more
 *                   than 148 SMs) the call returns ANY4_ERR_WORKSPACE and
 *                   launches nothing.
 *   set-up          the first call on a device looks up the array's device
 *                   address (cudaGetSymbolAddress, with that device current)
 *                   and caches it per device, keyed by the identity of the
 *                   current context: after a device reset (or a released and
 *                   re-created primary context) the next call looks it up
 *                   again.  Make the first call on a device, and the first
 *                   after a reset, before any stream capture.  A failed
 *                   look-up returns ANY4_ERR_CUDA.
 *   concurrency     every call on a device uses the same array: calls whose
 *                   kernels overlap on the GPU (different streams, or several
 *                   host threads) race on it and give undefined results.
 *                   Calls issued in order on one stream are safe.
 * Results are those of the one-pass prefill kernel (what
 * any4_matmul_ex(..., ANY4_PATH_PREFILL, ...) runs below M = 1024 or with a
 * workspace of only the one-pass size); at larger M they agree with the
 * two-pass route within the matmul tolerance above, not bit for bit.
 */
#define ANY4_STATIC_SCRATCH_BYTES ((size_t)148 * 262144 + 1024)
ANY4_API any4_status any4_matmul_static_scratch(const uint16_t* x, const uint8_t* packed,
                                                const uint16_t* lut, int64_t lut_row_stride,
                                                const uint16_t* scale, const uint16_t* offset,
                                                uint16_t* y, int64_t M, int64_t N, int64_t K,
                                                int64_t G, int32_t* dev_status,
                                                any4_stream_t stream);

/* Bytes of workspace any4_matmul needs for this shape (0 if none) to run its
 * fastest kernel.  Returns 0 as well for shapes that break the shape rules
 * (the call then fails).  On the prefill path at M >= 1024 the size includes
 * room for the dequantised weights (N * K * 2 bytes): the call then runs in two
 * passes (any4_dequant into the workspace, then a tensor-core GEMM that streams
 * those bf16 weights).  A smaller workspace, down to the one-pass size (the
 * size this function returns for M < 1024), runs the one-pass kernel, which
 * dequantises the weights tile by tile. */
ANY4_API size_t any4_matmul_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G);

/*
 * any4_repack -- the packed codes rearranged for the M = 1 decode kernel
 * (ANY4_FLAG_DECODE_LAYOUT).  The idea is the paper's (§4.2: its kernel reads
 * weights pre-permuted into the order its threads consume them); the order
 * here is this library's own.  Each row's codes go in 1024-column slices of
 * 128 32-bit words (word w of a slice: codes of columns 8w .. 8w + 7, the
 * even column in the low nibble, as any4_pack); within a slice, the 16-byte
 * chunk l (l = 0..31, bytes 16 l .. 16 l + 15) holds, as its words t = 0..3,
 * the input words 16 (4 h + (t XOR h)) + e with h = l / 16, e = l mod 16:
 * the four words lane l of the kernel reads, one per step, so a lane loads
 * them with one 16-byte load.  A permutation of whole 32-bit words within
 * each slice; the tables, scales and offsets are unchanged.
 *   packed    [N][K/2] uint8, any4_pack's layout                    (input)
 *   repacked  [N][K/2] uint8, the decode layout; must not overlap packed
 *   K         a multiple of 1024; N >= 1
 * Both pointers 16-byte aligned device memory.  Errors: ANY4_ERR_NULL,
 * ANY4_ERR_SHAPE, ANY4_ERR_ALIGN, ANY4_ERR_CUDA (launch).
 */
ANY4_API any4_status any4_repack(const uint8_t* packed, uint8_t* repacked, int64_t N, int64_t K,
                                 any4_stream_t stream);

/*
 * any4_matmul_grouped -- several weight matrices applied to the same x:
 *   y_i = x * dequant(W_i)^T   for i = 0 .. count-1
 * (the q, k and v projections of a transformer layer, or gate and up: the
 * matmuls of paper §4.1 Eq. 8 that share their input).  Each result is
 * exactly what any4_matmul_ex gives for that matrix alone (same bits).
 * At M = 1, on the shapes the weight-streaming decode kernel takes (G of 32,
 * 64 or 128 with K/G a multiple of 8), all matrices run in ONE launch whose
 * blocks stream the matrices' rows one after the other, so small matrices no
 * longer pay a launch and a pipeline ramp each; otherwise the matrices run
 * as count calls of any4_matmul_ex, one after the other on `stream`, sharing
 * the workspace.
 *   x          [M][K] bf16
 *   w          count descriptors (host memory, read during the call only):
 *              packed [N_i][K/2], lut (lut_row_stride 16: [N_i][16]; 0: one
 *              [16] table), scale and offset [N_i][K/G], y [M][N_i] bf16 (or
 *              fp32 with ANY4_FLAG_FP32_OUT), N_i >= 1; device pointers,
 *              16-byte aligned; no y may overlap another y or any input
 *   count      1 .. ANY4_GROUP_MAX
 *   workspace  at least the largest any4_matmul_workspace_size_ex(M, N_i, K,
 *              G, path) of the group where the per-matrix calls need one
 *   flags      as any4_matmul_ex (ANY4_FLAG_OVERLAP_PRIOR, _FP32_OUT,
 *              _TEST_STALL; ANY4_FLAG_PAIR_TABLE makes M = 1 take the
 *              per-matrix calls; ANY4_FLAG_DECODE_LAYOUT: every packed is
 *              in any4_repack's layout, M = 1 and G = 128 only)
 * Returns the first error of the validation (nothing launched), or of the
 * per-matrix calls (the earlier ones launched).
 */
#define ANY4_GROUP_MAX 4
typedef struct any4_weight {
  const uint8_t* packed;
  const uint16_t* lut;
  int64_t lut_row_stride;
  const uint16_t* scale;
  const uint16_t* offset;
  uint16_t* y;
  int64_t N;
} any4_weight;

ANY4_API any4_status any4_matmul_grouped(const uint16_t* x, const any4_weight* w, int32_t count,
                                         int64_t M, int64_t K, int64_t G, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status,
                                         any4_path path, uint32_t flags, any4_stream_t stream);

/* Same for an explicit path. */
ANY4_API size_t any4_matmul_workspace_size_ex(int64_t M, int64_t N, int64_t K, int64_t G,
                                     any4_path path);

/* The path any4_matmul would take for this M (ANY4_PATH_DECODE or _PREFILL). */
ANY4_API any4_path any4_matmul_choose_path(int64_t M, int64_t N, int64_t K, int64_t G);

/* Static description of an error code; never NULL. */
ANY4_API const char* any4_status_string(int32_t status);

/* Bits stored per weight for this format: 4 + 32/G + 256/K (16-bit LUT
 * entries, 16-bit scale and offset), the accounting of paper §2.4.1. */
ANY4_API double any4_bits_per_weight(int64_t K, int64_t G);

/* Library version, major * 10000 + minor * 100 + patch. */
ANY4_API int32_t any4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ANY4_H */
