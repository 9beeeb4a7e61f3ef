/*
 * any4 oracle: a plain, slow, obviously correct CPU statement of what the any4
 * W4A16 path computes.  TEST INFRASTRUCTURE ONLY: nothing in the product path
 * (the CUDA library or its Python binding) may include, link or call this file.
 * It is used by tests/, by __graft_entry__.smoke() and by bench.py's CPU
 * baseline leg, and by nothing else.  It shares no code with the CUDA path.
 *
 * Source of every definition: "any4: Learned 4-bit Numeric Representation for
 * LLMs" (Elhoushi & Johnson, arXiv 2507.04610):
 *   - §2.4.1: each row owns a 16-entry table (LUT) of 16-bit values; codes are
 *     4-bit indices into it; one 16-bit scale and one 16-bit zero point per
 *     group of g contiguous values of a row; 4.3125 bits/weight at g=128,
 *     K=4096.  The same section allows ONE table for a whole matrix (nf4/af4).
 *   - §2.5.1: group-wise scaling along the reduction dimension; group k holds
 *     columns k*g <= j < (k+1)*g (the printed range has a typo; this is the
 *     only reading that gives groups of g columns).
 *   - §2.5.2: dequant(w_Q) = alpha * w_Q + beta.  For any4, w_Q = LUT[code].
 *   - §4.1 Eq. 8: y_hat_i = sum_j dequant(w_Q[i,j]) * x_j.
 *   - §4.2: y = x * w^T with x of size M x K and w of size N x K; two any4
 *     codes share one byte.
 *
 * Precision readings (the pages give none for these steps):
 *   - LUT, scale, offset, x and y are bfloat16; they cross this interface as
 *     their raw 16-bit patterns (uint16_t).
 *   - Nibble order: the code of even column k sits in the LOW nibble of byte
 *     k/2, the code of odd column k in the HIGH nibble.
 *   - Dequant: W = bf16_rne( fmaf( (float)LUT, (float)scale, (float)offset ) ),
 *     i.e. one fp32 fused multiply-add (single rounding, C99 fmaf) followed by
 *     round-to-nearest-even to bfloat16.  No flush-to-zero.
 *   - Matmul: y[m][n] = sum over k ascending of (double)x[m][k] * (double)W[n][k]
 *     with W the bf16 dequantised weight, one fp64 accumulator per output.
 *     Products of two bf16 values are exact in fp64.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -fPIC -shared (no -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* bfloat16 <-> binary32.  bfloat16 is binary32 with the low 16 fraction bits */
/* dropped: 1 sign bit, 8 exponent bits, 7 fraction bits.                     */
/* ------------------------------------------------------------------------- */

/* Widening is exact: the bf16 pattern becomes the high half of the binary32. */
float oracle_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round a binary32 to the nearest bfloat16, ties to the even pattern
 * (IEEE 754 roundTiesToEven applied at the 7-bit fraction boundary).
 * Written from the definition: compare the 16 discarded bits with the
 * halfway point 0x8000.  Overflow past the largest finite value carries
 * into the exponent and yields infinity, as IEEE 754 requires.  A NaN
 * stays a NaN (sign kept, quiet bit set).  Subnormals are rounded like
 * any other value (no flush to zero). */
uint16_t oracle_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u) {
    return (uint16_t)((u >> 16) | 0x0040u); /* NaN: keep it a (quiet) NaN */
  }
  uint32_t kept = u >> 16;          /* sign, exponent, 7 fraction bits */
  uint32_t dropped = u & 0xffffu;   /* the 16 bits rounded away        */
  if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) {
    kept += 1u;                     /* may carry into the exponent     */
  }
  return (uint16_t)kept;
}

void oracle_bf16_rne_array(const float* f, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i) h[i] = oracle_bf16_rne(f[i]);
}

void oracle_bf16_to_f32_array(const uint16_t* h, float* f, int64_t n) {
  for (int64_t i = 0; i < n; ++i) f[i] = oracle_bf16_to_f32(h[i]);
}

/* ------------------------------------------------------------------------- */
/* Storage layout (§2.4.1, §4.2): two 4-bit codes per byte.                   */
/* ------------------------------------------------------------------------- */

/* packed[n][j] = idx[n][2j] | idx[n][2j+1] << 4, row-major, K even.
 * Returns the number of codes outside 0..15 (those are packed masked to
 * 4 bits; a non-zero return means the input was not a valid code array). */
int64_t oracle_pack(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K) {
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < K / 2; ++j) {
      uint8_t lo = idx[n * K + 2 * j];
      uint8_t hi = idx[n * K + 2 * j + 1];
      if (lo > 15) ++bad;
      if (hi > 15) ++bad;
      packed[n * (K / 2) + j] = (uint8_t)((lo & 15u) | ((hi & 15u) << 4));
    }
  }
  return bad;
}

/* The code of column k of row n. */
static unsigned code_at(const uint8_t* packed, int64_t K, int64_t n, int64_t k) {
  uint8_t byte = packed[n * (K / 2) + k / 2];
  return (k % 2 == 0) ? (byte & 15u) : (byte >> 4);
}

void oracle_unpack(const uint8_t* packed, uint8_t* idx, int64_t N, int64_t K) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      idx[n * K + k] = (uint8_t)code_at(packed, K, n, k);
}

/* The packed codes in the order the library's M = 1 decode kernel reads them
 * (§4.2: the paper's kernel reads weights pre-permuted into the order its
 * threads consume them).  In each row's 1024-column slice, thread l (0..31)
 * of a warp covers at step t (0..3) the 8 columns 128 q + 8 (l mod 16) .. + 7
 * of the slice, q = 4 h + (t XOR h) with h = l div 16; the layout stores the
 * 4 bytes holding those 8 codes, for l in order and, within l, t in order.
 * Returns 0, or -1 when K is not a positive multiple of 1024. */
int oracle_repack_decode_layout(const uint8_t* packed, uint8_t* out, int64_t N, int64_t K) {
  if (K <= 0 || K % 1024 != 0) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* src = packed + n * (K / 2);
    uint8_t* dst = out + n * (K / 2);
    for (int64_t s = 0; s < K / 1024; ++s)
      for (int l = 0; l < 32; ++l) {
        int h = l / 16, e = l % 16;
        for (int t = 0; t < 4; ++t) {
          int64_t col = 1024 * s + 128 * (4 * h + (t ^ h)) + 8 * e;
          int64_t at = 512 * s + 16 * l + 4 * t;
          for (int b = 0; b < 4; ++b) dst[at + b] = src[col / 2 + b];
        }
      }
  }
  return 0;
}

/* Bits stored per weight: the 4-bit code, plus a 16-bit scale and a 16-bit
 * zero point per group of G, plus a 16-entry table of lut_bits-wide values
 * per row of K weights (§2.4.1 works this out as 4 + 0.25 + 0.0625 = 4.3125
 * for G = 128, K = 4096 and 16-bit entries). */
double oracle_bits_per_weight(int64_t K, int64_t G, int64_t lut_bits, int64_t group_param_bits) {
  return 4.0 + (2.0 * (double)group_param_bits) / (double)G +
         (16.0 * (double)lut_bits) / (double)K;
}

/* ------------------------------------------------------------------------- */
/* Dequant (§2.5.2 with w_Q = LUT[code]).                                     */
/* ------------------------------------------------------------------------- */

/* One weight: W = bf16_rne(fmaf(LUT[c], scale, offset)). */
uint16_t oracle_dequant_one(uint16_t lut_c, uint16_t scale, uint16_t offset) {
  float w = fmaf(oracle_bf16_to_f32(lut_c), oracle_bf16_to_f32(scale),
                 oracle_bf16_to_f32(offset));
  return oracle_bf16_rne(w);
}

/* W[n][k] for the whole matrix.
 *   lut:          row n's table starts at lut + n * lut_row_stride.
 *                 lut_row_stride = 16 is any4 (one table per row);
 *                 lut_row_stride = 0 is one table for the whole matrix
 *                 (the nf4/af4 mode of §2.4.1).
 *   scale/offset: [N][K/G], the parameters of group k/G of row n. */
void oracle_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                    const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                    int64_t N, int64_t K, int64_t G) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      unsigned c = code_at(packed, K, n, k);
      int64_t g = k / G;
      W[n * K + k] = oracle_dequant_one(lut[n * lut_row_stride + c],
                                        scale[n * (K / G) + g],
                                        offset[n * (K / G) + g]);
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Matmul (§4.1 Eq. 8, §4.2 orientation y = x * W^T).                         */
/* ------------------------------------------------------------------------- */

/* y[m][n] = sum_{k=0..K-1} x[m][k] * W[n][k] in fp64, k ascending.
 * x: [M][K] bf16, W: [N][K] bf16 (already dequantised), y: [M][N] fp64. */
void oracle_matmul(const uint16_t* x, const uint16_t* W, double* y,
                   int64_t M, int64_t N, int64_t K) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        acc += (double)oracle_bf16_to_f32(x[m * K + k]) *
               (double)oracle_bf16_to_f32(W[n * K + k]);
      }
      y[m * N + n] = acc;
    }
  }
}

/* The same outputs for a chosen subset of weight rows, dequantising each
 * chosen row on the fly (so the full W is never materialised).  Used to
 * check sampled outputs of full-size problems.
 *   rows:  the n indices, count of them;  y: [M][count] fp64;
 *   wrow:  caller scratch of count * K uint16 (receives the dequantised rows). */
void oracle_matmul_rows(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                        int64_t lut_row_stride, const uint16_t* scale,
                        const uint16_t* offset, const int64_t* rows, int64_t count,
                        double* y, uint16_t* wrow, int64_t M, int64_t N, int64_t K,
                        int64_t G) {
  (void)N;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < count; ++r) {
    int64_t n = rows[r];
    uint16_t* w = wrow + r * K;
    for (int64_t k = 0; k < K; ++k) {
      unsigned c = code_at(packed, K, n, k);
      int64_t g = k / G;
      w[k] = oracle_dequant_one(lut[n * lut_row_stride + c], scale[n * (K / G) + g],
                                offset[n * (K / G) + g]);
    }
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        acc += (double)oracle_bf16_to_f32(x[m * K + k]) * (double)oracle_bf16_to_f32(w[k]);
      }
      y[m * count + r] = acc;
    }
  }
}

/* Number of OpenMP threads a parallel region here would use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int t) { omp_set_num_threads(t); }
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_num_threads(int t) { (void)t; }
#endif

/* ------------------------------------------------------------------------- */
/* Learning the table of each row.
 *
 * Follows the quantisation procedure of the same paper, for n-bit codes
 * (§4.1 Eq. 9: a set of 2^n values per row, "any n"; n = 4 is any4, and §5
 * evaluates any3 and any2):
 *   - §2.5.1 Eq. 1-2: per group of G columns, alpha = (max - min) / (Qmax - Qmin)
 *     with Qmax - Qmin = 2^n - 1, beta = min, and the scaled weight
 *     w_S = (w - beta) / alpha;
 *   - §4.1 E-step (Eq. 18): each scaled weight takes the nearest table entry;
 *   - §4.1 M-step (Eq. 23): each entry becomes the mean of its cluster's
 *     scaled weights, weighted by alpha_{i,j} * E|x_j|;
 *   - §4.1 / Appendix A.1 (Alg. 1): rows are independent; the steps
 *     alternate until the table stops changing.
 * Readings where the pages leave a step open:
 *   - w is bf16 (its -0 is read as +0); E|x_j| is fp32, >= 0, one per column.
 *   - alpha is the bf16 rounding of the fp32 quotient (max - min) / (2^n - 1)
 *     (both fp32 operations correctly rounded) and beta = min (exact in
 *     bf16); the k-means runs on w_S formed with these stored values, in fp64:
 *     w_S = ((double)w - beta) / alpha, or 0 for every column of a group
 *     whose stored alpha is 0.
 *   - Sample weight u_j = alpha_{g(j)} * E|x_j| in fp64 (exact: 8 x 24 bits).
 *   - Initial table: the quantiles of the row's sorted w_S, entry q at
 *     position floor(q (K - 1) / (2^n - 1)) (deterministic; scikit-learn's
 *     k-means++ seeding draws random numbers).
 *   - E-step: nearest by |w_S - c_q| in fp64, ties to the lowest q.
 *   - M-step: numerator and denominator summed in fp64 over ascending column
 *     index, each product rounded before its add; a cluster whose weights
 *     sum to 0 (empty, or all weights 0) keeps its entry.
 *   - Stop after max_iter M-steps, or as soon as an E-step changes no code.
 *   - Table: LUT_q = bf16_rne((float)c_q); the returned codes are a final
 *     E-step against these stored bf16 entries (the values dequant uses).
 */

static float canon_bf16(uint16_t h) { return oracle_bf16_to_f32(h) + 0.0f; }

/* Eq. 1-2 on every group: scale = bf16(alpha), offset = bf16(beta) = min. */
void oracle_group_scale_bits(const uint16_t* w, int64_t N, int64_t K, int64_t G, int bits,
                             uint16_t* scale, uint16_t* offset) {
  const float levels = (float)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < K / G; ++g) {
      float mn = canon_bf16(w[n * K + g * G]);
      float mx = mn;
      for (int64_t k = g * G; k < (g + 1) * G; ++k) {
        float v = canon_bf16(w[n * K + k]);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      float alpha = (mx - mn) / levels;
      scale[n * (K / G) + g] = oracle_bf16_rne(alpha);
      offset[n * (K / G) + g] = oracle_bf16_rne(mn);
    }
  }
}

void oracle_group_scale(const uint16_t* w, int64_t N, int64_t K, int64_t G, uint16_t* scale,
                        uint16_t* offset) {
  oracle_group_scale_bits(w, N, K, G, 4, scale, offset);
}

/* w_S = (w - beta) / alpha for one row, with the stored bf16 alpha and beta
 * (0 where alpha is 0). */
static void scaled_row(const uint16_t* w, const uint16_t* scale, const uint16_t* offset,
                       int64_t K, int64_t G, double* ws) {
  for (int64_t k = 0; k < K; ++k) {
    double alpha = (double)oracle_bf16_to_f32(scale[k / G]);
    double beta = (double)oracle_bf16_to_f32(offset[k / G]);
    ws[k] = alpha > 0.0 ? ((double)canon_bf16(w[k]) - beta) / alpha : 0.0;
  }
}

void oracle_scaled_weights(const uint16_t* w, const uint16_t* scale, const uint16_t* offset,
                           int64_t N, int64_t K, int64_t G, double* ws) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    scaled_row(w + n * K, scale + n * (K / G), offset + n * (K / G), K, G, ws + n * K);
}

static int cmp_double(const void* a, const void* b) {
  double x = *(const double*)a, y = *(const double*)b;
  return (x > y) - (x < y);
}

/* E-step (Eq. 18): nearest of the nq entries, ties to the lowest index.
 * Returns how many codes changed. */
static int64_t assign_nearest(const double* xs, int64_t K, const double* c, int nq,
                              uint8_t* code) {
  int64_t changed = 0;
  for (int64_t j = 0; j < K; ++j) {
    int best_q = 0;
    double best = fabs(xs[j] - c[0]);
    for (int q = 1; q < nq; ++q) {
      double d = fabs(xs[j] - c[q]);
      if (d < best) {
        best = d;
        best_q = q;
      }
    }
    if (code[j] != (uint8_t)best_q) ++changed;
    code[j] = (uint8_t)best_q;
  }
  return changed;
}

/* Weighted Lloyd iteration on one row with nq entries: samples xs[0..K),
 * weights u[0..K).  Out: c[nq] (fp64 centroids) and code[K] (the E-step
 * matching c).  Returns the number of M-steps run. */
static int64_t kmeans_row(const double* xs, const double* u, int64_t K, int nq,
                          int64_t max_iter, double* c, uint8_t* code) {
  double* sorted = (double*)malloc((size_t)K * sizeof(double));
  memcpy(sorted, xs, (size_t)K * sizeof(double));
  qsort(sorted, (size_t)K, sizeof(double), cmp_double);
  for (int q = 0; q < nq; ++q) c[q] = sorted[(q * (K - 1)) / (nq - 1)];
  free(sorted);

  memset(code, 0, (size_t)K);
  assign_nearest(xs, K, c, nq, code);
  int64_t it = 0;
  while (it < max_iter) {
    double num[16], den[16];
    for (int q = 0; q < nq; ++q) num[q] = den[q] = 0.0;
    for (int64_t j = 0; j < K; ++j) {           /* M-step (Eq. 23) */
      num[code[j]] += u[j] * xs[j];
      den[code[j]] += u[j];
    }
    for (int q = 0; q < nq; ++q)
      if (den[q] > 0.0) c[q] = num[q] / den[q];
    ++it;
    if (assign_nearest(xs, K, c, nq, code) == 0) break;
  }
  return it;
}

int64_t oracle_kmeans_row_bits(const double* xs, const double* u, int64_t K, int bits,
                               int64_t max_iter, double* c, uint8_t* code) {
  return kmeans_row(xs, u, K, 1 << bits, max_iter, c, code);
}

int64_t oracle_kmeans_row(const double* xs, const double* u, int64_t K, int64_t max_iter,
                          double* c, uint8_t* code) {
  return kmeans_row(xs, u, K, 16, max_iter, c, code);
}

/* The whole quantiser for an [N][K] bf16 weight and n-bit codes: scale,
 * offset, LUT [N][2^n] and codes [N][K].  iters[n] (may be NULL) receives the
 * M-steps run on row n. */
void oracle_quantize_bits(const uint16_t* w, const float* ex, int64_t N, int64_t K, int64_t G,
                          int bits, int64_t max_iter, uint8_t* code, uint16_t* lut,
                          uint16_t* scale, uint16_t* offset, int64_t* iters) {
  const int nq = 1 << bits;
  oracle_group_scale_bits(w, N, K, G, bits, scale, offset);
#pragma omp parallel for schedule(dynamic)
  for (int64_t n = 0; n < N; ++n) {
    double* xs = (double*)malloc((size_t)K * sizeof(double));
    double* u = (double*)malloc((size_t)K * sizeof(double));
    scaled_row(w + n * K, scale + n * (K / G), offset + n * (K / G), K, G, xs);
    for (int64_t k = 0; k < K; ++k)
      u[k] = (double)oracle_bf16_to_f32(scale[n * (K / G) + k / G]) * (double)ex[k];
    double c[16], table[16];
    int64_t it = kmeans_row(xs, u, K, nq, max_iter, c, code + n * K);
    if (iters) iters[n] = it;
    for (int q = 0; q < nq; ++q) {
      lut[n * nq + q] = oracle_bf16_rne((float)c[q]);
      table[q] = (double)oracle_bf16_to_f32(lut[n * nq + q]);
    }
    assign_nearest(xs, K, table, nq, code + n * K);
    free(xs);
    free(u);
  }
}

void oracle_any4_quantize(const uint16_t* w, const float* ex, int64_t N, int64_t K, int64_t G,
                          int64_t max_iter, uint8_t* code, uint16_t* lut, uint16_t* scale,
                          uint16_t* offset, int64_t* iters) {
  oracle_quantize_bits(w, ex, N, K, G, 4, max_iter, code, lut, scale, offset, iters);
}

/* ------------------------------------------------------------------------- */
/* n-bit storage (any3, any2; any4 is n = 4).  The pages give no layout below
 * 4 bits.  Reading: the codes of a row form one little-endian bit stream,
 * code k in bits [n k, n k + n) (bit i of the stream is bit i % 8 of byte
 * i / 8); for n = 4 this is the nibble order above.  A row of K codes takes
 * n K / 8 bytes (K % 8 == 0).  The table of a row has 2^n bf16 entries.      */
/* ------------------------------------------------------------------------- */

/* Returns how many codes were >= 2^bits (they are packed masked). */
int64_t oracle_pack_bits(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K, int bits) {
  const int64_t row_bytes = bits * K / 8;
  const unsigned mask = (1u << bits) - 1u;
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    uint8_t* row = packed + n * row_bytes;
    memset(row, 0, (size_t)row_bytes);
    for (int64_t k = 0; k < K; ++k) {
      unsigned c = idx[n * K + k];
      if (c > mask) ++bad;
      for (int b = 0; b < bits; ++b) {
        int64_t bit = (int64_t)bits * k + b;
        if ((c >> b) & 1u) row[bit / 8] |= (uint8_t)(1u << (bit % 8));
      }
    }
  }
  return bad;
}

static unsigned code_at_bits(const uint8_t* row, int64_t k, int bits) {
  unsigned c = 0;
  for (int b = 0; b < bits; ++b) {
    int64_t bit = (int64_t)bits * k + b;
    c |= (unsigned)((row[bit / 8] >> (bit % 8)) & 1u) << b;
  }
  return c;
}

void oracle_unpack_bits(const uint8_t* packed, uint8_t* idx, int64_t N, int64_t K, int bits) {
  const int64_t row_bytes = bits * K / 8;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      idx[n * K + k] = (uint8_t)code_at_bits(packed + n * row_bytes, k, bits);
}

/* W[n][k] = bf16_rne(fmaf(LUT[n][c], scale, offset)) with c the n-bit code;
 * lut_row_stride is 2^bits (a table per row) or 0 (one table). */
void oracle_dequant_bits(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                         const uint16_t* scale, const uint16_t* offset, uint16_t* W, int64_t N,
                         int64_t K, int64_t G, int bits) {
  const int64_t row_bytes = bits * K / 8;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      unsigned c = code_at_bits(packed + n * row_bytes, k, bits);
      int64_t g = k / G;
      W[n * K + k] = oracle_dequant_one(lut[n * lut_row_stride + c], scale[n * (K / G) + g],
                                        offset[n * (K / G) + g]);
    }
  }
}

/* Storage per weight for n-bit codes: n + (2 x 16-bit group parameters) / G +
 * 2^n x 16-bit table entries / K (the §2.4.1 accounting for any n). */
double oracle_bits_per_weight_n(int64_t K, int64_t G, int bits) {
  return (double)bits + 32.0 / (double)G + (16.0 * (double)(1 << bits)) / (double)K;
}

/* Per-group sums of the activations: xsum[m][g] = sum over the columns k of
 * group g (k = g*G .. g*G+G-1, §2.5.1) of x[m][k], in fp64, k ascending.
 * This is the factor that multiplies the group offset beta when Eq. 8's
 * product is taken with the group-affine weights alpha*LUT[c] + beta
 * (§4.1 Eq. 8, §2.5.2):  sum_k x*(alpha*LUT + beta)
 *   = alpha * sum_k x*LUT + beta * xsum.
 * x: [M][K] bf16, xsum: [M][K/G] fp64. */
void oracle_group_sums(const uint16_t* x, double* xsum, int64_t M, int64_t K, int64_t G) {
  const int64_t groups = K / G;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t g = 0; g < groups; ++g) {
      double acc = 0.0;
      for (int64_t k = g * G; k < (g + 1) * G; ++k) acc += (double)oracle_bf16_to_f32(x[m * K + k]);
      xsum[m * groups + g] = acc;
    }
  }
}
