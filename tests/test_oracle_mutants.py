"""Every plausible mistake planted in a copy of the oracle source must fail at
least one pin (CPU only).  The real oracle source is never modified: each
mutant is a text substitution compiled into a temporary library."""
import os
import subprocess

import pytest

import oracle
from oracle import build as oracle_build
from tests import oracle_pins

# (name, original text, planted mistake)
MUTANTS = [
    ("nibble_order_unpack", "(k % 2 == 0) ? (byte & 15u) : (byte >> 4)",
     "(k % 2 == 0) ? (byte >> 4) : (byte & 15u)"),
    ("nibble_order_pack", "(uint8_t)((lo & 15u) | ((hi & 15u) << 4))",
     "(uint8_t)((hi & 15u) | ((lo & 15u) << 4))"),
    ("scale_offset_swapped", "fmaf(oracle_bf16_to_f32(lut_c), oracle_bf16_to_f32(scale),\n"
     "                 oracle_bf16_to_f32(offset))",
     "fmaf(oracle_bf16_to_f32(lut_c), oracle_bf16_to_f32(offset),\n"
     "                 oracle_bf16_to_f32(scale))"),
    ("offset_dropped", "oracle_bf16_to_f32(offset));\n  return oracle_bf16_rne(w);",
     "0.0f); (void)offset;\n  return oracle_bf16_rne(w);"),
    # (a plain multiply-then-add equals fmaf for bf16 operands: the 8x8-bit
    # product is exact in fp32, so only a perturbed product is a real mistake)
    ("perturbed_product", "float w = fmaf(oracle_bf16_to_f32(lut_c), oracle_bf16_to_f32(scale),\n"
     "                 oracle_bf16_to_f32(offset));",
     "float w = (float)(oracle_bf16_to_f32(lut_c) * oracle_bf16_to_f32(scale));\n"
     "  w = (float)(w * 1.0009765625f) + oracle_bf16_to_f32(offset);"),
    ("truncate_not_round", "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) {",
     "if (0) {"),
    ("ties_away", "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) {",
     "if (dropped >= 0x8000u) {"),
    ("group_off_by_one", "      int64_t g = k / G;\n      W[n * K + k]",
     "      int64_t g = (k + 1) / G; if (g >= K / G) g = K / G - 1;\n      W[n * K + k]"),
    ("lut_of_row_zero", "lut[n * lut_row_stride + c],\n                                        scale",
     "lut[c],\n                                        scale"),
    ("scale_of_row_zero", "scale[n * (K / G) + g],\n                                        offset",
     "scale[g],\n                                        offset"),
    ("matmul_drops_last_term", "for (int64_t k = 0; k < K; ++k) {\n        acc += (double)oracle_bf16_to_f32(x[m * K + k]) *\n",
     "for (int64_t k = 0; k < K - 1; ++k) {\n        acc += (double)oracle_bf16_to_f32(x[m * K + k]) *\n"),
    ("matmul_sign", "        acc += (double)oracle_bf16_to_f32(x[m * K + k]) *\n               (double)oracle_bf16_to_f32(W[n * K + k]);",
     "        acc += (double)oracle_bf16_to_f32(x[m * K + k]) *\n               (double)oracle_bf16_to_f32(W[n * K + k]) * (k == 3 ? -1.0 : 1.0);"),
    ("matmul_fp32_accumulate", "      double acc = 0.0;\n      for (int64_t k = 0; k < K; ++k) {\n        acc += (double)oracle_bf16_to_f32(x[m * K + k])",
     "      float acc = 0.0f;\n      for (int64_t k = 0; k < K; ++k) {\n        acc += (float)oracle_bf16_to_f32(x[m * K + k])"),
    ("matmul_rows_wrong_row", "    int64_t n = rows[r];", "    int64_t n = rows[r] + (r > 0);"),
    ("widen_wrong_shift", "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    ("alpha_over_16", "float alpha = (mx - mn) / levels;", "float alpha = (mx - mn) / (levels + 1.0f);"),
    ("beta_is_max", "offset[n * (K / G) + g] = oracle_bf16_rne(mn);",
     "offset[n * (K / G) + g] = oracle_bf16_rne(mx);"),
    ("scaled_without_offset", "ws[k] = alpha > 0.0 ? ((double)canon_bf16(w[k]) - beta) / alpha : 0.0;",
     "ws[k] = alpha > 0.0 ? (double)canon_bf16(w[k]) / alpha : 0.0; (void)beta;"),
    ("quantile_off_by_one", "c[q] = sorted[(q * (K - 1)) / (nq - 1)];", "c[q] = sorted[(q * K) / nq];"),
    ("ties_to_highest", "      if (d < best) {", "      if (d <= best) {"),
    ("mstep_unweighted", "      num[code[j]] += u[j] * xs[j];\n      den[code[j]] += u[j];",
     "      num[code[j]] += xs[j];\n      den[code[j]] += 1.0;"),
    ("mstep_weight_squared", "      num[code[j]] += u[j] * xs[j];\n      den[code[j]] += u[j];",
     "      num[code[j]] += u[j] * u[j] * xs[j];\n      den[code[j]] += u[j] * u[j];"),
    ("empty_cluster_zeroed", "if (den[q] > 0.0) c[q] = num[q] / den[q];",
     "c[q] = den[q] > 0.0 ? num[q] / den[q] : 0.0;"),
    ("sample_weight_without_alpha",
     "u[k] = (double)oracle_bf16_to_f32(scale[n * (K / G) + k / G]) * (double)ex[k];",
     "u[k] = (double)ex[k];"),
    ("codes_from_unrounded_centroids", "    assign_nearest(xs, K, table, nq, code + n * K);\n", "\n"),
    ("one_lloyd_step_only", "    if (assign_nearest(xs, K, c, nq, code) == 0) break;",
     "    assign_nearest(xs, K, c, nq, code);\n    break;"),
    ("pack_bits_msb_first", "if ((c >> b) & 1u) row[bit / 8] |= (uint8_t)(1u << (bit % 8));",
     "if ((c >> b) & 1u) row[bit / 8] |= (uint8_t)(0x80u >> (bit % 8));"),
    ("unpack_bits_reversed", "c |= (unsigned)((row[bit / 8] >> (bit % 8)) & 1u) << b;",
     "c |= (unsigned)((row[bit / 8] >> (bit % 8)) & 1u) << (bits - 1 - b);"),
    ("dequant_bits_row_zero_table",
     "W[n * K + k] = oracle_dequant_one(lut[n * lut_row_stride + c], scale[n * (K / G) + g],",
     "W[n * K + k] = oracle_dequant_one(lut[c], scale[n * (K / G) + g],"),
    ("levels_is_two_to_the_n", "const float levels = (float)((1 << bits) - 1);",
     "const float levels = (float)(1 << bits);"),
    ("bits_per_weight_n_sixteen_entries",
     "return (double)bits + 32.0 / (double)G + (16.0 * (double)(1 << bits)) / (double)K;",
     "return (double)bits + 32.0 / (double)G + (16.0 * 16.0) / (double)K;"),
    ("group_sums_boundary_shifted", "for (int64_t k = g * G; k < (g + 1) * G; ++k) acc +=",
     "for (int64_t k = g * G + (g > 0); k < (g + 1) * G + (g + 1 < groups); ++k) acc +="),
    ("group_sums_row_zero", "acc += (double)oracle_bf16_to_f32(x[m * K + k]);\n      xsum",
     "acc += (double)oracle_bf16_to_f32(x[k]);\n      xsum"),
    ("group_sums_fp32_accumulate", "      double acc = 0.0;\n      for (int64_t k = g * G;",
     "      float acc = 0.0f;\n      for (int64_t k = g * G;"),
    ("storage_bits_one_param", "4.0 + (2.0 * (double)group_param_bits) / (double)G",
     "4.0 + (1.0 * (double)group_param_bits) / (double)G"),
    ("repack_without_xor", "int64_t col = 1024 * s + 128 * (4 * h + (t ^ h)) + 8 * e;",
     "int64_t col = 1024 * s + 128 * (4 * h + t) + 8 * e;"),
    ("repack_halves_interleaved", "int h = l / 16, e = l % 16;", "int h = l % 2, e = l / 2;"),
    ("repack_steps_reversed", "int64_t at = 512 * s + 16 * l + 4 * t;",
     "int64_t at = 512 * s + 16 * l + 4 * (3 - t);"),
]


@pytest.mark.parametrize("name,orig,mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, orig, mutant):
    src = open(oracle_build.SRC).read()
    assert src.count(orig) >= 1, f"mutation site for {name} not found in the oracle source"
    bad = src.replace(orig, mutant, 1)
    c_path = tmp_path / f"{name}.c"
    so_path = tmp_path / f"lib{name}.so"
    c_path.write_text(bad)
    subprocess.run(["gcc", *[f for f in oracle_build.CFLAGS if not f.startswith("-W")],
                    str(c_path), "-o", str(so_path), "-lm"], check=True)
    failed = []
    with oracle.swapped_library(str(so_path)):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except Exception as e:  # AssertionError, or a crash of the wrapper
                failed.append((pin.__name__, type(e).__name__))
                break
    assert failed, f"planted mistake {name!r} passed every pin"
