"""any4_quantize (learning the per-row tables on the GPU) against the oracle.

The quantiser is group-wise scaling (paper §2.5.1 Eq. 1-2) followed by a
weighted k-means per row (§4.1 E-step Eq. 18, M-step Eq. 23; Appendix A.1).
Every step is taken in the same precision and order on both sides, so codes,
tables, scales, offsets and iteration counts must agree bit for bit.  At the
full Llama3-8B layer sizes the oracle checks sampled rows (rows are
independent) and every row's scale and offset.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import assert_matmul_close, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


def _gpu(w_bits, ex, G, max_iter):
    packed, lut, scale, offset, iters = any4.any4_quantize(
        dev_bf16(w_bits), torch.from_numpy(np.ascontiguousarray(ex, dtype=np.float32)).cuda(), G,
        max_iter, return_iters=True)
    torch.cuda.synchronize()
    return (packed.cpu().numpy(), host_bits(lut), host_bits(scale), host_bits(offset),
            iters.cpu().numpy())


def _assert_rows_equal(got, w_bits, ex, G, max_iter, rows=None):
    sub = w_bits if rows is None else w_bits[rows]
    codes, lut, scale, offset, iters = oracle.quantize(sub, ex, G, max_iter)
    if rows is not None:
        got = tuple(a[rows] for a in got)
    g_packed, g_lut, g_scale, g_offset, g_iters = got
    assert np.array_equal(g_scale, scale), "scale"
    assert np.array_equal(g_offset, offset), "offset"
    assert np.array_equal(g_iters, iters), "M-steps per row"
    assert np.array_equal(g_lut, lut), "table"
    assert np.array_equal(g_packed, oracle.pack(codes)), "codes"


def _problem(N, K, G, seed):
    s = workloads.QuantShape(f"q{N}x{K}", N, K, G, seed)
    return workloads.draw_dense_weight(s), workloads.draw_abs_act_mean(s)


@pytest.mark.parametrize("N,K,G,max_iter", [
    (64, 256, 64, 50),      # several rows, a sort of exactly K
    (37, 4096, 128, 100),   # a Llama row length, ragged row count
    (33, 160, 32, 30),      # K not a power of two: the sort pads to 256
    (3, 32, 32, 10),        # the smallest row
    (16, 1024, 32, 0),      # no M-step: the quantile table itself
    (16, 1024, 32, 1),      # one M-step
    (5, 16384, 128, 100),   # the longest row the kernel takes
    (7, 14336, 14336, 60),  # one group per row (G = K)
])
def test_quantize_matches_oracle(N, K, G, max_iter):
    w, ex = _problem(N, K, G, 7000 + N + K)
    _assert_rows_equal(_gpu(w, ex, G, max_iter), w, ex, G, max_iter)


def test_quantize_degenerate_rows_and_statistics():
    N, K, G = 12, 512, 64
    w, ex = _problem(N, K, G, 7100)
    w[0, :] = w[0, 3]                       # constant row: scale 0 everywhere
    w[1, G:3 * G] = w[1, G + 1]             # two constant groups
    w[2, :] = 0x8000                        # a row of -0 (read as +0)
    w[3, ::2] = 0x0000                      # +0 next to signed values
    w[4, 100:200] = 0x8000
    ex = ex.copy()
    ex[:K // 3] = 0.0                       # a third of the columns weigh nothing
    _assert_rows_equal(_gpu(w, ex, G, 40), w, ex, G, 40)
    # no activation weight at all: every cluster keeps its quantile entry
    zero = np.zeros(K, np.float32)
    _assert_rows_equal(_gpu(w, zero, G, 40), w, zero, G, 40)


def test_quantize_repeatable():
    w, ex = _problem(48, 2048, 128, 7200)
    a = _gpu(w, ex, 128, 80)
    b = _gpu(w, ex, 128, 80)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("shape", workloads.QUANTIZE_LLAMA3_8B, ids=lambda s: s.name)
def test_quantize_llama3_8b_layers_sampled_rows(shape):
    w = workloads.draw_dense_weight(shape)
    ex = workloads.draw_abs_act_mean(shape)
    got = _gpu(w, ex, shape.G, 100)
    # every row's scale and offset (Eq. 1-2), from the oracle over the whole matrix
    scale, offset = oracle.group_scale(w, shape.G)
    assert np.array_equal(got[2], scale) and np.array_equal(got[3], offset)
    rng = np.random.default_rng(shape.seed)
    rows = np.unique(np.concatenate([[0, shape.N - 1], rng.choice(shape.N, 10, replace=False)]))
    _assert_rows_equal(got, w, ex, shape.G, 100, rows)
    assert np.all(got[4] >= 1) and np.all(got[4] <= 100)


def test_quantized_weights_feed_the_matmul():
    """The quantiser's outputs are the matmul's inputs: the product with the
    learned representation matches the oracle's dequant-then-matmul."""
    N, K, G = 320, 1024, 128
    w, ex = _problem(N, K, G, 7300)
    packed, lut, scale, offset = any4.any4_quantize(
        dev_bf16(w), torch.from_numpy(ex).cuda(), G, 60)
    x = workloads.draw_x(workloads.Shape("qx", 6, K, N, G, 0, 7301))
    y = any4.any4_matmul(dev_bf16(x), packed, lut, scale, offset, G)
    torch.cuda.synchronize()
    codes, lut_r, scale_r, offset_r, _ = oracle.quantize(w, ex, G, 60)
    y_ref = oracle.any4_matmul(x, oracle.pack(codes), lut_r, scale_r, offset_r, G)
    assert_matmul_close(host_bits(y), y_ref, "quantize -> matmul")
