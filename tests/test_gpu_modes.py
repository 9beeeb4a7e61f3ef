"""The int4 and nf4-style modes through the same kernels (one 16-entry table
for the whole matrix, lut_row_stride = 0), on every matmul path.

int4: the table {-8..7} with offset' = beta + 8 alpha reproduces grouped
asymmetric int4 (paper §2.1, §2.5.1 Eq. 1-2, §2.5.2); nf4-style: one table
built from normal quantiles with an exact zero, as nf4/af4 use (§2.4.1; the
published nf4 constants are not on the pages).  References: the fp64 oracle in
its shared-table mode; any4_dequant bit for bit.
"""
from statistics import NormalDist

import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, bits_to_f64, dev_bf16, host_bits
from tests.oracle_pins import torch_bf16_bits

pytestmark = pytest.mark.gpu


def _int4_problem(shape):
    """Weights quantised to grouped asymmetric int4 (codes 0..15 by round to
    nearest), expressed as the table {-8..7}, scale alpha, offset beta + 8 alpha."""
    rng = np.random.default_rng(shape.weight_seed)
    N, K, G = shape.N, shape.K, shape.G
    w = rng.normal(0, 0.02, size=(N, K))
    wg = w.reshape(N, K // G, G)
    beta = wg.min(axis=2)
    alpha = (wg.max(axis=2) - beta) / 15.0
    idx = np.rint((wg - beta[..., None]) / alpha[..., None]).clip(0, 15).astype(np.uint8)
    table = torch_bf16_bits(np.arange(-8, 8, dtype=np.float32))
    scale = torch_bf16_bits(alpha.astype(np.float32))
    offset = torch_bf16_bits((beta + 8 * alpha).astype(np.float32))
    x = torch_bf16_bits(np.random.default_rng(shape.x_seed).normal(0, 1, (shape.M, K)).astype(np.float32))
    return idx.reshape(N, K), table, scale, offset, x


def _nf4_table():
    nd = NormalDist()
    neg = [-nd.inv_cdf(0.5 + 0.5 * (1 - (i + 0.5) / 8)) for i in range(8)]
    pos = [nd.inv_cdf(0.5 + 0.5 * (i + 1) / 8.5) for i in range(7)]
    t = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    t = t / np.abs(t).max()
    return torch_bf16_bits(t.astype(np.float32))


@pytest.mark.parametrize("M", [1, 4, 300])
def test_int4_mode_matmul(M):
    shape = workloads.Shape(f"int4_m{M}", M, 2048, 1000, 128, 9951, 9952)
    idx, table, scale, offset, x = _int4_problem(shape)
    packed_ref = oracle.pack(idx)
    packed = any4.any4_pack(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), packed_ref)
    y = any4.any4_matmul(dev_bf16(x), packed, dev_bf16(table), dev_bf16(scale), dev_bf16(offset),
                         shape.G)
    torch.cuda.synchronize()
    y_ref = oracle.any4_matmul(x, packed_ref, table, scale, offset, shape.G, per_tensor_lut=True)
    assert_matmul_close(host_bits(y), y_ref, shape.name)


def test_int4_mode_dequant_bit_exact():
    shape = workloads.Shape("int4_dq", 1, 1024, 777, 64, 9953, 9954)
    idx, table, scale, offset, _ = _int4_problem(shape)
    packed_ref = oracle.pack(idx)
    W = any4.any4_dequant(torch.from_numpy(packed_ref).cuda(), dev_bf16(table), dev_bf16(scale),
                          dev_bf16(offset), shape.G)
    torch.cuda.synchronize()
    W_ref = oracle.dequant(packed_ref, table, scale, offset, shape.G, per_tensor_lut=True)
    assert np.array_equal(host_bits(W), W_ref)
    # and the int4 reading itself: alpha * (q - 8) + (beta + 8 alpha) = alpha q + beta
    a = bits_to_f64(scale).repeat(shape.G, axis=1)
    o = bits_to_f64(offset).repeat(shape.G, axis=1)
    direct = (idx.astype(np.float64) - 8) * a + o
    assert np.allclose(bits_to_f64(host_bits(W)), direct, rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("M", [1, 8, 256])
def test_nf4_style_shared_table_matmul(M):
    shape = workloads.Shape(f"nf4_m{M}", M, 4096, 1536, 64, 9961, 9962 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    table = _nf4_table()
    y = any4.any4_matmul(d.x, d.packed, dev_bf16(table), d.scale, d.offset, shape.G)
    torch.cuda.synchronize()
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, table, p.scale, p.offset, shape.G,
                               per_tensor_lut=True)
    assert_matmul_close(host_bits(y), y_ref, shape.name)
