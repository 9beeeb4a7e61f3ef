"""Prefill-path any4_matmul (tcgen05 tensor cores) on the GPU against the oracle.

Full-size M = 2048 shapes are checked on sampled weight rows (every x row of
each sampled weight row), computed one by one by the oracle; smaller shapes
are checked in full.  Tolerance as for the decode path."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import (DeviceProblem, assert_matmul_close, bits_to_f64, dev_bf16,
                               host_bits)
from tests.oracle_pins import torch_bf16_bits

pytestmark = pytest.mark.gpu


def _run(d, shape, path="prefill", status=None):
    y = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, path=path,
                         dev_status=status)
    torch.cuda.synchronize()
    return y


def sampled_x_rows(M, seed, n_random=16):
    """Rows of x (rows of y) to check at full size: both edges of the first
    two 256-row tiles, the last row, and random rows."""
    rng = np.random.default_rng(seed)
    fixed = [r for r in (0, 1, 127, 128, 255, 256, M - 1) if r < M]
    return np.unique(np.concatenate([fixed, rng.choice(M, min(M, n_random), replace=False)]))


@pytest.mark.parametrize("shape", workloads.PREFILL, ids=lambda s: s.name)
def test_prefill_full_shapes_sampled_rows(shape):
    """Full-size M = 2048 shapes: sampled rows of x, each whole output row
    computed by the oracle, so the tolerance uses the rms of the full row."""
    p = workloads.make(shape)
    d = DeviceProblem(p)
    assert any4.any4_matmul_choose_path(shape.M, shape.N, shape.K, shape.G) == "prefill"
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = host_bits(_run(d, shape, path="auto", status=status))
    assert int(status.item()) == 0
    rows = sampled_x_rows(shape.M, shape.weight_seed)
    y_ref = oracle.any4_matmul(p.x[rows], d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    st = assert_matmul_close(y[rows], y_ref, shape.name)
    print(shape.name, "sampled x rows", len(rows), st)


SMALL = [
    workloads.Shape("pf_ragged", 300, 1056, 520, 32, 9701, 9711),     # M, N, K all ragged
    workloads.Shape("pf_one_tile", 256, 1024, 256, 128, 9702, 9712),
    workloads.Shape("pf_g64", 520, 4096, 777, 64, 9703, 9713, "student_t4"),
    workloads.Shape("pf_kmin", 129, 32, 300, 32, 9704, 9714),
    workloads.Shape("pf_many_tiles", 1030, 2048, 2304, 128, 9705, 9715),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
def test_prefill_small_shapes_full(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = host_bits(_run(d, shape, status=status))
    assert int(status.item()) == 0
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(y, y_ref, shape.name)


@pytest.mark.parametrize("M", [1, 2, 7, 16, 17, 31, 32, 33])
def test_prefill_any_m(M):
    shape = workloads.Shape(f"pf_m{M}", M, 2048, 640, 128, 9801, 9820 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    y = host_bits(_run(d, shape))
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(y, y_ref, shape.name)


def test_sweep_m32_takes_prefill():
    shape = [s for s in workloads.SKINNY_SWEEP if s.M == 32][0]
    p = workloads.make(shape)
    d = DeviceProblem(p)
    assert any4.any4_matmul_choose_path(shape.M, shape.N, shape.K, shape.G) == "prefill"
    y = host_bits(_run(d, shape, path="auto"))
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(y, y_ref, shape.name)


def test_prefill_identity_is_exact():
    """x = I (M = K) returns W^T bit for bit: every output is one product."""
    K = 1024
    shape = workloads.Shape("pf_identity", K, K, 700, 128, 9901, 9902)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    eye = torch_bf16_bits(np.eye(K, dtype=np.float32))
    y = any4.any4_matmul(dev_bf16(eye), d.packed, d.lut, d.scale, d.offset, shape.G,
                         path="prefill")
    torch.cuda.synchronize()
    W_ref = oracle.dequant(d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    got = bits_to_f64(host_bits(y))
    assert np.array_equal(got, bits_to_f64(W_ref).T)


def test_prefill_deterministic_and_shared_table():
    shape = workloads.Shape("pf_shared", 384, 2048, 1000, 128, 9911, 9912)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    table = p.lut[5].copy()
    t = dev_bf16(table)
    y1 = any4.any4_matmul(d.x, d.packed, t, d.scale, d.offset, shape.G, path="prefill")
    y2 = any4.any4_matmul(d.x, d.packed, t, d.scale, d.offset, shape.G, path="prefill")
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, table, p.scale, p.offset, shape.G,
                               per_tensor_lut=True)
    assert_matmul_close(host_bits(y1), y_ref, "shared")


def test_prefill_one_pass_with_small_workspace():
    """At M >= 1024 the full workspace selects the two-pass kernel (weights
    dequantised into it first); a workspace of only the one-pass size must
    run the one-pass kernel instead, with the same accuracy."""
    shape = workloads.Shape("pf_onepass", 1024, 2048, 1100, 128, 9971, 9972)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    one_pass = any4.any4_matmul_workspace_size(300, shape.N, shape.K, shape.G)
    full = any4.any4_matmul_workspace_size(shape.M, shape.N, shape.K, shape.G)
    assert full >= one_pass + shape.N * shape.K * 2
    ws = torch.empty(one_pass, dtype=torch.uint8, device="cuda")
    y1 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, workspace=ws,
                          path="prefill")
    y2 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, path="prefill")
    torch.cuda.synchronize()
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(host_bits(y1), y_ref, "one pass")
    assert_matmul_close(host_bits(y2), y_ref, "two passes")


@pytest.mark.parametrize("M,K,N,G,shared", [(1030, 1056, 777, 32, False),
                                            (1024, 2080, 300, 32, True),
                                            (1500, 1024, 513, 64, False)])
def test_prefill_two_pass_edges(M, K, N, G, shared):
    """The two-pass kernel (M >= 1024, full workspace) with a ragged last
    K stage (K % 64 == 32), ragged M and N, the one-table mode and G = 32."""
    shape = workloads.Shape(f"pf2_{M}_{K}_{N}", M, K, N, G, 9981 + N, 9982 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    lut = p.lut[7 % N].copy() if shared else p.lut
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = any4.any4_matmul(d.x, d.packed, dev_bf16(lut), d.scale, d.offset, shape.G,
                         path="prefill", dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, lut, p.scale, p.offset, shape.G,
                               per_tensor_lut=shared)
    assert_matmul_close(host_bits(y), y_ref, shape.name)
