"""Decode-path any4_matmul (M <= 16) on the GPU against the fp64 oracle.

Tolerance: |y - y_ref| <= 1e-2 * rms(y_ref[m, :]) + ulp_bf16(y_ref) per
element (the stated 1e-2 * rms per output row, plus one bf16 ulp because even
the correctly rounded bf16 of y_ref exceeds 1e-2 * rms on heavy-tailed rows).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import (DeviceProblem, assert_matmul_close, bits_to_f64, dev_bf16,
                               dev_u8, host_bits)
from tests.oracle_pins import torch_bf16_bits

pytestmark = pytest.mark.gpu

DECODE_SHAPES = (workloads.TINY + workloads.LLAMA3_8B_DECODE
                 + [s for s in workloads.SKINNY_SWEEP if s.M <= 16]
                 + workloads.LLAMA3_70B_DECODE)


NO_WORKSPACE = "no_workspace"
PAIR = "pair_table"


def _ws_args(workspace):
    """workspace None: the binding allocates what the path asks for (M = 2
    then runs the pair-table kernel, M = 1 the weight-streaming kernel);
    NO_WORKSPACE: none is passed, so M = 2 runs the skinny kernel; PAIR: the
    workspace plus ANY4_FLAG_PAIR_TABLE, the pair-table kernel at M = 1 too."""
    if workspace == NO_WORKSPACE:
        return dict(workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    if workspace == PAIR:
        return dict(workspace=None, pair_table=True)
    return dict(workspace=workspace)


def _run(d, shape, path="auto", workspace=None):
    y = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, path=path,
                         **_ws_args(workspace))
    torch.cuda.synchronize()
    return host_bits(y)


@pytest.mark.parametrize("shape", DECODE_SHAPES, ids=lambda s: s.name)
def test_decode_full_shapes(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p)
    assert any4.any4_matmul_choose_path(shape.M, shape.N, shape.K, shape.G) == "decode"
    y = _run(d, shape)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    st = assert_matmul_close(y, y_ref, shape.name)
    print(shape.name, st)
    if shape.M <= 2:
        # the same shape on the other kernel that takes it
        other = PAIR if shape.M == 1 else NO_WORKSPACE
        y = _run(d, shape, workspace=other)
        st = assert_matmul_close(y, y_ref, f"{shape.name} {other}")
        print(shape.name, other, st)


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_decode_every_m_ragged(M):
    """Every M the decode path takes, on a shape with a ragged last slice
    (K = 1056 is not a multiple of the 1024-column slice) and ragged rows."""
    shape = workloads.Shape(f"ragged_m{M}", M, 1056, 333, 32, 9201, 9700 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    for ws in (None, NO_WORKSPACE, PAIR):
        y = _run(d, shape, path="decode", workspace=ws)
        assert_matmul_close(y, y_ref, f"{shape.name} {ws}")


@pytest.mark.parametrize("K,N,G", [(32, 1, 32), (64, 7, 32), (96, 7, 32), (96, 1000, 32),
                                   (2048, 5, 64), (33792, 40, 128)])
def test_decode_edge_shapes(K, N, G):
    """Tiny and ragged shapes; (32, 1, 32) and (96, 7, 32) end the scale and
    offset tensors on a lone group at an even flat index (N * K/G odd)."""
    for M in (1, 2, 3):
        shape = workloads.Shape(f"edge_{K}_{N}_m{M}", M, K, N, G, 9300 + N, 9800 + K // 32)
        p = workloads.make(shape)
        d = DeviceProblem(p)
        y = _run(d, shape, path="decode")
        y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
        assert_matmul_close(y, y_ref, shape.name)


@pytest.mark.parametrize("workspace", [PAIR, None])
def test_decode_one_hot_is_exact(workspace):
    """x = e_k returns column k of the dequantised weight, bit for bit: the
    fused group-affine form reduces to fmaf(LUT, scale, offset) rounded once.
    Both M = 1 kernels (pair table on request, weight streaming by default)."""
    shape = workloads.Shape("onehot", 1, 4096, 2000, 128, 9401, 9901)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    W_ref = oracle.dequant(d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    one = torch_bf16_bits(np.array([1.0], np.float32))[0]
    for k in (0, 1, 31, 32, 127, 128, 1023, 1024, 2047, 4095):
        x = np.zeros((1, shape.K), np.uint16)
        x[0, k] = one
        y = any4.any4_matmul(dev_bf16(x), d.packed, d.lut, d.scale, d.offset, shape.G,
                             **_ws_args(workspace))
        torch.cuda.synchronize()
        got = bits_to_f64(host_bits(y))[0]
        assert np.array_equal(got, bits_to_f64(W_ref[:, k])), k


def test_decode_zero_x_and_determinism():
    shape = workloads.LLAMA3_8B_DECODE[4]
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    z = torch.zeros_like(d.x)
    y0 = any4.any4_matmul(z, d.packed, d.lut, d.scale, d.offset, shape.G)
    y1 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G)
    y2 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G)
    torch.cuda.synchronize()
    assert (bits_to_f64(host_bits(y0)) == 0).all()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_decode_shared_table():
    shape = workloads.Shape("shared_m4", 4, 4096, 1536, 128, 9501, 9951)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    table = p.lut[3].copy()
    y = any4.any4_matmul(d.x, d.packed, dev_bf16(table), d.scale, d.offset, shape.G)
    torch.cuda.synchronize()
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, table, p.scale, p.offset, shape.G,
                               per_tensor_lut=True)
    assert_matmul_close(host_bits(y), y_ref, "shared")


@pytest.mark.parametrize("M", [1, 2, 5])
def test_decode_writes_only_its_output(M):
    """Guard bands around y stay untouched."""
    shape = workloads.Shape(f"guard_m{M}", M, 1024, 999, 64, 9601, 9961)
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    pad = 4096
    buf = torch.full((pad + shape.M * shape.N + pad,), -7, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + shape.M * shape.N].view(shape.M, shape.N).view(torch.bfloat16)
    any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, y=y)
    torch.cuda.synchronize()
    assert (buf[:pad] == -7).all() and (buf[pad + shape.M * shape.N:] == -7).all()
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(host_bits(y), y_ref, "guard")


@pytest.mark.parametrize("M,workspace", [(1, PAIR), (2, None), (1, None), (2, NO_WORKSPACE),
                                         (4, None), (12, None)])
def test_decode_overlap_prior_chain(M, workspace):
    """ANY4_FLAG_OVERLAP_PRIOR: x is produced by the kernel just before each
    call and y is consumed by the kernel just after; a chain of overlapped
    calls must match the same chain run without overlap, bit for bit, and the
    oracle within tolerance (M = 1: weight streaming, or the pair-table
    kernel on request; M = 2: pair table, or skinny without a workspace;
    M > 2: skinny)."""
    shape = workloads.Shape(f"overlap_m{M}", M, 4096, 4096, 128, 9701, 9702 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    wa = _ws_args(workspace)
    def chain(overlap):
        x = d.x.clone()
        outs = []
        for i in range(6):
            x = (x.float() * 0.5 + 0.25).to(torch.bfloat16)      # written by the preceding kernel
            y = any4.any4_matmul(x, d.packed, d.lut, d.scale, d.offset, shape.G,
                                 overlap_prior=overlap, **wa)
            outs.append(y.clone())                              # read by the following kernel
            x = torch.cat([y[:, :shape.K]], dim=1) if shape.N >= shape.K else x
            x = (x.float() / (x.float().abs().max() + 1)).to(torch.bfloat16)
        torch.cuda.synchronize()
        return outs
    a = chain(False)
    b = chain(True)
    for ya, yb in zip(a, b):
        assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    y1 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, overlap_prior=True,
                          **wa)
    torch.cuda.synchronize()
    assert_matmul_close(host_bits(y1), y_ref, "overlap")


@pytest.mark.parametrize("K,N,G,shared", [(1024, 1000, 32, False), (1280, 777, 32, False),
                                          (3072, 300, 64, False), (8192, 2050, 128, False),
                                          (4096, 1500, 128, True), (2048, 9, 64, True)])
def test_decode_m1_streamed_variants(K, N, G, shared):
    """M = 1 shapes of both tensor-memory-streamed decode kernels (the
    pair-table kernel on request, the shuffle kernel by default): every
    group size they take, ragged rows, a last slice cut short, the one table
    mode; dev_status must stay clear."""
    shape = workloads.Shape(f"m1_{K}_{N}_{G}", 1, K, N, G, 9901 + K + N, 9951 + G)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    lut = p.lut[11 % N].copy() if shared else p.lut
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, lut, p.scale, p.offset, shape.G,
                               per_tensor_lut=shared)
    for ws in (PAIR, None):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = any4.any4_matmul(d.x, d.packed, dev_bf16(lut), d.scale, d.offset, shape.G,
                             dev_status=status, **_ws_args(ws))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_matmul_close(host_bits(y), y_ref, f"{shape.name} {ws}")
