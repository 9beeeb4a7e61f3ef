"""any4_pack and any4_dequant on the GPU against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, dev_bf16, dev_u8, host_bits
from tests.oracle_pins import torch_bf16_bits

pytestmark = pytest.mark.gpu

FULL_SHAPES = (workloads.TINY + workloads.LLAMA3_8B_DECODE + [workloads.SKINNY_SWEEP[-1]]
               + [s for s in workloads.LLAMA3_70B_DECODE if s.M == 1] + workloads.PREFILL)

EDGE_SHAPES = [
    workloads.Shape("edge_min", 1, 32, 1, 32, 9001, 9501),
    workloads.Shape("edge_k_eq_g", 3, 128, 5, 128, 9002, 9502),
    workloads.Shape("edge_ragged", 2, 1056, 257, 32, 9003, 9503),
    workloads.Shape("edge_tail_chunks", 1, 96, 1000, 32, 9004, 9504),
    workloads.Shape("edge_g64", 1, 3072, 77, 64, 9005, 9505, "student_t4"),
]


@pytest.mark.parametrize("shape", FULL_SHAPES + EDGE_SHAPES, ids=lambda s: s.name)
def test_pack_and_dequant_bit_exact(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p)  # checks any4_pack against oracle.pack bit for bit
    W = any4.any4_dequant(d.packed, d.lut, d.scale, d.offset, shape.G)
    torch.cuda.synchronize()
    W_ref = oracle.dequant(d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    got = host_bits(W)
    bad = np.argwhere(got != W_ref)
    assert bad.size == 0, f"{shape.name}: {len(bad)} mismatches, first {bad[:3].tolist()}"


def test_pack_reports_out_of_range_codes():
    idx = np.random.default_rng(1).integers(0, 16, size=(64, 256), dtype=np.uint8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    any4.any4_pack(dev_u8(idx), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx[37, 101] = 16
    status.zero_()
    any4.any4_pack(dev_u8(idx), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_RANGE
    idx[37, 101] = 255
    status.zero_()
    any4.any4_pack(dev_u8(idx), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_RANGE


def _special_problem(rng, N, K, G):
    """Tables and group parameters that hit subnormals, signed zeros, overflow
    to infinity, exact ties of the bf16 rounding and a zero scale."""
    specials = np.array([0.0, -0.0, 1e-40, -3e-39, 2.0**-133, 3.0e38, -3.0e38, 1.0,
                         1.0 + 2.0**-8, -(1.0 + 3 * 2.0**-8), 65504.0, 1e-20, 7.5, -8.0,
                         2.0**-126, 0.1], dtype=np.float32)
    lut = torch_bf16_bits(np.stack([rng.permutation(specials) for _ in range(N)]))
    sc = rng.choice(np.array([0.0, 1.0, -1.0, 1e-38, 3.0, 2.0**-10, 1e20, 0.5], np.float32),
                    size=(N, K // G))
    of = rng.choice(np.array([0.0, -0.0, 1e-39, 2.0**-9, -1.0, 3.0e38, 1e-3, 5.0], np.float32),
                    size=(N, K // G))
    idx = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    return idx, lut, torch_bf16_bits(sc), torch_bf16_bits(of)


def test_dequant_special_values_bit_exact():
    rng = np.random.default_rng(2)
    N, K, G = 64, 512, 32
    idx, lut, sc, of = _special_problem(rng, N, K, G)
    packed_ref = oracle.pack(idx)
    W = any4.any4_dequant(dev_u8(packed_ref), dev_bf16(lut), dev_bf16(sc), dev_bf16(of), G)
    torch.cuda.synchronize()
    W_ref = oracle.dequant(packed_ref, lut, sc, of, G)
    got = host_bits(W)
    # NaN payloads are not part of the contract: compare NaN-ness there
    nan_ref = (W_ref & 0x7FFF) > 0x7F80
    nan_got = (got & 0x7FFF) > 0x7F80
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(got[~nan_ref], W_ref[~nan_ref])
    # the cases this test exists for really occur
    vals = W_ref[~nan_ref]
    assert ((vals & 0x7F80) == 0).any() and (vals != 0).any()          # subnormal results
    assert ((vals & 0x7FFF) == 0x7F80).any()                            # overflow to inf


def test_dequant_shared_table():
    """One table for the whole matrix (lut_row_stride = 0, the nf4/af4 mode)."""
    rng = np.random.default_rng(3)
    N, K, G = 300, 1024, 128
    p = workloads.make(workloads.Shape("shared", 1, K, N, G, 9101, 9601))
    table = p.lut[7].copy()
    packed_ref = oracle.pack(p.idx)
    W = any4.any4_dequant(dev_u8(packed_ref), dev_bf16(table), dev_bf16(p.scale),
                          dev_bf16(p.offset), G)
    torch.cuda.synchronize()
    W_ref = oracle.dequant(packed_ref, table, p.scale, p.offset, G, per_tensor_lut=True)
    assert np.array_equal(host_bits(W), W_ref)


def test_dequant_is_deterministic_and_respects_streams():
    p = workloads.make(workloads.LLAMA3_8B_DECODE[1])
    d = DeviceProblem(p, check_pack=False)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        W1 = any4.any4_dequant(d.packed, d.lut, d.scale, d.offset, p.shape.G)
        W2 = any4.any4_dequant(d.packed, d.lut, d.scale, d.offset, p.shape.G)
    s.synchronize()
    assert torch.equal(W1.view(torch.int16), W2.view(torch.int16))
