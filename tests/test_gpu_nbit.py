"""any3 / any2 (n-bit codes, §4.1 Eq. 9 and §5) on the GPU against the oracle:
packing, dequant and table learning, all bit for bit.  Storage: one
little-endian bit stream of codes per row."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import dev_bf16, dev_u8, host_bits
from tests.oracle_pins import random_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("N,K", [(5, 64), (37, 4096), (3, 14336)])
def test_pack_bits(bits, N, K):
    rng = np.random.default_rng(8000 + bits * 7 + N)
    idx = rng.integers(0, 1 << bits, size=(N, K), dtype=np.uint8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = any4.any4_pack_bits(dev_u8(idx), bits, dev_status=status)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), oracle.pack_bits(idx, bits))
    assert int(status.item()) == 0


@pytest.mark.parametrize("bits", [2, 3])
def test_pack_bits_flags_out_of_range_codes(bits):
    rng = np.random.default_rng(8100 + bits)
    idx = rng.integers(0, 1 << bits, size=(4, 256), dtype=np.uint8)
    idx[2, 77] = 1 << bits
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    any4.any4_pack_bits(dev_u8(idx), bits, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_RANGE


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("N,K,G,shared", [(7, 256, 32, False), (300, 4096, 128, False),
                                          (3, 14336, 14336, False), (50, 1024, 64, True)])
def test_dequant_bits(bits, N, K, G, shared):
    rng = np.random.default_rng(8200 + bits * 13 + N)
    nq = 1 << bits
    idx = rng.integers(0, nq, size=(N, K), dtype=np.uint8)
    lut = random_bf16(rng, (nq,) if shared else (N, nq), -3, 2)
    scale = random_bf16(rng, (N, K // G), -9, -5)
    offset = random_bf16(rng, (N, K // G), -10, -6)
    packed = oracle.pack_bits(idx, bits)
    W = any4.any4_dequant_bits(dev_u8(packed), dev_bf16(lut), dev_bf16(scale), dev_bf16(offset),
                               G, bits)
    torch.cuda.synchronize()
    ref = oracle.dequant_bits(packed, lut, scale, offset, G, bits, K, per_tensor_lut=shared)
    assert np.array_equal(host_bits(W), ref)


def _quant(w_bits, ex, G, bits, max_iter):
    packed, lut, scale, offset, iters = any4.any4_quantize_bits(
        dev_bf16(w_bits), torch.from_numpy(np.ascontiguousarray(ex, np.float32)).cuda(), G, bits,
        max_iter, return_iters=True)
    torch.cuda.synchronize()
    return (packed.cpu().numpy(), host_bits(lut), host_bits(scale), host_bits(offset),
            iters.cpu().numpy())


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("N,K,G,max_iter", [(40, 256, 64, 50), (17, 4096, 128, 100),
                                            (4, 14336, 128, 100), (9, 1024, 32, 0)])
def test_quantize_bits(bits, N, K, G, max_iter):
    s = workloads.QuantShape(f"nb{N}", N, K, G, 8300 + bits + N)
    w, ex = workloads.draw_dense_weight(s), workloads.draw_abs_act_mean(s)
    got = _quant(w, ex, G, bits, max_iter)
    codes, lut, scale, offset, iters = oracle.quantize_bits(w, ex, G, bits, max_iter)
    assert np.array_equal(got[2], scale) and np.array_equal(got[3], offset)
    assert np.array_equal(got[4], iters)
    assert np.array_equal(got[1], lut)
    assert np.array_equal(got[0], oracle.pack_bits(codes, bits))


@pytest.mark.parametrize("bits", [2, 3])
def test_quantize_bits_then_dequant_round_trip(bits):
    """The learned n-bit encoding dequantises (on the GPU) to the oracle's W."""
    s = workloads.QuantShape("nb_rt", 64, 2048, 128, 8400 + bits)
    w, ex = workloads.draw_dense_weight(s), workloads.draw_abs_act_mean(s)
    packed, lut, scale, offset = any4.any4_quantize_bits(dev_bf16(w), torch.from_numpy(ex).cuda(),
                                                         s.G, bits, 60)
    W = any4.any4_dequant_bits(packed, lut, scale, offset, s.G, bits)
    torch.cuda.synchronize()
    codes, lut_r, scale_r, offset_r, _ = oracle.quantize_bits(w, ex, s.G, bits, 60)
    ref = oracle.dequant_bits(oracle.pack_bits(codes, bits), lut_r, scale_r, offset_r, s.G, bits,
                              s.K)
    assert np.array_equal(host_bits(W), ref)
