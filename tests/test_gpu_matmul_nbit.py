"""any4_matmul_bits: the matmul with 2- and 3-bit codes (any2 / any3, paper
§4.1 Eq. 9: a table of 2^n values per row, §5), against the fp64 oracle
(oracle.dequant_bits then oracle.matmul).

M = 1 on the shapes the weight-streaming kernel takes reads the n-bit codes
directly; everything else runs two passes (n-bit dequant into the
workspace, then the tensor-core GEMM).  Tolerance as for any4:
|y - y_ref| <= 1e-2 * rms(y_ref[m, :]) + one bf16 ulp, and 1e-3 * rms on the
unrounded fp32 sums (ANY4_FLAG_FP32_OUT) of the fused kernel."""
import numpy as np
import pytest
import torch

import oracle
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import assert_matmul_close, dev_bf16, dev_u8, host_bits
from tests.oracle_pins import torch_bf16_bits

pytestmark = pytest.mark.gpu


def _problem(M, K, N, G, bits, seed, shared=False):
    """Workload-style generators with 2^bits table entries per row."""
    rng = np.random.default_rng(seed)
    nq = 1 << bits
    idx = rng.integers(0, nq, size=(N, K), dtype=np.uint8)
    tab = np.sort(rng.normal(0.0, 0.5, size=(nq,) if shared else (N, nq)), axis=-1)
    lut = torch_bf16_bits(tab.astype(np.float32))
    scale = torch_bf16_bits((np.abs(rng.normal(0, 0.01, size=(N, K // G))) + 1e-3)
                            .astype(np.float32))
    offset = torch_bf16_bits(rng.normal(0, 0.002, size=(N, K // G)).astype(np.float32))
    x = torch_bf16_bits(rng.normal(0, 1, size=(M, K)).astype(np.float32))
    packed = oracle.pack_bits(idx, bits)
    return x, packed, lut, scale, offset


def _run(x, packed, lut, scale, offset, G, bits, fp32=False):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = any4.any4_matmul_bits(dev_bf16(x), dev_u8(packed), dev_bf16(lut), dev_bf16(scale),
                              dev_bf16(offset), G, bits, dev_status=status, fp32_out=fp32)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y


def _ref(x, packed, lut, scale, offset, G, bits, K):
    W = oracle.dequant_bits(packed, lut, scale, offset, G, bits, K, per_tensor_lut=lut.ndim == 1)
    return oracle.matmul(x, W)


FUSED = [  # (K, N, G, shared): M = 1 shapes of the weight-streaming kernel
    (4096, 4096, 128, False),
    (4096, 14336, 128, False),   # the Llama3-8B gate / up matrix
    (2048, 333, 64, False),      # ragged rows
    (1280, 777, 32, False),      # a last slice of 256 columns
    (4096, 1500, 128, True),     # one table for the matrix
    (8192, 1024, 128, False),
]


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("K,N,G,shared", FUSED, ids=lambda v: str(v))
def test_nbit_m1_fused_decode(bits, K, N, G, shared):
    assert any4.any4_matmul_bits_workspace_size(1, N, K, G, bits) == 0  # the fused kernel
    x, packed, lut, scale, offset = _problem(1, K, N, G, bits, 13000 + bits * 101 + N + K, shared)
    y_ref = _ref(x, packed, lut, scale, offset, G, bits, K)
    y = _run(x, packed, lut, scale, offset, G, bits)
    assert_matmul_close(host_bits(y), y_ref, f"any{bits} {K}x{N}")
    y32 = _run(x, packed, lut, scale, offset, G, bits, fp32=True).cpu().numpy()
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    worst = float(np.max(np.abs(y32 - y_ref) / (1e-3 * rms)))
    assert worst <= 1.0, f"fp32 sums off by {worst:.3g} x 1e-3 rms"


@pytest.mark.parametrize("bits", [2, 3])
def test_nbit_m1_one_hot_is_exact(bits):
    """x = e_k gives column k of the dequantised weight bit for bit."""
    K, N, G = 4096, 700, 128
    _, packed, lut, scale, offset = _problem(1, K, N, G, bits, 13300 + bits)
    W = oracle.dequant_bits(packed, lut, scale, offset, G, bits, K)
    one = torch_bf16_bits(np.array([1.0], np.float32))[0]
    for k in (0, 1, 10, 11, 21, 22, 31, 32, 1023, 1024, 4095):
        x = np.zeros((1, K), np.uint16)
        x[0, k] = one
        y = _run(x, packed, lut, scale, offset, G, bits)
        assert np.array_equal(host_bits(y)[0], W[:, k]), k


TWO_PASS = [  # (M, K, N, G, shared): M > 1, or a shape the fused kernel does not take
    (1, 1056, 100, 32, False),   # K / G = 33 (and n K not a multiple of 128)
    (1, 4096, 500, 256, False),  # G = 256
    (2, 4096, 1000, 128, False),
    (8, 2048, 640, 64, True),
    (300, 1024, 520, 32, False),
]


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("M,K,N,G,shared", TWO_PASS, ids=lambda v: str(v))
def test_nbit_two_pass(bits, M, K, N, G, shared):
    assert any4.any4_matmul_bits_workspace_size(M, N, K, G, bits) > 0
    x, packed, lut, scale, offset = _problem(M, K, N, G, bits, 13500 + bits * 7 + M + N, shared)
    y = _run(x, packed, lut, scale, offset, G, bits)
    assert_matmul_close(host_bits(y), _ref(x, packed, lut, scale, offset, G, bits, K),
                        f"any{bits} M={M}")


@pytest.mark.parametrize("bits", [2, 3])
def test_nbit_prefill_m2048_sampled_rows(bits):
    """The Llama3-8B gate shape at M = 2048 (two passes), checked on whole
    output rows for a sample of x rows."""
    M, K, N, G = 2048, 4096, 14336, 128
    x, packed, lut, scale, offset = _problem(M, K, N, G, bits, 13700 + bits)
    y = host_bits(_run(x, packed, lut, scale, offset, G, bits))
    rows = np.array([0, 1, 255, 256, 1023, 2047])
    y_ref = _ref(x[rows], packed, lut, scale, offset, G, bits, K)
    assert_matmul_close(y[rows], y_ref, f"any{bits} prefill")


def test_nbit_four_bits_is_any4_matmul():
    K, N, G = 4096, 512, 128
    x, packed, lut, scale, offset = _problem(1, K, N, G, 4, 13900)
    a = _run(x, packed, lut, scale, offset, G, 4)
    b = any4.any4_matmul(dev_bf16(x), dev_u8(packed), dev_bf16(lut), dev_bf16(scale),
                         dev_bf16(offset), G)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
