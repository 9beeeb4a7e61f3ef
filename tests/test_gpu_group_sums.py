"""any4_group_sums on the GPU against the oracle's fp64 group sums.

Bound: any order of the G fp32 additions of one group lies within
gamma_{G-1} * sum |x| of the exact sum (gamma_n = n u / (1 - n u),
u = 2^-24; Higham, Accuracy and Stability of Numerical Algorithms, §4.2);
the oracle's fp64 sums are exact to far below that, so each result must lie
within the bound of the oracle's value.  The calls are also bit-identical
from run to run (fixed summation order)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import dev_bf16

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _bound(x_bits: np.ndarray, G: int) -> np.ndarray:
    M, K = x_bits.shape
    ax = np.abs(oracle.bf16_to_f32(x_bits).astype(np.float64)).reshape(M, K // G, G).sum(axis=2)
    n = G - 1
    return n * U / (1 - n * U) * ax + 1e-300


def _x(M, K, seed, heavy=False):
    rng = np.random.default_rng(seed)
    v = rng.standard_t(4, size=(M, K)) if heavy else rng.normal(0.0, 1.0, size=(M, K))
    t = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


CASES = [  # (M, K, G): several units per row, ragged last units, wide groups
    (1, 32, 32),
    (1, 1024, 128),
    (3, 1056, 32),       # 33 groups: one full unit of 64 groups is not reached
    (5, 4096, 64),
    (2, 6144, 96),       # 21 groups per unit, the row ends mid-unit
    (4, 14336, 128),
    (2, 3072, 1536),     # one group per unit, 192 chunks in one pass
    (3, 8192, 4096),     # a group spans two passes
    (2, 10240, 10240),   # one group per row, five passes
    (7, 2112, 2112),     # one group per row, a ragged second pass
]


@pytest.mark.parametrize("M,K,G", CASES, ids=lambda v: str(v))
def test_group_sums_match_oracle(M, K, G):
    for heavy in (False, True):
        x = _x(M, K, 9100 + M * 7 + K + G, heavy)
        ref = oracle.group_sums(x, G)
        got = any4.any4_group_sums(dev_bf16(x), G)
        torch.cuda.synchronize()
        got = got.cpu().numpy().astype(np.float64)
        assert got.shape == (M, K // G)
        err = np.abs(got - ref)
        bound = _bound(x, G)
        assert (err <= bound).all(), f"worst {float(np.max(err / bound)):.3g} x bound"


@pytest.mark.parametrize("shape", workloads.PREFILL + workloads.LLAMA3_8B_DECODE[:1],
                         ids=lambda s: s.name)
def test_group_sums_workload_shapes(shape):
    """The activations of the prefill and decode workloads at full size."""
    x = workloads.draw_x(shape)
    ref = oracle.group_sums(x, shape.G)
    got = any4.any4_group_sums(dev_bf16(x), shape.G)
    torch.cuda.synchronize()
    again = any4.any4_group_sums(dev_bf16(x), shape.G)
    torch.cuda.synchronize()
    assert torch.equal(got, again), "not deterministic"
    err = np.abs(got.cpu().numpy().astype(np.float64) - ref)
    assert (err <= _bound(x, shape.G)).all()


def test_group_sums_exact_cases():
    """Inputs whose fp32 sums are exact: small integers, and a constant row."""
    M, K, G = 3, 4096, 128
    rng = np.random.default_rng(9201)
    ints = rng.integers(-8, 9, size=(M, K)).astype(np.float32)
    x = torch.from_numpy(ints).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = any4.any4_group_sums(dev_bf16(x), G).cpu().numpy()
    assert np.array_equal(got.astype(np.float64), oracle.group_sums(x, G))
    xc = np.full((1, K), x[0, 0], dtype=np.uint16)
    got = any4.any4_group_sums(dev_bf16(xc), G).cpu().numpy()
    assert (got == G * float(ints[0, 0])).all()


def test_group_sums_writes_only_its_output():
    M, K, G = 2, 2048, 64
    x = _x(M, K, 9301)
    pad = 64
    buf = torch.full((pad + M * (K // G) + pad,), -7.0, dtype=torch.float32, device="cuda")
    out = buf[pad:pad + M * (K // G)].view(M, K // G)
    any4.any4_group_sums(dev_bf16(x), G, xsum=out)
    torch.cuda.synchronize()
    assert (buf[:pad] == -7.0).all() and (buf[-pad:] == -7.0).all()
    assert np.abs(out.cpu().numpy() - oracle.group_sums(x, G)).max() <= _bound(x, G).max()


def test_group_sums_rejects_bad_shapes():
    x = dev_bf16(_x(2, 1024, 9401))
    with pytest.raises(ValueError):
        any4.any4_group_sums(x, 100)           # K % G != 0
    with pytest.raises(any4.Any4Error):
        any4.any4_group_sums(x, 16)            # G % 32 != 0
    lib = any4.library()
    assert lib.any4_group_sums(x.data_ptr(), None, 2, 1024, 128, None) == any4.ANY4_ERR_NULL
    out = torch.empty(2 * 8 + 1, dtype=torch.float32, device="cuda")
    assert (lib.any4_group_sums(x.data_ptr(), out.data_ptr() + 4, 2, 1024, 128, None)
            == any4.ANY4_ERR_ALIGN)
