"""The accumulation of every matmul kernel, checked on its unrounded fp32
sums (ANY4_FLAG_FP32_OUT) against the exact fp64 dequant-then-matmul:

    max |y32 - y_ref| <= 1e-3 * rms(y_ref[m, :])   for every element of row m

The bf16 results are held to the wider 1e-2 * rms + one bf16 ulp elsewhere,
because rounding y to bf16 alone can exceed 1e-2 * rms on heavy-tailed rows;
this check separates that rounding from the kernels' arithmetic: a dropped
term, a wrong scale or an accumulation with bf16 partial sums fails it,
correct fp32 sums of the bf16 weights pass with orders of magnitude to spare.
The same calls' bf16 outputs report the literal statistic
max |y - y_ref| / rms(y_ref[m, :]) per configuration in the test log.

Routes: the pair-table decode kernel (M = 2 with its workspace, M = 1 on
request), the weight-streaming shuffle kernel (M = 1), the generic decode kernel
(a group size the streaming kernels do not take), the skinny kernel
(3 <= M <= 16), and the tensor-core prefill in one pass (below M = 1024, or
with a one-pass workspace) and in two passes (M >= 1024).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, matmul_stats, host_bits

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-3


def _check_fp32(y32: np.ndarray, y_ref: np.ndarray, what: str) -> float:
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    err = np.abs(y32.astype(np.float64) - y_ref)
    assert np.isfinite(y32).all(), what
    worst = float(np.max(err / (FP32_TOL * rms)))
    assert worst <= 1.0, f"{what}: fp32 sums off by {worst:.3g} x 1e-3 rms"
    return worst


def _call(d, shape, workspace=None, path="auto", pair_table=False):
    """bf16 and fp32 outputs of one call route."""
    outs = {}
    for fp32 in (False, True):
        y = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, path=path,
                             workspace=workspace, fp32_out=fp32, pair_table=pair_table)
        torch.cuda.synchronize()
        outs[fp32] = y.cpu().numpy() if fp32 else host_bits(y)
    return outs[False], outs[True]


def _report(name, route, y16, y32, y_ref):
    worst = _check_fp32(y32, y_ref, f"{name} {route}")
    st = matmul_stats(y16, y_ref)
    print(f"{name} [{route}] fp32: worst/1e-3rms = {worst:.3g}; bf16: literal "
          f"max|y-y_ref|/rms = {st['max_err_over_rms']:.4g}, worst/bound = "
          f"{st['worst_vs_bound']:.3g}")
    assert st["worst_vs_bound"] <= 1.0, f"{name} {route} bf16 {st}"


def _empty():
    return torch.empty(0, dtype=torch.uint8, device="cuda")


M1 = (workloads.TINY + workloads.LLAMA3_8B_DECODE
      + [s for s in workloads.SKINNY_SWEEP if s.M == 1]
      + [s for s in workloads.LLAMA3_70B_DECODE if s.M == 1])


@pytest.mark.parametrize("shape", M1, ids=lambda s: s.name)
def test_fp32_m1_decode_kernels(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    y16, y32 = _call(d, shape, pair_table=True)      # pair-table kernel
    _report(shape.name, "pair table", y16, y32, y_ref)
    y16, y32 = _call(d, shape)                       # weight-streaming shuffle kernel
    _report(shape.name, "shuffle stream", y16, y32, y_ref)


SKINNY = ([s for s in workloads.SKINNY_SWEEP if 2 <= s.M <= 16]
          + [s for s in workloads.LLAMA3_70B_DECODE if s.M == 8])


@pytest.mark.parametrize("shape", SKINNY, ids=lambda s: s.name)
def test_fp32_batch_decode_kernels(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    y16, y32 = _call(d, shape)
    _report(shape.name, "pair table" if shape.M <= 2 else "skinny", y16, y32, y_ref)
    if shape.M <= 2:
        y16, y32 = _call(d, shape, workspace=_empty())
        _report(shape.name, "skinny", y16, y32, y_ref)


def test_fp32_generic_decode_kernel():
    """G = 256: neither streaming kernel takes it, the generic decode kernel runs."""
    shape = workloads.Shape("g256_m1", 1, 4096, 3000, 256, 8711, 8712)
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    y16, y32 = _call(d, shape)
    _report(shape.name, "generic decode", y16, y32, y_ref)


def test_fp32_prefill_one_pass_small():
    for shape in (workloads.Shape("pf32_ragged", 300, 1056, 520, 32, 8721, 8722),
                  [s for s in workloads.SKINNY_SWEEP if s.M == 32][0]):
        p = workloads.make(shape)
        d = DeviceProblem(p, check_pack=False)
        y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
        y16, y32 = _call(d, shape)
        _report(shape.name, "prefill one pass", y16, y32, y_ref)


@pytest.mark.parametrize("shape", workloads.PREFILL, ids=lambda s: s.name)
def test_fp32_prefill_full_shapes(shape):
    """M = 2048: two passes (full workspace) and one pass (one-pass workspace),
    checked on sampled rows of x whose whole output rows the oracle computes."""
    from tests.test_gpu_matmul_prefill import sampled_x_rows
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    rows = sampled_x_rows(shape.M, shape.weight_seed + 1)
    y_ref = oracle.any4_matmul(p.x[rows], d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    y16, y32 = _call(d, shape)
    _report(shape.name, "prefill two passes", y16[rows], y32[rows], y_ref)
    one = any4.any4_matmul_workspace_size(300, shape.N, shape.K, shape.G)
    ws = torch.empty(one, dtype=torch.uint8, device="cuda")
    y16, y32 = _call(d, shape, workspace=ws)
    _report(shape.name, "prefill one pass", y16[rows], y32[rows], y_ref)
