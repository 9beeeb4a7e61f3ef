"""Helpers for the GPU parity tests: host <-> device marshalling and the
matmul tolerance.  The expected values always come from the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4

REL_TOL = 1e-2  # |y - y_ref| <= REL_TOL * rms(y_ref[m, :]) per output row (+ one bf16 ulp)


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 CUDA tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16))
    return t.cuda().view(torch.bfloat16)


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (7 fraction bits; subnormal spacing 2^-133)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0**-126)))
    return np.power(2.0, e - 7)


def matmul_stats(y_bits: np.ndarray, y_ref: np.ndarray) -> dict:
    """Compare a bf16 result with the fp64 oracle.  Returns the worst ratio of
    the error to the allowed bound, and the literal statistic
    max_row max|y - y_ref| / rms(y_ref[row])."""
    y = bits_to_f64(y_bits)
    err = np.abs(y - y_ref)
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    bound = REL_TOL * rms + ulp_bf16(y_ref)
    return {
        "worst_vs_bound": float(np.max(err / bound)),
        "max_err_over_rms": float(np.max(np.max(err, axis=1, keepdims=True) / rms)),
        "nonfinite": int(np.count_nonzero(~np.isfinite(y))),
    }


def assert_matmul_close(y_bits: np.ndarray, y_ref: np.ndarray, what: str = ""):
    st = matmul_stats(y_bits, y_ref)
    assert st["nonfinite"] == 0, f"{what}: non-finite outputs {st}"
    assert st["worst_vs_bound"] <= 1.0, f"{what}: outside tolerance {st}"
    return st


class DeviceProblem:
    """A workload's inputs on the device, packed by any4_pack (checked)."""

    def __init__(self, p: workloads.Problem, check_pack: bool = True):
        self.p = p
        s = p.shape
        self.idx = dev_u8(p.idx)
        self.packed = any4.any4_pack(self.idx)
        self.packed_ref = oracle.pack(p.idx)
        if check_pack:
            got = self.packed.cpu().numpy()
            assert np.array_equal(got, self.packed_ref), f"{s.name}: any4_pack differs"
        self.lut = dev_bf16(p.lut)
        self.scale = dev_bf16(p.scale)
        self.offset = dev_bf16(p.offset)
        self.x = dev_bf16(p.x)
