"""Seeded synthetic any4 workloads: shapes, seeds and input generators.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds NONE of the method's arithmetic (no packing, no dequant, no matmul): it
only draws the inputs of the path -- 4-bit codes, per-row 16-entry tables,
per-group scale and offset, activations -- as raw arrays.  bf16 inputs are
returned as uint16 bit patterns; the fp32 -> bf16 rounding of the drawn values
uses torch's own conversion (round to nearest even).

Shapes stand in for the Llama3 linear layers the any4 paper quantises
("any4: Learned 4-bit Numeric Representation for LLMs", §5: all key, query,
value, output, gate, up and down projections) and for its speed study (§5,
Fig. 3: a 1 x K activation times a K x K weight).  No model weights or
datasets are used.

Recipe (one numpy SeedSequence per weight set, spawn(4) children for idx, LUT,
scale, offset in that order; a separate SeedSequence for x):
  idx     integers(0, 16) iid uniform, uint8 [N, K]
  LUT[n]  16 draws of normal(0, 0.5) (or 0.5 * standard_t(4) for the heavy
          tailed 70B-shaped sets), sorted ascending, fp64 -> fp32 -> bf16
  scale   |normal(0, 0.01)| + 1e-3 -> bf16, [N, K/G]
  offset  normal(0, 0.002) -> bf16, [N, K/G]
  x       normal(0, 1) -> bf16, [M, K]
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


@dataclass(frozen=True)
class Shape:
    """One any4 matmul problem: y[M, N] = x[M, K] * W[N, K]^T with groups of G."""
    name: str
    M: int
    K: int
    N: int
    G: int
    weight_seed: int
    x_seed: int
    lut_dist: str = "normal"   # "normal" or "student_t4"

    @property
    def weights(self) -> int:
        return self.N * self.K

    def alg_bytes(self) -> int:
        """Bytes the path must move per call: packed codes, scale and offset,
        the tables, x and y (the dense bf16 W it avoids is not counted)."""
        return (self.N * self.K // 2 + 4 * self.N * (self.K // self.G) + 32 * self.N
                + 2 * self.M * self.K + 2 * self.M * self.N)

    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass
class Problem:
    shape: Shape
    idx: np.ndarray      # uint8 [N, K], codes 0..15
    lut: np.ndarray      # uint16 (bf16 bits) [N, 16]
    scale: np.ndarray    # uint16 (bf16 bits) [N, K/G]
    offset: np.ndarray   # uint16 (bf16 bits) [N, K/G]
    x: np.ndarray        # uint16 (bf16 bits) [M, K]
    meta: dict = field(default_factory=dict)


def draw_weights(s: Shape):
    """(idx, lut, scale, offset) for a shape, from its weight seed."""
    ss = np.random.SeedSequence(s.weight_seed)
    r_idx, r_lut, r_scale, r_off = [np.random.default_rng(c) for c in ss.spawn(4)]
    idx = r_idx.integers(0, 16, size=(s.N, s.K), dtype=np.uint8)
    if s.lut_dist == "normal":
        lut64 = r_lut.normal(0.0, 0.5, size=(s.N, 16))
    elif s.lut_dist == "student_t4":
        lut64 = 0.5 * r_lut.standard_t(4, size=(s.N, 16))
    else:
        raise ValueError(s.lut_dist)
    lut64.sort(axis=1)
    lut = _to_bf16_bits(lut64.astype(np.float32))
    ng = s.K // s.G
    scale = _to_bf16_bits((np.abs(r_scale.normal(0.0, 0.01, size=(s.N, ng))) + 1e-3)
                          .astype(np.float32))
    offset = _to_bf16_bits(r_off.normal(0.0, 0.002, size=(s.N, ng)).astype(np.float32))
    return idx, lut, scale, offset


def draw_x(s: Shape, M: int | None = None) -> np.ndarray:
    M = s.M if M is None else M
    rng = np.random.default_rng(np.random.SeedSequence(s.x_seed))
    return _to_bf16_bits(rng.normal(0.0, 1.0, size=(M, s.K)).astype(np.float32))


def make(s: Shape) -> Problem:
    idx, lut, scale, offset = draw_weights(s)
    return Problem(s, idx, lut, scale, offset, draw_x(s))


def _s(name, M, K, N, G, ws, xs, dist="normal"):
    return Shape(name, M, K, N, G, ws, xs, dist)


# The five workload families.  Seeds are fixed constants.
TINY = [_s("tiny", 1, 1024, 1024, 128, 4001, 5001)]

LLAMA3_8B_DECODE = [
    _s("8b_q", 1, 4096, 4096, 128, 4101, 5101),
    _s("8b_k", 1, 4096, 1024, 128, 4102, 5102),
    _s("8b_v", 1, 4096, 1024, 128, 4103, 5103),
    _s("8b_o", 1, 4096, 4096, 128, 4104, 5104),
    _s("8b_gate", 1, 4096, 14336, 128, 4105, 5105),
    _s("8b_up", 1, 4096, 14336, 128, 4106, 5106),
    _s("8b_down", 1, 14336, 4096, 128, 4107, 5107),
]

# Skinny sweep: the weight set (seed 4201) is shared across M; x changes with M.
SKINNY_SWEEP = [_s(f"sweep_m{M}", M, 4096, 14336, 128, 4201, 5200 + M)
                for M in (1, 2, 4, 8, 16, 32)] + [
    _s("sweep_g64_m1", 1, 4096, 14336, 64, 4202, 5290)]

LLAMA3_70B_DECODE = [
    _s(f"70b_{nm}_m{M}", M, K, N, 128, ws, 5300 + 10 * i + M, "student_t4")
    for i, (nm, K, N, ws) in enumerate([("gate", 8192, 28672, 4301),
                                        ("up", 8192, 28672, 4302),
                                        ("down", 28672, 8192, 4303)])
    for M in (1, 8)]

PREFILL = [
    _s("prefill_gate", 2048, 4096, 14336, 128, 4401, 5401),
    _s("prefill_down", 2048, 14336, 4096, 128, 4402, 5402),
]

CONFIGS = {
    "tiny": TINY,
    "llama3_8b_decode": LLAMA3_8B_DECODE,
    "skinny_sweep": SKINNY_SWEEP,
    "llama3_70b_decode": LLAMA3_70B_DECODE,
    "prefill": PREFILL,
}


def all_shapes():
    for group in CONFIGS.values():
        yield from group


# --------------------------------------------------------------------------
# Inputs of the quantiser (learning the tables): a dense bf16 weight and the
# mean absolute activation of each input column, E|x_j| (the statistic the
# paper's §4.1 Eq. 23 weights the M-step with, taken from a calibration
# prompt; here drawn, since no model or prompt is run).
#   w        normal(0, 0.02) -> bf16, [N, K] (the spread of Llama-sized
#            linear weights)
#   E|x_j|   lognormal(-0.5, 0.8), then 1 column in 200 (seeded choice)
#            multiplied by 20: the few outlier channels LLM activations have;
#            fp32 [K]
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class QuantShape:
    """One weight matrix to quantise: W[N, K] with groups of G columns."""
    name: str
    N: int
    K: int
    G: int
    seed: int


def draw_dense_weight(s: QuantShape) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence(s.seed))
    return _to_bf16_bits(rng.normal(0.0, 0.02, size=(s.N, s.K)).astype(np.float32))


def draw_abs_act_mean(s: QuantShape) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence(s.seed + 1_000_000))
    ex = rng.lognormal(-0.5, 0.8, size=s.K)
    outliers = rng.choice(s.K, size=max(1, s.K // 200), replace=False)
    ex[outliers] *= 20.0
    return ex.astype(np.float32)


# The Llama3-8B linear layers (§5) as matrices to quantise.
QUANTIZE_LLAMA3_8B = [
    QuantShape("8b_q", 4096, 4096, 128, 4501),
    QuantShape("8b_k", 1024, 4096, 128, 4502),
    QuantShape("8b_gate", 14336, 4096, 128, 4505),
    QuantShape("8b_down", 4096, 14336, 128, 4507),
]
