"""Pins for the any4 oracle: checks against facts fixed by the pages and by
mathematics, never against the oracle itself.

Every pin is a plain function that raises AssertionError on failure, so the
same pins run against the real oracle (tests/test_oracle_pins.py) and against
copies of the oracle source with a planted mistake (tests/test_oracle_mutants.py,
which requires that every planted mistake fails at least one pin).

Kinds of pin used (paper: "any4: Learned 4-bit Numeric Representation for
LLMs", arXiv 2507.04610):
  * worked examples the pages print (storage accounting, §2.4.1), as fixtures
    under tests/golden/;
  * values fixed by the IEEE 754 definition of round-to-nearest-even, and a
    library routine (torch's fp32 -> bf16 conversion) on a million inputs;
  * special cases that reduce to a textbook format: the LUT {-8..7} reproduces
    grouped asymmetric int4 (§2.1, §2.5.1 Eq. 1-2, §2.5.2 Eq. 4 and dequant);
    one shared table reproduces the nf4/af4 mode (§2.4.1);
  * exact rational arithmetic (Python fractions) for the fused multiply-add;
  * invariants (LUT permutation, constant codes, zero scale, one-hot and
    identity activations, linearity with exactly representable inputs);
  * brute force with an independent summation (math.fsum, exact) on tiny
    shapes, within the fp64 error bound of an ascending-k sum.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# helpers that use only torch / numpy / fractions, never the oracle
# --------------------------------------------------------------------------

def torch_bf16_bits(f32: np.ndarray) -> np.ndarray:
    """torch's own fp32 -> bf16 conversion (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def torch_bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def exact_fma_then_bf16(a: float, b: float, c: float) -> int:
    """bf16 bits of RNE_bf16(RNE_f32(a*b + c)) with a*b + c formed exactly.

    The exact value is a Fraction; fp64 -> fp32 rounding is done by numpy on a
    value that is checked to be exact in fp64 first, fp32 -> bf16 by torch."""
    exact = Fraction(a) * Fraction(b) + Fraction(c)
    as64 = float(exact)
    assert Fraction(as64) == exact, "test input not exact in fp64"
    f32 = np.array([as64], dtype=np.float64).astype(np.float32)
    return int(torch_bf16_bits(f32)[0])


def read_golden(name: str):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line)
    return rows


def random_bf16(rng, shape, lo_exp=-12, hi_exp=2):
    """bf16 bit patterns of random sign, exponent in [lo_exp, hi_exp), 7-bit fraction."""
    sign = rng.integers(0, 2, size=shape)
    e = rng.integers(lo_exp, hi_exp, size=shape)
    frac = rng.integers(0, 128, size=shape)
    vals = (1 + frac / 128.0) * np.power(2.0, e) * np.where(sign, -1.0, 1.0)
    return torch_bf16_bits(vals.astype(np.float32))


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------

def pin_bf16_rne_definition_cases():
    for row in read_golden("bf16_rne_cases.txt"):
        src, dst = [s.strip() for s in row.split("->", 1)]
        dst = dst.split()[0]
        f = np.array([int(src, 16)], dtype=np.uint32).view(np.float32)
        got = int(oracle.bf16_rne(f)[0])
        assert got == int(dst, 16), f"bf16_rne({src}) = {got:04x}, expected {dst}"


def pin_bf16_rne_vs_torch():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2**32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    # force many exact ties and near-ties
    bits[:200_000] = (bits[:200_000] & 0xFFFF0000) | 0x8000
    bits[200_000:300_000] = (bits[200_000:300_000] & 0xFFFF0000) | 0x7FFF
    f = bits.view(np.float32)
    finite = np.isfinite(f) | np.isinf(f)
    f = f[finite & ~np.isnan(f)]
    ours = oracle.bf16_rne(f)
    ref = torch_bf16_bits(f)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first f32 bits {f[bad[:3]].view(np.uint32)}"
    nan = np.array([np.nan, -np.nan], dtype=np.float32)
    assert np.isnan(oracle.bf16_to_f32(oracle.bf16_rne(nan))).all()


def pin_bf16_widen_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        ours = oracle.bf16_to_f32(bits).astype(np.float64)
    ref = torch_bf16_to_f64(bits)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours[~both_nan], ref[~both_nan])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def pin_pack_worked_examples():
    for row in read_golden("pack_example.txt"):
        codes, bytes_ = [s.strip() for s in row.split("->")]
        idx = np.array([[int(c) for c in codes.split()]], dtype=np.uint8)
        want = np.array([[int(b, 16) for b in bytes_.split()]], dtype=np.uint8)
        got = oracle.pack(idx)
        assert np.array_equal(got, want), f"pack({codes}) = {got}, expected {want}"


def pin_pack_roundtrip_exhaustive():
    # every byte value unpacks to two codes that pack back to the same byte
    all_bytes = np.arange(256, dtype=np.uint8).reshape(1, 256)
    codes = oracle.unpack(all_bytes)
    assert codes.max() <= 15
    assert np.array_equal(oracle.pack(codes), all_bytes)
    # every ordered pair of codes packs to a distinct byte and round-trips
    a, b = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    pairs = np.stack([a.ravel(), b.ravel()], axis=1).astype(np.uint8).reshape(1, 512)
    packed = oracle.pack(pairs)
    assert len(set(packed.ravel().tolist())) == 256
    assert np.array_equal(oracle.unpack(packed), pairs)


def pin_pack_rejects_bad_codes():
    try:
        oracle.pack(np.array([[3, 16]], dtype=np.uint8))
    except ValueError:
        return
    raise AssertionError("a code of 16 was accepted")


def pin_pack_multirow_layout():
    # row-major [N][K/2]: row n's bytes depend only on row n's codes
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 16, size=(5, 64), dtype=np.uint8)
    full = oracle.pack(idx)
    for n in range(5):
        assert np.array_equal(full[n], oracle.pack(idx[n:n + 1])[0])
    assert full.shape == (5, 32)


# --------------------------------------------------------------------------
# storage accounting (worked example printed in §2.4.1)
# --------------------------------------------------------------------------

def pin_storage_bits_worked_example():
    for row in read_golden("storage_bits.txt"):
        K, G, lb, gb, bits = row.split()
        got = oracle.bits_per_weight(int(K), int(G), int(lb), int(gb))
        assert abs(got - float(bits)) < 1e-12, f"{row}: got {got}"


def pin_storage_bits_match_array_sizes():
    # the byte count of an actual any4 weight set matches the accounting
    N, K, G = 8, 4096, 128
    idx = np.zeros((N, K), dtype=np.uint8)
    packed = oracle.pack(idx)
    lut = np.zeros((N, 16), dtype=np.uint16)
    scale = np.zeros((N, K // G), dtype=np.uint16)
    offset = np.zeros((N, K // G), dtype=np.uint16)
    total_bits = 8 * (packed.nbytes + lut.nbytes + scale.nbytes + offset.nbytes)
    assert total_bits / (N * K) == oracle.bits_per_weight(K, G)


# --------------------------------------------------------------------------
# dequant
# --------------------------------------------------------------------------

def pin_dequant_one_exact_fma():
    """The fused multiply-add rounds once: compare with exact rational arithmetic."""
    rng = np.random.default_rng(5)
    a = random_bf16(rng, 4000)
    b = random_bf16(rng, 4000)
    c = random_bf16(rng, 4000)
    av, bv, cv = torch_bf16_to_f64(a), torch_bf16_to_f64(b), torch_bf16_to_f64(c)
    for i in range(4000):
        want = exact_fma_then_bf16(av[i], bv[i], cv[i])
        got = oracle.dequant_one(int(a[i]), int(b[i]), int(c[i]))
        assert got == want, f"case {i}: {av[i]}*{bv[i]}+{cv[i]}: {got:04x} vs {want:04x}"


def pin_dequant_single_rounding_of_fma():
    """A case where fmaf and a separately rounded multiply then add differ:
    (1 + 2^-7) * (1 + 2^-7) = 1 + 2^-6 + 2^-14; adding -(1 + 2^-6) leaves
    2^-14 exactly with one rounding.  A mul-then-add in fp32 would also keep
    it, so use a product that does not fit fp32: choose values whose product
    has more than 24 significant bits is impossible for bf16 inputs (8 x 8
    bits), hence the fp32 fmaf and an exact evaluation always agree before
    the final bf16 rounding.  Check the zero-offset and zero-scale corners."""
    one = int(torch_bf16_bits(np.array([1.0], np.float32))[0])
    zero = 0
    # LUT * 1 + 0 is the LUT value itself
    for v in random_bf16(np.random.default_rng(6), 500):
        assert oracle.dequant_one(int(v), one, zero) == int(v)
        # LUT * 0 + offset is the offset itself (nonzero offset)
        assert oracle.dequant_one(one, zero, int(v)) == int(v)


def _int4_asymmetric_groups(w, G):
    """Eq. 2 (asymmetric) scale per group: alpha = (max - min) / (Qmax - Qmin),
    beta = min, with Qmin = 0 and Qmax = 15 for the 16 codes; Eq. 1 then Eq. 4
    (round to nearest) give codes 0..15."""
    N, K = w.shape
    wg = w.reshape(N, K // G, G)
    beta = wg.min(axis=2)
    alpha = (wg.max(axis=2) - beta) / 15.0
    q = np.rint((wg - beta[..., None]) / alpha[..., None]).clip(0, 15).astype(np.uint8)
    return q.reshape(N, K), alpha, beta


def pin_dequant_int4_special_case():
    """A LUT of {-8..7} with offset' = beta + 8*alpha reproduces grouped
    asymmetric int4 dequant alpha*q + beta (§2.1 int4 range -8..7, §2.5.2),
    bit for bit, where q = code in 0..15 and the int4 value is q - 8."""
    rng = np.random.default_rng(7)
    N, K, G = 16, 512, 128
    w = rng.normal(0, 0.02, size=(N, K))
    q, alpha, beta = _int4_asymmetric_groups(w, G)
    a_b = torch_bf16_bits(alpha.astype(np.float32))
    off_b = torch_bf16_bits((beta + 8 * alpha).astype(np.float32))
    lut_int4 = torch_bf16_bits(np.arange(-8, 8, dtype=np.float32))
    lut = np.tile(lut_int4, (N, 1))
    W = oracle.dequant(oracle.pack(q), lut, a_b, off_b, G)
    a_v = torch_bf16_to_f64(a_b)
    o_v = torch_bf16_to_f64(off_b)
    for n in range(N):
        for k in range(0, K, 7):
            g = k // G
            want = exact_fma_then_bf16(float(int(q[n, k]) - 8), a_v[n, g], o_v[n, g])
            assert W[n, k] == want, (n, k)
    # reconstruction error of the int4 round trip is at most alpha/2 plus the
    # bf16 roundings of alpha, offset and the result
    Wv = torch_bf16_to_f64(W)
    err = np.abs(Wv - w).reshape(N, K // G, G).max(axis=2)
    bound = alpha / 2 + 16 * np.abs(alpha) * 2.0**-8 + np.abs(beta) * 2.0**-7 + 0.05 * 2.0**-7
    assert (err <= bound).all(), float((err / bound).max())


def pin_dequant_shared_table_mode():
    """One 16-entry table for the whole matrix (the nf4/af4 mode, §2.4.1)
    equals the per-row mode with that table repeated on every row, and each
    weight equals T[code]*scale + offset rounded once to fp32 then to bf16.
    The table here is built like nf4 (asymmetric, an exact zero, in [-1, 1]);
    the published nf4 constants are not on the pages."""
    rng = np.random.default_rng(8)
    N, K, G = 12, 256, 64
    from statistics import NormalDist
    nd = NormalDist()
    neg = [nd.inv_cdf(p) for p in np.linspace(0.02, 0.5, 8)[:-1]]
    pos = [nd.inv_cdf(p) for p in np.linspace(0.5, 0.98, 9)[1:]]
    table = np.array(neg + [0.0] + pos)
    table = table / np.abs(table).max()
    T = torch_bf16_bits(table.astype(np.float32))
    assert T.size == 16 and 0 in T.tolist()
    idx = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    packed = oracle.pack(idx)
    scale = random_bf16(rng, (N, K // G), -8, -4)
    offset = random_bf16(rng, (N, K // G), -10, -7)
    W_shared = oracle.dequant(packed, T, scale, offset, G, per_tensor_lut=True)
    W_rows = oracle.dequant(packed, np.tile(T, (N, 1)), scale, offset, G)
    assert np.array_equal(W_shared, W_rows)
    Tv, sv, ov = torch_bf16_to_f64(T), torch_bf16_to_f64(scale), torch_bf16_to_f64(offset)
    for n in range(N):
        for k in range(0, K, 5):
            want = exact_fma_then_bf16(Tv[idx[n, k]], sv[n, k // G], ov[n, k // G])
            assert W_shared[n, k] == want


def pin_dequant_invariants():
    rng = np.random.default_rng(9)
    N, K, G = 6, 384, 128
    idx = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    lut = random_bf16(rng, (N, 16), -3, 1)
    scale = random_bf16(rng, (N, K // G), -8, -5)
    offset = random_bf16(rng, (N, K // G), -10, -8)
    W = oracle.dequant(oracle.pack(idx), lut, scale, offset, G)
    # permuting each row's table and relabelling its codes leaves W unchanged
    for trial in range(3):
        perm = np.stack([rng.permutation(16) for _ in range(N)])  # slot j holds old entry perm[j]
        inv = np.argsort(perm, axis=1)                              # old entry c sits at slot inv[c]
        lut_p = np.take_along_axis(lut, perm, axis=1)
        idx_p = np.take_along_axis(inv, idx.astype(np.int64), axis=1).astype(np.uint8)
        assert np.array_equal(oracle.dequant(oracle.pack(idx_p), lut_p, scale, offset, G), W)
    # constant codes give LUT[c] * scale + offset for every column of a group
    for c in (0, 5, 15):
        Wc = oracle.dequant(oracle.pack(np.full((N, K), c, np.uint8)), lut, scale, offset, G)
        for n in range(N):
            for g in range(K // G):
                blk = Wc[n, g * G:(g + 1) * G]
                assert (blk == blk[0]).all()
                assert blk[0] == oracle.dequant_one(int(lut[n, c]), int(scale[n, g]),
                                                    int(offset[n, g]))
    # zero scale gives the offset everywhere
    Wz = oracle.dequant(oracle.pack(idx), lut, np.zeros_like(scale), offset, G)
    assert np.array_equal(Wz, np.repeat(offset, G, axis=1))
    # each group uses its own parameters: change one group's scale only
    s2 = scale.copy()
    s2[2, 1] = torch_bf16_bits(np.array([7.0], np.float32))[0]
    W2 = oracle.dequant(oracle.pack(idx), lut, s2, offset, G)
    diff = np.argwhere(W2 != W)
    assert diff.size and (diff[:, 0] == 2).all()
    assert (diff[:, 1] >= G).all() and (diff[:, 1] < 2 * G).all()


# --------------------------------------------------------------------------
# matmul
# --------------------------------------------------------------------------

def _small_problem(rng, M, N, K, G):
    idx = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    lut = torch_bf16_bits(np.sort(rng.normal(0, 0.5, size=(N, 16)), axis=1).astype(np.float32))
    scale = torch_bf16_bits((np.abs(rng.normal(0, 0.01, size=(N, K // G))) + 1e-3)
                            .astype(np.float32))
    offset = torch_bf16_bits(rng.normal(0, 0.002, size=(N, K // G)).astype(np.float32))
    x = torch_bf16_bits(rng.normal(0, 1, size=(M, K)).astype(np.float32))
    return idx, lut, scale, offset, x


def pin_matmul_one_hot():
    rng = np.random.default_rng(12)
    N, K, G = 24, 256, 64
    idx, lut, scale, offset, _ = _small_problem(rng, 1, N, K, G)
    W = oracle.dequant(oracle.pack(idx), lut, scale, offset, G)
    Wv = torch_bf16_to_f64(W)
    one = torch_bf16_bits(np.array([1.0], np.float32))[0]
    for k in (0, 1, 63, 64, 200, 255):
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = one
        y = oracle.matmul(x, W)
        assert np.array_equal(y[0], Wv[:, k]), k


def pin_matmul_identity():
    rng = np.random.default_rng(13)
    N, K, G = 40, 128, 32
    idx, lut, scale, offset, _ = _small_problem(rng, 1, N, K, G)
    W = oracle.dequant(oracle.pack(idx), lut, scale, offset, G)
    eye = torch_bf16_bits(np.eye(K, dtype=np.float32))
    y = oracle.matmul(eye, W)
    assert np.array_equal(y, torch_bf16_to_f64(W).T)
    assert np.array_equal(oracle.any4_matmul(eye, oracle.pack(idx), lut, scale, offset, G),
                          torch_bf16_to_f64(W).T)


def pin_matmul_brute_force():
    """Tiny shapes against an exact sum (math.fsum) of the exact products;
    an ascending fp64 sum of K terms is within K * 2^-53 * sum|terms|."""
    rng = np.random.default_rng(14)
    for (M, N, K, G) in [(1, 8, 64, 32), (3, 16, 128, 64), (4, 64, 256, 128)]:
        idx, lut, scale, offset, x = _small_problem(rng, M, N, K, G)
        W = oracle.dequant(oracle.pack(idx), lut, scale, offset, G)
        y = oracle.matmul(x, W)
        xv, Wv = torch_bf16_to_f64(x), torch_bf16_to_f64(W)
        for m in range(M):
            for n in range(N):
                terms = xv[m] * Wv[n]           # exact: 8-bit x 8-bit significands
                exact = math.fsum(terms.tolist())
                bound = K * 2.0**-53 * float(np.abs(terms).sum()) + 1e-300
                assert abs(y[m, n] - exact) <= bound, (M, N, K, m, n)
        # dequant-then-matmul orientation: y = x W^T, not x W
        assert y.shape == (M, N)


def pin_matmul_zero_and_linearity():
    rng = np.random.default_rng(15)
    M, N, K, G = 3, 20, 256, 128
    idx, lut, scale, offset, _ = _small_problem(rng, M, N, K, G)
    W = oracle.dequant(oracle.pack(idx), lut, scale, offset, G)
    assert (oracle.matmul(np.zeros((M, K), np.uint16), W) == 0).all()
    # small integers are exact in bf16 and the sums below are exact in fp64
    x1 = rng.integers(-2, 3, size=(M, K)).astype(np.float32)
    x2 = rng.integers(-2, 3, size=(M, K)).astype(np.float32)
    y1 = oracle.matmul(torch_bf16_bits(x1), W)
    y2 = oracle.matmul(torch_bf16_bits(x2), W)
    y12 = oracle.matmul(torch_bf16_bits(x1 + x2), W)
    assert np.array_equal(y12, y1 + y2)
    y3 = oracle.matmul(torch_bf16_bits(3 * x1), W)
    assert np.array_equal(y3, 3 * y1)


def pin_matmul_rows_equals_full():
    rng = np.random.default_rng(16)
    M, N, K, G = 2, 33, 192, 64
    idx, lut, scale, offset, x = _small_problem(rng, M, N, K, G)
    packed = oracle.pack(idx)
    full = oracle.any4_matmul(x, packed, lut, scale, offset, G)
    rows = np.array([0, 5, 32, 7], dtype=np.int64)
    part = oracle.matmul_rows(x, packed, lut, scale, offset, G, rows)
    assert np.array_equal(part, full[:, rows])


def pin_group_sums_brute_force_exact():
    """Tiny shapes: every group sum against the exact rational sum of the
    group's bf16 values (Fractions).  Exponents span [-20, 12): 32 binades
    plus 8 significand bits plus 7 bits of carries for 128 terms fit in the
    53 bits of fp64, so its sum is exact and the values must be identical
    (an fp32 accumulator, 24 bits, is not)."""
    rng = np.random.default_rng(17)
    for (M, K, G) in [(1, 64, 32), (3, 256, 64), (2, 384, 128)]:
        x = random_bf16(rng, (M, K), lo_exp=-20, hi_exp=12)
        xs = oracle.group_sums(x, G)
        xv = torch_bf16_to_f64(x)
        assert xs.shape == (M, K // G)
        for m in range(M):
            for g in range(K // G):
                exact = sum((Fraction(float(v)) for v in xv[m, g * G:(g + 1) * G]), Fraction(0))
                assert Fraction(float(xs[m, g])) == exact, (M, K, G, m, g)


def pin_group_sums_constant_and_one_hot():
    """Constant rows sum to G * c; a single nonzero column lands in its own
    group k // G and nowhere else (a shifted group boundary fails this)."""
    M, K, G = 2, 512, 128
    c = torch_bf16_bits(np.array([0.75], np.float32))[0]
    xs = oracle.group_sums(np.full((M, K), c, dtype=np.uint16), G)
    assert (xs == G * 0.75).all()
    one = torch_bf16_bits(np.array([1.0], np.float32))[0]
    for k in (0, 1, 127, 128, 129, 383, 384, 511):
        x = np.zeros((M, K), dtype=np.uint16)
        x[1, k] = one
        xs = oracle.group_sums(x, G)
        want = np.zeros((M, K // G))
        want[1, k // G] = 1.0
        assert np.array_equal(xs, want), k


def pin_group_sums_expand_eq8_with_group_affine_weights():
    """The reason the sums exist: with unrounded group-affine weights
    W = LUT[c] * alpha + beta, x W^T equals
    sum_g alpha_g * (sum_{k in g} x * LUT[c]) + beta_g * xsum_g (exact algebra;
    both sides in fp64 with numpy, equal to within rounding)."""
    rng = np.random.default_rng(18)
    M, N, K, G = 3, 10, 256, 64
    idx, lut, scale, offset, x = _small_problem(rng, M, N, K, G)
    xv = torch_bf16_to_f64(x)
    T = torch_bf16_to_f64(lut)
    a = np.repeat(torch_bf16_to_f64(scale), G, axis=1)
    b = np.repeat(torch_bf16_to_f64(offset), G, axis=1)
    Wq = np.take_along_axis(T, idx.astype(np.int64), axis=1)        # LUT[n][c]
    direct = xv @ (Wq * a + b).T
    xs = oracle.group_sums(x, G)                                     # [M, K/G]
    lut_part = np.einsum("mgk,ngk->mng", xv.reshape(M, K // G, G), Wq.reshape(N, K // G, G))
    expanded = (np.einsum("mng,ng->mn", lut_part, torch_bf16_to_f64(scale))
                + xs @ torch_bf16_to_f64(offset).T)
    assert np.allclose(expanded, direct, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# learning the table: §2.5.1 Eq. 1-2 scaling, §4.1 E-step (Eq. 18) and M-step
# (Eq. 23), Appendix A.1 Alg. 1 (k-means per row, sample weight alpha * E|x|)
# --------------------------------------------------------------------------

def _quantile_init(xs, nq=16):
    """The initial table read from the pages: entry q is the element at
    position floor(q (K - 1) / (nq - 1)) of the row sorted by numpy."""
    s = np.sort(np.asarray(xs, dtype=np.float64))
    return s[[(q * (xs.size - 1)) // (nq - 1) for q in range(nq)]]


def _nearest(xs, table):
    """Eq. 18 by brute force: numpy's argmin returns the first (lowest) index on a tie."""
    return np.argmin(np.abs(xs[:, None] - table[None, :]), axis=1).astype(np.uint8)


def _numpy_scale(w_bits, G, levels=15):
    """Eq. 1-2 with numpy fp32 (each operation correctly rounded) and torch's bf16 rounding."""
    N, K = w_bits.shape
    wf = torch_bf16_to_f64(w_bits).astype(np.float32).reshape(N, K // G, G) + np.float32(0)
    mn, mx = wf.min(axis=2), wf.max(axis=2)
    return torch_bf16_bits((mx - mn) / np.float32(levels)), torch_bf16_bits(mn)


def _sklearn_kmeans(xs, u, max_iter=500, nq=16):
    """scikit-learn's weighted Lloyd k-means (the library Appendix C.2 names),
    started from the quantile table."""
    from sklearn.cluster import KMeans
    km = KMeans(n_clusters=nq, init=_quantile_init(xs, nq)[:, None], n_init=1,
                max_iter=max_iter, tol=0.0, algorithm="lloyd").fit(xs[:, None], sample_weight=u)
    return km.cluster_centers_[:, 0], km.labels_.astype(np.uint8)


def _levels_problem(rng, N, K, G, levels):
    """Groups holding exactly beta_g + alpha_g * levels (each level
    G / len(levels) times, shuffled), alpha_g a power of two: every value is
    exact in bf16."""
    w = np.empty((N, K), dtype=np.float64)
    for n in range(N):
        for g in range(K // G):
            alpha = 2.0 ** -(5 + (n + g) % 3)
            beta = -(1 + (n * 7 + g) % 5) / 32.0
            vals = beta + alpha * np.repeat(levels, G // len(levels))
            w[n, g * G:(g + 1) * G] = rng.permutation(vals)
    bits = torch_bf16_bits(w.astype(np.float32))
    assert np.array_equal(torch_bf16_to_f64(bits), w), "levels not exact in bf16"
    return bits


def pin_group_scale_closed_form():
    rng = np.random.default_rng(101)
    N, K, G = 6, 256, 64
    w = random_bf16(rng, (N, K), lo_exp=-9, hi_exp=-3)
    scale, offset = oracle.group_scale(w, G)
    s_ref, o_ref = _numpy_scale(w, G)
    assert np.array_equal(scale, s_ref) and np.array_equal(offset, o_ref)
    # a constant group has scale 0; a group of zeros signed either way has offset +0
    w2 = w.copy()
    w2[0, :G] = w2[0, 5]
    w2[1, G:2 * G] = 0x8000
    w2[1, G + 3] = 0x0000
    scale2, offset2 = oracle.group_scale(w2, G)
    assert scale2[0, 0] == 0 and offset2[0, 0] == w2[0, 5]
    assert scale2[1, 1] == 0 and offset2[1, 1] == 0x0000


def pin_scaled_weights_range_and_reconstruction():
    rng = np.random.default_rng(102)
    N, K, G = 5, 384, 128
    w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    scale, offset = oracle.group_scale(w, G)
    ws = oracle.scaled_weights(w, scale, offset, G)
    a = torch_bf16_to_f64(scale).repeat(G, axis=1)
    b = torch_bf16_to_f64(offset).repeat(G, axis=1)
    wf = torch_bf16_to_f64(w)
    g = ws.reshape(N, K // G, G)
    assert np.all(g.min(axis=2) == 0.0)               # the minimum maps to 0 exactly
    assert np.allclose(g.max(axis=2), 15.0, rtol=2 ** -7, atol=0)
    assert np.all(np.abs(a * ws + b - wf) <= 2 ** -50 * (np.abs(wf) + np.abs(b)))
    # groups on the int4 grid: w = beta + alpha * k gives w_S = k exactly
    levels = np.arange(16, dtype=np.float64)
    w3 = _levels_problem(rng, 2, 256, 64, levels)
    s3, o3 = oracle.group_scale(w3, 64)
    ws3 = oracle.scaled_weights(w3, s3, o3, 64)
    assert np.array_equal(ws3, np.round(ws3)) and ws3.min() == 0 and ws3.max() == 15


def pin_kmeans_initial_table_and_nearest():
    rng = np.random.default_rng(103)
    xs = rng.uniform(0, 15, 300)
    c, code, it = oracle.kmeans_row(xs, np.ones(300), 0)
    assert it == 0
    assert np.array_equal(c, _quantile_init(xs))
    assert np.array_equal(code, _nearest(xs, c))


def pin_kmeans_ties_go_to_lowest_entry():
    # 16 levels 0..15 (8 copies each) and the 15 midpoints between them: the
    # quantile table is exactly 0..15 and every midpoint is a tie.
    mids = np.arange(15) + 0.5
    xs = np.sort(np.concatenate([np.repeat(np.arange(16.0), 8), mids]))
    c, code, _ = oracle.kmeans_row(xs, np.ones(xs.size), 0)
    assert np.array_equal(c, np.arange(16.0))
    for m in range(15):
        assert code[np.searchsorted(xs, m + 0.5)] == m
    assert np.array_equal(code, _nearest(xs, c))


def _pairs_problem():
    """Cluster q holds 10q (weight 3) and 10q + 1 (weight 1); entry 15 starts at 151."""
    xs = np.array([v for q in range(16) for v in (10.0 * q, 10.0 * q + 1)])
    u = np.tile([3.0, 1.0], 16)
    return xs, u


def pin_kmeans_weighted_mean_closed_form():
    xs, u = _pairs_problem()
    c, code, it = oracle.kmeans_row(xs, u, 20)
    assert np.array_equal(code, np.repeat(np.arange(16), 2))
    assert np.array_equal(c, 10.0 * np.arange(16) + 0.25)   # (3 * 10q + (10q + 1)) / 4
    assert it == 1


def pin_kmeans_zero_weight_cluster_keeps_entry():
    xs, u = _pairs_problem()
    u[10:12] = 0.0                                           # cluster 5 weighs nothing
    c, _, _ = oracle.kmeans_row(xs, u, 20)
    init = _quantile_init(xs)
    assert c[5] == init[5] == 50.0
    assert np.array_equal(np.delete(c, 5), np.delete(10.0 * np.arange(16) + 0.25, 5))


def pin_kmeans_matches_scikit_learn():
    rng = np.random.default_rng(104)
    for K in (400, 1024):
        xs = np.clip(rng.normal(7.5, 2.5, K), 0, 15)
        u = rng.gamma(2.0, 1.0, K)
        c, code, it = oracle.kmeans_row(xs, u, 500)
        c_ref, code_ref = _sklearn_kmeans(xs, u)
        assert 0 < it < 500
        assert np.allclose(c, c_ref, rtol=1e-12, atol=1e-12)
        assert np.array_equal(code, code_ref)


def pin_kmeans_objective_never_increases():
    rng = np.random.default_rng(105)
    xs = rng.uniform(0, 15, 700) ** 1.5 / 15 ** 0.5
    u = rng.gamma(1.5, 1.0, 700)
    prev = None
    for t in range(12):
        c, code, _ = oracle.kmeans_row(xs, u, t)
        obj = math.fsum(u * (xs - c[code]) ** 2)
        if prev is not None:
            assert obj <= prev * (1 + 1e-12)
        prev = obj


def pin_quantize_matches_scikit_learn_pipeline():
    rng = np.random.default_rng(106)
    N, K, G = 3, 256, 64
    w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    ex = np.abs(rng.normal(0, 1, K)).astype(np.float32) + np.float32(0.05)
    codes, lut, scale, offset, _ = oracle.quantize(w, ex, G, 300)
    s_ref, o_ref = _numpy_scale(w, G)
    assert np.array_equal(scale, s_ref) and np.array_equal(offset, o_ref)
    a = torch_bf16_to_f64(s_ref).repeat(G, axis=1)
    b = torch_bf16_to_f64(o_ref).repeat(G, axis=1)
    ws = (torch_bf16_to_f64(w) - b) / a
    for n in range(N):
        u = a[n] * ex.astype(np.float64)
        c_ref, _ = _sklearn_kmeans(ws[n], u, 300)
        lut_ref = torch_bf16_bits(c_ref.astype(np.float32))
        assert np.array_equal(lut[n], lut_ref)
        assert np.array_equal(codes[n], _nearest(ws[n], torch_bf16_to_f64(lut_ref)))


def pin_quantize_recovers_exact_levels():
    rng = np.random.default_rng(107)
    levels = np.array([0, 0.5, 1.25, 2, 3.5, 4, 5.75, 6, 7.5, 8.25, 9, 10.5, 11.75, 13, 14.25,
                       15])
    N, K, G = 3, 512, 128
    w = _levels_problem(rng, N, K, G, levels)
    ex = rng.uniform(0.1, 2.0, K).astype(np.float32)
    codes, lut, scale, offset, _ = oracle.quantize(w, ex, G, 50)
    assert np.array_equal(torch_bf16_to_f64(lut), np.tile(levels, (N, 1)))
    a = torch_bf16_to_f64(scale).repeat(G, axis=1)
    b = torch_bf16_to_f64(offset).repeat(G, axis=1)
    assert np.array_equal(a * levels[codes] + b, torch_bf16_to_f64(w))


def pin_quantize_invariant_to_power_of_two_activation_scale():
    rng = np.random.default_rng(108)
    w = torch_bf16_bits(rng.normal(0, 0.02, (4, 512)).astype(np.float32))
    ex = rng.lognormal(0, 1, 512).astype(np.float32)
    r1 = oracle.quantize(w, ex, 128, 40)
    r2 = oracle.quantize(w, ex * np.float32(8), 128, 40)
    for a, b in zip(r1, r2):
        assert np.array_equal(a, b)


def pin_quantize_degenerate_rows():
    rng = np.random.default_rng(109)
    N, K, G = 3, 256, 64
    w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    w[0, :] = torch_bf16_bits(np.array([0.125], dtype=np.float32))[0]   # constant row
    w[1, G:2 * G] = w[1, G]                                             # one constant group
    ex = np.abs(rng.normal(0, 1, K)).astype(np.float32)
    codes, lut, scale, offset, _ = oracle.quantize(w, ex, G, 30)
    assert np.all(scale[0] == 0) and np.all(lut[0] == 0) and np.all(codes[0] == 0)
    assert np.all(offset[0] == w[0, 0])
    assert scale[1, 1] == 0 and offset[1, 1] == w[1, G]
    # no activation weight anywhere: every cluster keeps its entry of the quantile table
    codes2, lut2, scale2, offset2, it2 = oracle.quantize(w, np.zeros(K, np.float32), G, 30)
    ws = (torch_bf16_to_f64(w[2]) - torch_bf16_to_f64(offset2[2]).repeat(G)) / \
        torch_bf16_to_f64(scale2[2]).repeat(G)
    assert np.array_equal(lut2[2], torch_bf16_bits(_quantile_init(ws).astype(np.float32)))
    assert it2[2] == 1


def pin_quantize_beats_int4_rounding():
    """The paper's premise (§4.1) at toy scale: on Gaussian rows the learned
    table has a lower weighted error than the int4 grid on the same scaling,
    by more when a group spans the whole row (G = K) than at G = 128."""
    rng = np.random.default_rng(110)
    N, K = 6, 1024
    for G, bound in ((128, 0.9), (K, 0.75)):
        w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
        ex = rng.lognormal(0, 1, K).astype(np.float32)
        codes, lut, scale, offset, _ = oracle.quantize(w, ex, G, 100)
        a = torch_bf16_to_f64(scale).repeat(G, axis=1)
        b = torch_bf16_to_f64(offset).repeat(G, axis=1)
        ws = (torch_bf16_to_f64(w) - b) / a
        u = a * ex.astype(np.float64)
        rec = np.take_along_axis(torch_bf16_to_f64(lut), codes.astype(np.int64), 1)
        err_any4 = math.fsum((u * (ws - rec) ** 2).ravel())
        err_int4 = math.fsum((u * (ws - np.clip(np.round(ws), 0, 15)) ** 2).ravel())
        assert err_any4 < bound * err_int4, (G, err_any4 / err_int4)


# --------------------------------------------------------------------------
# n-bit variants: any3 and any2 (§4.1 Eq. 9: 2^n values per row; §5).  The
# storage reading (the pages give none below 4 bits): a row's codes form one
# little-endian bit stream, code k in bits [n k, n k + n).
# --------------------------------------------------------------------------

def pin_pack_bits_worked_examples():
    # any3, codes 1..7 then 0: the 24-bit little-endian word sum(c_k << 3k)
    # = 1 + 2*8 + 3*64 + 4*512 + 5*4096 + 6*32768 + 7*262144 = 0x1F58D1
    assert oracle.pack_bits(np.array([[1, 2, 3, 4, 5, 6, 7, 0]], np.uint8), 3).tolist() == \
        [[0xD1, 0x58, 0x1F]]
    # any2, codes 0 1 2 3 | 3 2 1 0: bytes 0b11100100 and 0b00011011
    assert oracle.pack_bits(np.array([[0, 1, 2, 3, 3, 2, 1, 0]], np.uint8), 2).tolist() == \
        [[0xE4, 0x1B]]


def pin_pack_bits_is_a_little_endian_bit_stream():
    rng = np.random.default_rng(120)
    for bits in (2, 3, 4):
        idx = rng.integers(0, 1 << bits, size=(5, 64), dtype=np.uint8)
        packed = oracle.pack_bits(idx, bits)
        assert packed.shape == (5, bits * 64 // 8)
        stream = np.unpackbits(packed, axis=1, bitorder="little").reshape(5, 64, bits)
        assert np.array_equal((stream << np.arange(bits)).sum(axis=2), idx)   # numpy's decoder
        assert np.array_equal(oracle.unpack_bits(packed, bits, 64), idx)
        if bits == 4:
            assert np.array_equal(packed, oracle.pack(idx))          # the any4 nibble order
        bad = idx.copy()
        bad[2, 7] = 1 << bits
        try:
            oracle.pack_bits(bad, bits)
        except ValueError:
            pass
        else:
            raise AssertionError("out-of-range code accepted")


def pin_dequant_bits_reduces_to_any4():
    """n-bit codes with a 2^n-entry table equal any4 codes with the table
    padded to 16 entries (the padding is never indexed)."""
    rng = np.random.default_rng(121)
    N, K, G = 6, 256, 64
    for bits in (2, 3):
        nq = 1 << bits
        idx = rng.integers(0, nq, size=(N, K), dtype=np.uint8)
        lut = random_bf16(rng, (N, nq))
        pad = random_bf16(rng, (N, 16 - nq))
        scale = random_bf16(rng, (N, K // G), -8, -4)
        offset = random_bf16(rng, (N, K // G), -10, -6)
        W = oracle.dequant_bits(oracle.pack_bits(idx, bits), lut, scale, offset, G, bits, K)
        W4 = oracle.dequant(oracle.pack(idx), np.concatenate([lut, pad], axis=1), scale, offset, G)
        assert np.array_equal(W, W4)
        one = lut[0]
        Ws = oracle.dequant_bits(oracle.pack_bits(idx, bits), one, scale, offset, G, bits, K,
                                 per_tensor_lut=True)
        W4s = oracle.dequant(oracle.pack(idx), np.concatenate([one, pad[0]]), scale, offset, G,
                             per_tensor_lut=True)
        assert np.array_equal(Ws, W4s)


def pin_bits_per_weight_n_accounting():
    # the §2.4.1 accounting with 2^n table entries: any4 4.3125 (the paper's
    # worked example), any3 3 + 0.25 + 0.03125, any2 2 + 0.25 + 0.015625
    for bits, expect in ((4, 4.3125), (3, 3.28125), (2, 2.265625)):
        assert oracle.bits_per_weight_n(4096, 128, bits) == expect
    N, K, G = 3, 512, 64
    for bits in (2, 3, 4):
        nbytes = N * bits * K // 8 + 2 * 2 * N * (K // G) + 2 * N * (1 << bits)
        assert oracle.bits_per_weight_n(K, G, bits) == 8 * nbytes / (N * K)


def pin_quantize_bits_matches_scikit_learn_pipeline():
    rng = np.random.default_rng(122)
    N, K, G = 3, 256, 64
    for bits in (2, 3):
        nq = 1 << bits
        w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
        ex = np.abs(rng.normal(0, 1, K)).astype(np.float32) + np.float32(0.05)
        codes, lut, scale, offset, _ = oracle.quantize_bits(w, ex, G, bits, 300)
        s_ref, o_ref = _numpy_scale(w, G, levels=nq - 1)
        assert np.array_equal(scale, s_ref) and np.array_equal(offset, o_ref)
        a = torch_bf16_to_f64(s_ref).repeat(G, axis=1)
        b = torch_bf16_to_f64(o_ref).repeat(G, axis=1)
        ws = (torch_bf16_to_f64(w) - b) / a
        for n in range(N):
            c_ref, _ = _sklearn_kmeans(ws[n], a[n] * ex.astype(np.float64), 300, nq)
            lut_ref = torch_bf16_bits(c_ref.astype(np.float32))
            assert np.array_equal(lut[n], lut_ref)
            assert np.array_equal(codes[n], _nearest(ws[n], torch_bf16_to_f64(lut_ref)))


def pin_quantize_bits_four_is_any4():
    rng = np.random.default_rng(123)
    w = torch_bf16_bits(rng.normal(0, 0.02, (5, 512)).astype(np.float32))
    ex = rng.lognormal(0, 1, 512).astype(np.float32)
    for a, b in zip(oracle.quantize_bits(w, ex, 128, 4, 60), oracle.quantize(w, ex, 128, 60)):
        assert np.array_equal(a, b)


def pin_quantize_bits_recovers_exact_levels():
    rng = np.random.default_rng(124)
    levels = np.array([0, 1, 2.5, 3, 4.25, 5.5, 6, 7])
    N, K, G = 3, 256, 64
    w = _levels_problem(rng, N, K, G, levels)
    ex = rng.uniform(0.1, 2, K).astype(np.float32)
    codes, lut, scale, offset, _ = oracle.quantize_bits(w, ex, G, 3, 50)
    assert np.array_equal(torch_bf16_to_f64(lut), np.tile(levels, (N, 1)))
    a = torch_bf16_to_f64(scale).repeat(G, axis=1)
    b = torch_bf16_to_f64(offset).repeat(G, axis=1)
    assert np.array_equal(a * levels[codes] + b, torch_bf16_to_f64(w))


def pin_quantize_bits_error_falls_with_more_bits():
    """Weighted reconstruction error of w (weights E|x|): any2 > any3 > any4."""
    rng = np.random.default_rng(125)
    N, K, G = 4, 1024, 128
    w = torch_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    ex = rng.lognormal(0, 1, K).astype(np.float32)
    wf = torch_bf16_to_f64(w)
    errs = []
    for bits in (2, 3, 4):
        codes, lut, scale, offset, _ = oracle.quantize_bits(w, ex, G, bits, 100)
        rec = (np.take_along_axis(torch_bf16_to_f64(lut), codes.astype(np.int64), 1)
               * torch_bf16_to_f64(scale).repeat(G, axis=1)
               + torch_bf16_to_f64(offset).repeat(G, axis=1))
        errs.append(math.fsum((ex.astype(np.float64) * (wf - rec) ** 2).ravel()))
    assert errs[0] > 2 * errs[1] > 4 * errs[2], errs


# --------------------------------------------------------------------------
# the M = 1 decode layout (any4_repack): positions worked by hand, invariants
# --------------------------------------------------------------------------

def _word_index_rows(K: int) -> np.ndarray:
    """One row whose 32-bit word w holds the value w in each of its bytes
    (w < 256), so a byte of the repacked row names the word it came from."""
    words = np.arange(K // 8, dtype=np.uint32)
    assert words.max() < 256
    return np.repeat(words.astype(np.uint8), 4).reshape(1, K // 2)


def pin_repack_decode_layout_worked_positions():
    for row in read_golden("repack_decode_layout.txt"):
        K, lane, w0, w1, w2, w3, sl = (int(v) for v in row.split())
        got = oracle.repack_decode_layout(_word_index_rows(K))[0]
        for t, want in enumerate((w0, w1, w2, w3)):
            at = 512 * sl + 16 * lane + 4 * t
            assert np.all(got[at:at + 4] == want), (K, lane, t, got[at:at + 4], want)


def pin_repack_decode_layout_is_a_word_permutation():
    # whole 32-bit words move, inside their own 1024-column slice, row by row
    rng = np.random.default_rng(11)
    packed = rng.integers(0, 256, size=(3, 14336 // 2), dtype=np.uint8)
    out = oracle.repack_decode_layout(packed)
    for n in range(3):
        a = packed[n].view(np.uint32).reshape(-1, 128)
        b = out[n].view(np.uint32).reshape(-1, 128)
        for sl in range(a.shape[0]):
            assert np.array_equal(np.sort(a[sl]), np.sort(b[sl])), (n, sl)
        assert np.array_equal(out[n], oracle.repack_decode_layout(packed[n:n + 1])[0])
    try:
        oracle.repack_decode_layout(np.zeros((1, 768), dtype=np.uint8))
    except ValueError:
        return
    raise AssertionError("K = 1536 was accepted")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
