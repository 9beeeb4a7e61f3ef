"""any4_matmul_grouped: matrices that share x (q/k/v, gate/up) in one call.

Each y_i is checked against the fp64 oracle for its own matrix (tolerance of
the other matmul tests: |y - y_ref| <= 1e-2 * rms(y_ref[m, :]) + one bf16 ulp)
and must equal, bit for bit, the same matrix run alone through any4_matmul
(the grouped launch changes which block streams a row, not a row's sums)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


def _problems(M, K, G, Ns, seed, shared=()):
    """One DeviceProblem per matrix, all with the same x."""
    probs = []
    x = None
    for i, N in enumerate(Ns):
        s = workloads.Shape(f"grp{i}_{N}", M, K, N, G, seed + 17 * i, seed + 1000)
        p = workloads.make(s)
        if x is None:
            x = p.x
        assert np.array_equal(p.x, x)   # same x seed and shape: the same activations
        lut = p.lut[3 % N].copy() if i in shared else p.lut
        probs.append((s, p, DeviceProblem(p, check_pack=False), lut))
    return x, probs


def _check(M, K, G, Ns, seed, shared=(), path="auto", fp32=False, **kw):
    x, probs = _problems(M, K, G, Ns, seed, shared)
    xd = dev_bf16(x)
    weights = [(d.packed, dev_bf16(lut), d.scale, d.offset) for (_, _, d, lut) in probs]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = any4.any4_matmul_grouped(xd, weights, G, path=path, dev_status=status, fp32_out=fp32,
                                  **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (s, p, d, lut), y, w in zip(probs, ys, weights):
        alone = any4.any4_matmul(xd, *w, G, path=path, fp32_out=fp32, **kw)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int32 if fp32 else torch.int16),
                           alone.view(torch.int32 if fp32 else torch.int16)), s.name
        y_ref = oracle.any4_matmul(x, d.packed_ref, lut, p.scale, p.offset, G,
                                   per_tensor_lut=lut.ndim == 1)
        if fp32:
            rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
            assert (np.abs(y.cpu().numpy() - y_ref) <= 1e-3 * rms).all(), s.name
        else:
            assert_matmul_close(host_bits(y), y_ref, s.name)
    return ys


def test_grouped_llama3_8b_qkv():
    _check(1, 4096, 128, (4096, 1024, 1024), 12001)


def test_grouped_llama3_8b_gate_up():
    _check(1, 4096, 128, (14336, 14336), 12101)


@pytest.mark.parametrize("G", [32, 64, 128])
def test_grouped_ragged_rows_and_one_table(G):
    """Four matrices (the most a group takes) with row counts that end mid
    block, one of them in the one-table mode."""
    _check(1, 2048, G, (333, 7, 1000, 64), 12201 + G, shared=(1,))


def test_grouped_single_matrix():
    _check(1, 3072, 64, (777,), 12301)


def test_grouped_fp32_sums():
    _check(1, 4096, 128, (4096, 1024), 12401, fp32=True)


@pytest.mark.parametrize("M,G", [(2, 128), (5, 128), (1, 256), (40, 64)])
def test_grouped_other_paths_run_per_matrix(M, G):
    """Where the one-launch kernel does not apply (M > 1, or G = 256) the
    group runs as calls of any4_matmul one after the other."""
    _check(M, 2048, G, (640, 96, 1200), 12501 + M)


def test_grouped_pair_table_at_m1():
    _check(1, 4096, 128, (2048, 512), 12601, pair_table=True)


def test_grouped_stall_times_out_cleanly():
    """ANY4_FLAG_TEST_STALL on the one-launch kernel: block 0 stops its stream,
    the call ends with ANY4_ERR_TIMEOUT, nothing outside the outputs is
    written, and the next call on the stream is correct."""
    x, probs = _problems(1, 4096, 128, (14336, 1024), 12701)
    xd = dev_bf16(x)
    weights = [(d.packed, d.lut, d.scale, d.offset) for (_, _, d, _) in probs]
    pad = 512
    bufs, ys = [], []
    for (s, _, _, _) in probs:
        b = torch.full((pad + s.N + pad,), -3, dtype=torch.int16, device="cuda")
        bufs.append(b)
        ys.append(b[pad:pad + s.N].view(1, s.N).view(torch.bfloat16))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    any4.any4_matmul_grouped(xd, weights, 128, ys=ys, dev_status=status, test_stall=True)
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_TIMEOUT
    for b in bufs:
        assert (b[:pad] == -3).all() and (b[-pad:] == -3).all()
    status.zero_()
    out = any4.any4_matmul_grouped(xd, weights, 128, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (s, p, d, _), y in zip(probs, out):
        y_ref = oracle.any4_matmul(x, d.packed_ref, p.lut, p.scale, p.offset, 128)
        assert_matmul_close(host_bits(y), y_ref, s.name + " after the stall")


@pytest.mark.parametrize("M,K,G,Ns,seed", [
    (1, 4096, 128, (4096, 1024, 1024), 12101),   # q/k/v, the folded-table kernel
    (1, 2048, 64, (333, 1024), 12102),           # G = 64 and a ragged N: the per-weight kernel
    (4, 1024, 128, (512,), 12103),               # M > 1: one matrix per launch
])
def test_prepared_weights_equal_plain_call(M, K, G, Ns, seed):
    """Weights checked once (any4_prepare) give the same bits as the plain call."""
    x, probs = _problems(M, K, G, Ns, seed)
    xd = dev_bf16(x)
    weights = [(d.packed, dev_bf16(lut), d.scale, d.offset) for (_, _, d, lut) in probs]
    prepared = [any4.any4_prepare(*w, G) for w in weights]
    plain = any4.any4_matmul_grouped(xd, weights, G)
    fast = any4.any4_matmul_grouped(xd, prepared, G)
    ys = [torch.empty_like(y) for y in plain]
    fast2 = any4.any4_matmul_grouped(xd, prepared, G, ys=ys)
    torch.cuda.synchronize()
    assert all(a is b for a, b in zip(fast2, ys))
    for a, b, c in zip(plain, fast, fast2):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_prepared_weights_check_x_and_y():
    x, probs = _problems(1, 1024, 128, (256,), 12104)
    _, _, d, lut = probs[0]
    w = any4.any4_prepare(d.packed, dev_bf16(lut), d.scale, d.offset, 128)
    xd = dev_bf16(x)
    with pytest.raises(ValueError):
        any4.any4_matmul_grouped(xd[:, :512].contiguous(), [w], 128)       # wrong K
    with pytest.raises(ValueError):
        any4.any4_matmul_grouped(xd, [w], 64)                              # another G
    with pytest.raises(ValueError):
        any4.any4_matmul_grouped(xd, [w], 128,
                                 ys=[torch.empty((1, 255), dtype=torch.bfloat16, device="cuda")])
    with pytest.raises(TypeError):
        any4.any4_matmul_grouped(xd.float(), [w], 128)
    with pytest.raises(TypeError):
        any4.any4_matmul_grouped(xd, [w, (d.packed, dev_bf16(lut), d.scale, d.offset)], 128)
