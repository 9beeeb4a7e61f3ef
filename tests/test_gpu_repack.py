"""any4_repack and the M = 1 decode layout (ANY4_FLAG_DECODE_LAYOUT).

The repacked codes must equal the oracle's statement of the layout byte for
byte, and a matmul on them must give the same bits as the same call on
any4_pack's layout (which the other decode tests hold to the oracle), for
single and grouped calls, shared and per-row tables, fp32 output and the
prepared-weights path.  Calls the layout does not serve are refused."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, dev_bf16, dev_u8, host_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(1, 1024), (5, 4096), (33, 14336), (7, 8192), (1000, 2048)])
def test_repack_matches_oracle(N, K):
    rng = np.random.default_rng(N * 7 + K)
    packed = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    got = any4.any4_repack(dev_u8(packed))
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), oracle.repack_decode_layout(packed))


def _problem(name, M, K, N, G, seed):
    s = workloads.Shape(name, M, K, N, G, seed, seed + 1)
    return s, workloads.make(s)


@pytest.mark.parametrize("K,N,shared,fp32", [
    (4096, 4096, False, False),
    (4096, 333, False, False),     # a ragged row count
    (14336, 1024, False, False),   # several slices per warp
    (8192, 700, True, False),      # one table for the matrix
    (4096, 1536, False, True),     # the fp32 sums
])
def test_decode_layout_matmul_equals_plain(K, N, shared, fp32):
    s, p = _problem(f"dl_{K}_{N}", 1, K, N, 128, 4000 + K + N)
    d = DeviceProblem(p, check_pack=False)
    lut = dev_bf16(p.lut[5]) if shared else d.lut
    rep = any4.any4_repack(d.packed)
    plain = any4.any4_matmul(d.x, d.packed, lut, d.scale, d.offset, 128, fp32_out=fp32)
    fast = any4.any4_matmul(d.x, rep, lut, d.scale, d.offset, 128, fp32_out=fp32,
                            decode_layout=True, overlap_prior=True)
    torch.cuda.synchronize()
    view = torch.int32 if fp32 else torch.int16
    assert torch.equal(plain.view(view), fast.view(view))
    if not fp32:
        lut_ref = p.lut[5] if shared else p.lut
        y_ref = oracle.any4_matmul(p.x, d.packed_ref, lut_ref, p.scale, p.offset, 128,
                                   per_tensor_lut=shared)
        assert_matmul_close(host_bits(fast), y_ref, s.name)


def test_decode_layout_grouped_and_prepared():
    K, G = 4096, 128
    probs = []
    for i, N in enumerate((4096, 1024, 1024)):
        s = workloads.Shape(f"dlg{i}", 1, K, N, G, 4100 + 17 * i, 4200)
        probs.append(DeviceProblem(workloads.make(s), check_pack=False))
    x = probs[0].x
    plain = [(d.packed, d.lut, d.scale, d.offset) for d in probs]
    reps = [(any4.any4_repack(d.packed), d.lut, d.scale, d.offset) for d in probs]
    ys_plain = any4.any4_matmul_grouped(x, plain, G)
    ys_rep = any4.any4_matmul_grouped(x, reps, G, decode_layout=True)
    prepared = [any4.any4_prepare(*w, G, decode_layout=True) for w in reps]
    ys_prep = any4.any4_matmul_grouped(x, prepared, G, overlap_prior=True)
    torch.cuda.synchronize()
    for a, b, c in zip(ys_plain, ys_rep, ys_prep):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_decode_layout_refused_where_not_served():
    s, p = _problem("dl_bad", 2, 4096, 256, 128, 4300)
    d = DeviceProblem(p, check_pack=False)
    rep = any4.any4_repack(d.packed)
    with pytest.raises(any4.Any4Error) as e:          # M = 2
        any4.any4_matmul(d.x, rep, d.lut, d.scale, d.offset, 128, decode_layout=True)
    assert e.value.status == any4.ANY4_ERR_UNSUPPORTED
    s64, p64 = _problem("dl_g64", 1, 4096, 256, 64, 4301)
    d64 = DeviceProblem(p64, check_pack=False)
    with pytest.raises(any4.Any4Error) as e:          # G = 64
        any4.any4_matmul(d64.x, any4.any4_repack(d64.packed), d64.lut, d64.scale, d64.offset, 64,
                         decode_layout=True)
    assert e.value.status == any4.ANY4_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        any4.any4_prepare(d64.packed, d64.lut, d64.scale, d64.offset, 64, decode_layout=True)
