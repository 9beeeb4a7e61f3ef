"""The pair-table decode kernel (M = 2 given its workspace, M = 1 on request)
against the fp64 oracle: the stream-K split of 64-row sets over the blocks, its cross-block
exchange (partial sums published with a per-launch flag), repeated calls and
CUDA-graph replays that reuse one workspace, and the shape edges of the
kernel (ragged rows and chunks, every group size, one table for the matrix).

Tolerance as in the other matmul tests: |y - y_ref| <= 1e-2 * rms(y_ref[m, :])
+ ulp_bf16(y_ref) per element.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, dev_bf16, host_bits

pytestmark = pytest.mark.gpu

# M = 1 runs the weight-streaming kernel unless the pair-table kernel is asked for
_mm = functools.partial(any4.any4_matmul, pair_table=True)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _ws(M, N, K, G):
    need = any4.any4_matmul_workspace_size(M, N, K, G)
    assert need > 0, "the pair-table kernel takes this shape"
    # garbage in the workspace: the kernel must not depend on its contents
    return torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("M,K,N,G", [
    (1, 4096, 64, 128),      # one row set split over 32 blocks (every block a contributor)
    (1, 4096, 4096, 128),    # 64 row sets, 2048 chunks: sets split between 2 blocks
    (2, 4096, 4096, 128),
    (1, 1024, 1024, 128),    # fewer units than SMs: one chunk per block
    (1, 14336, 100, 128),    # 2 row sets over every block, the second one ragged
    (2, 2048, 333, 64),      # ragged rows, G = 64
    (1, 1280, 777, 32),      # G = 32: a window every second chunk
    (1, 1280, 129, 32),      # one row more than two sets
    (2, 768, 65, 32),        # six chunks, 65 rows
    (1, 256, 5, 32),         # two chunks, five rows (K/G = 8 makes K a multiple of 256)
    (2, 8192, 28672 // 8, 128),
    (1, 1152, 300, 128),     # K / G = 9 groups per row (odd)
    (2, 640, 77, 64),        # K / G = 10
    (1, 384, 1000, 32),      # three chunks, twelve groups per row
])
def test_pair_stream_k_shapes(M, K, N, G):
    shape = workloads.Shape(f"pair_{M}_{K}_{N}_{G}", M, K, N, G, 8801 + N, 8802 + K // 32)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, G)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _mm(d.x, d.packed, d.lut, d.scale, d.offset, G, workspace=_ws(M, N, K, G),
                         dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_matmul_close(host_bits(y), y_ref, shape.name)


@pytest.mark.parametrize("M", [1, 2])
def test_pair_shared_table(M):
    shape = workloads.Shape(f"pair_shared_m{M}", M, 4096, 1500, 128, 8901, 8902)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    table = p.lut[7].copy()
    y = _mm(d.x, d.packed, dev_bf16(table), d.scale, d.offset, shape.G,
                         workspace=_ws(M, shape.N, shape.K, shape.G))
    torch.cuda.synchronize()
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, table, p.scale, p.offset, shape.G,
                               per_tensor_lut=True)
    assert_matmul_close(host_bits(y), y_ref, shape.name)


def test_pair_repeated_calls_share_one_workspace():
    """Calls in a row on one workspace with different x, and a call of another
    shape in between: every result matches its own oracle (a flag left by an
    earlier launch must never be taken for the current one's)."""
    a = workloads.Shape("pair_rep_a", 1, 4096, 4096, 128, 8911, 8912)
    b = workloads.Shape("pair_rep_b", 2, 14336, 700, 128, 8913, 8914)
    pa, pb = workloads.make(a), workloads.make(b)
    da, db = DeviceProblem(pa), DeviceProblem(pb)
    ws = torch.randint(0, 256, (max(any4.any4_matmul_workspace_size(1, a.N, a.K, a.G),
                                    any4.any4_matmul_workspace_size(2, b.N, b.K, b.G)),),
                       dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(8915)
    for i in range(4):
        xa = workloads._to_bf16_bits(rng.normal(0, 1, (1, a.K)).astype(np.float32))
        ya = _mm(dev_bf16(xa), da.packed, da.lut, da.scale, da.offset, a.G,
                              workspace=ws)
        yb = _mm(db.x, db.packed, db.lut, db.scale, db.offset, b.G, workspace=ws)
        torch.cuda.synchronize()
        assert_matmul_close(host_bits(ya), oracle.any4_matmul(xa, da.packed_ref, pa.lut,
                                                              pa.scale, pa.offset, a.G), f"a{i}")
        assert_matmul_close(host_bits(yb), oracle.any4_matmul(pb.x, db.packed_ref, pb.lut,
                                                              pb.scale, pb.offset, b.G), f"b{i}")


def test_pair_graph_replays():
    """One call captured in a CUDA graph and replayed with new contents of x
    between replays (same pointers): each replay is a new launch, and its
    result matches the oracle for the x it saw."""
    shape = workloads.Shape("pair_graph", 1, 4096, 2048, 128, 8921, 8922)
    p = workloads.make(shape)
    d = DeviceProblem(p)
    ws = _ws(1, shape.N, shape.K, shape.G)
    x = d.x.clone()
    y = torch.empty((1, shape.N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _mm(x, d.packed, d.lut, d.scale, d.offset, shape.G, y=y, workspace=ws)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _mm(x, d.packed, d.lut, d.scale, d.offset, shape.G, y=y, workspace=ws)
    rng = np.random.default_rng(8923)
    for i in range(3):
        xb = workloads._to_bf16_bits(rng.normal(0, 1, (1, shape.K)).astype(np.float32))
        x.copy_(dev_bf16(xb))
        g.replay()
        torch.cuda.synchronize()
        y_ref = oracle.any4_matmul(xb, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
        assert_matmul_close(host_bits(y), y_ref, f"replay {i}")
    del g


def test_pair_is_deterministic():
    shape = workloads.Shape("pair_det", 2, 14336, 4096, 128, 8931, 8932)
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    ws = _ws(2, shape.N, shape.K, shape.G)
    y1 = _mm(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, workspace=ws)
    y2 = _mm(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
