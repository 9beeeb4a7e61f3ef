"""The bounded waits of the kernels run out on purpose (ANY4_FLAG_TEST_STALL):
block 0 stops its weight or x stream after the first stage, every wait of the
kernel gives up after 1 ms, and the call must end with ANY4_ERR_TIMEOUT in
dev_status, write nothing outside y, and leave the stream usable: a normal
call right after it on the same stream is correct.  No fault is provoked: the
stall is a stream that is never issued, not a bad address or a wrong byte
count."""
import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, host_bits

pytestmark = pytest.mark.gpu

CASES = [
    # (name, M, K, N, G, workspace): the kernel that runs
    # shapes where warp 0 of block 0 has several stages to stream
    ("pair_table", 1, 4096, 14336, 128, "auto"),      # pair-table decode
    ("pair_table_m2", 2, 4096, 14336, 128, "auto"),
    ("shuffle_stream", 1, 4096, 14336, 128, "none"),  # weight-streaming decode
    ("prefill_one_pass", 300, 2048, 1024, 128, "auto"),
    ("prefill_two_pass", 1024, 2048, 1024, 128, "auto"),
]


@pytest.mark.parametrize("name,M,K,N,G,ws", CASES, ids=[c[0] for c in CASES])
def test_stalled_stream_times_out_cleanly(name, M, K, N, G, ws):
    shape = workloads.Shape(f"stall_{name}", M, K, N, G, 8601, 8602 + M)
    p = workloads.make(shape)
    d = DeviceProblem(p, check_pack=False)
    if ws == "none":
        workspace = torch.empty(0, dtype=torch.uint8, device="cuda")
    else:
        need = any4.any4_matmul_workspace_size(M, N, K, G)
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
    pad = 1024
    buf = torch.full((pad + M * N + pad,), -3, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + M * N].view(M, N).view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, G, y=y, workspace=workspace,
                     dev_status=status, test_stall=True, pair_table=name == "pair_table")
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_TIMEOUT
    assert (buf[:pad] == -3).all() and (buf[pad + M * N:] == -3).all()
    # the same stream, right after: a normal call is correct (a workspace that
    # saw a timed-out call is cleared before its next use, as the header asks)
    if workspace is not None:
        workspace.zero_()
    status.zero_()
    y2 = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, G, workspace=workspace,
                          dev_status=status, pair_table=name == "pair_table")
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    y_ref = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, G)
    assert_matmul_close(host_bits(y2), y_ref, name + " after the stall")


@pytest.mark.parametrize("bits", [2, 3])
def test_stalled_nbit_stream_times_out_cleanly(bits):
    """The weight-streaming kernel on n-bit codes (any4_matmul_bits, M = 1):
    the same stall, the same clean end, then a correct call."""
    import numpy as np
    from tests.gpu_helpers import dev_bf16, dev_u8
    from tests.oracle_pins import torch_bf16_bits
    K, N, G = 4096, 14336, 128
    rng = np.random.default_rng(8700 + bits)
    nq = 1 << bits
    idx = rng.integers(0, nq, size=(N, K), dtype=np.uint8)
    lut = torch_bf16_bits(np.sort(rng.normal(0, 0.5, (N, nq)), axis=1).astype(np.float32))
    scale = torch_bf16_bits((np.abs(rng.normal(0, 0.01, (N, K // G))) + 1e-3).astype(np.float32))
    offset = torch_bf16_bits(rng.normal(0, 0.002, (N, K // G)).astype(np.float32))
    x = torch_bf16_bits(rng.normal(0, 1, (1, K)).astype(np.float32))
    packed = oracle.pack_bits(idx, bits)
    args = (dev_bf16(x), dev_u8(packed), dev_bf16(lut), dev_bf16(scale), dev_bf16(offset), G, bits)
    pad = 1024
    buf = torch.full((pad + N + pad,), -3, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + N].view(1, N).view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    any4.any4_matmul_bits(*args, y=y, dev_status=status, test_stall=True)
    torch.cuda.synchronize()
    assert int(status.item()) == any4.ANY4_ERR_TIMEOUT
    assert (buf[:pad] == -3).all() and (buf[pad + N:] == -3).all()
    status.zero_()
    y2 = any4.any4_matmul_bits(*args, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    W = oracle.dequant_bits(packed, lut, scale, offset, G, bits, K)
    assert_matmul_close(host_bits(y2), oracle.matmul(x, W), f"any{bits} after the stall")
