"""any4_matmul_static_scratch: the prefill kernel with the library's fixed
scratch array in place of a caller-supplied workspace.

The file name sorts last so that the GPU test runs after every other test in a
full session, and it also passes alone in a fresh process (the first call on a
device then does the array's address look-up).  The entry point is compared
with the existing workspace entry point (any4_matmul on the prefill path) on
two calls in a row -- the second call checks that the stream-K flags in the
fixed array are cleared again -- within the matmul tolerance of the other
tests, and with the fp64 oracle.
"""
import os
import re

import pytest
import torch

import oracle
import workloads
import learned_bit_lut_any4_b200 as any4
from tests.gpu_helpers import DeviceProblem, assert_matmul_close, bits_to_f64, host_bits

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "any4.h")


def test_static_scratch_size_matches_header():
    """The binding's constant is the header's ANY4_STATIC_SCRATCH_BYTES."""
    text = open(HEADER).read()
    m = re.search(r"#define ANY4_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) \* (\d+) \+ (\d+)\)", text)
    assert m, "ANY4_STATIC_SCRATCH_BYTES not found in any4.h"
    a, b, c = (int(v) for v in m.groups())
    assert any4.ANY4_STATIC_SCRATCH_BYTES == a * b + c


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [
    # ragged in M, N and the last K stage; several stream-K blocks share tiles
    workloads.Shape("noalloc_ragged", 300, 1056, 520, 32, 9931, 9932),
    # 2 x 4 tiles of 32 stages over 64 blocks: every tile split across blocks
    workloads.Shape("noalloc_split", 512, 2048, 1024, 128, 9933, 9934),
    # M >= 1024: the workspace entry point runs the two-pass route here (its
    # workspace holds the dequantised weights), this entry point the one-pass
    # kernel; they agree within the matmul tolerance, not bit for bit
    workloads.Shape("noalloc_m1024", 1024, 1024, 1024, 128, 9935, 9936),
], ids=lambda s: s.name)
def test_static_scratch_matches_workspace_entry(shape):
    p = workloads.make(shape)
    d = DeviceProblem(p)
    y_ws = any4.any4_matmul(d.x, d.packed, d.lut, d.scale, d.offset, shape.G, path="prefill")
    torch.cuda.synchronize()
    y_ws_bits = host_bits(y_ws)
    y_oracle = oracle.any4_matmul(p.x, d.packed_ref, p.lut, p.scale, p.offset, shape.G)
    assert_matmul_close(y_ws_bits, y_oracle, shape.name + " workspace entry")

    y = torch.empty((shape.M, shape.N), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        y.view(torch.int16).fill_(0x7FC1)  # a NaN pattern: a call that writes nothing fails
        any4.any4_matmul_static_scratch(d.x, d.packed, d.lut, d.scale, d.offset, shape.G,
                                        y=y, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, call
        got = host_bits(y)
        # the existing entry point as the reference, with the tests' tolerance
        assert_matmul_close(got, bits_to_f64(y_ws_bits), f"{shape.name} call {call} vs workspace")
        assert_matmul_close(got, y_oracle, f"{shape.name} call {call} vs oracle")
