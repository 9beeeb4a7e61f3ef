"""any4_read_probe: the read-only stream used as the decode matmuls' read
roofline must really read every byte once.  Its result, the XOR of all 32-bit
words, is checked against numpy's reduction of the same bytes for sizes that
leave the grid-stride loop a ragged tail, sizes smaller than one pass of the
grid, and the empty buffer."""
import numpy as np
import pytest
import torch

import learned_bit_lut_any4_b200 as any4

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096 + 16, 148 * 8 * 256 * 16 + 48, 50 * 2**20 + 208])
def test_read_probe_xor_of_every_word(nbytes):
    rng = np.random.default_rng(nbytes)
    host = rng.integers(0, 2**32, size=nbytes // 4, dtype=np.uint32)
    buf = torch.from_numpy(host.view(np.int32)).cuda()
    got = any4.any4_read_probe(buf)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host)
    assert int(got.cpu().numpy().view(np.uint32)[0]) == int(want)


def test_read_probe_every_word_counts():
    # flipping one bit anywhere (here: the last word, the tail of the grid
    # stride) changes the result
    host = np.zeros(148 * 8 * 256 * 4 * 4 + 12, dtype=np.uint32)
    host[-1] = 1 << 7
    buf = torch.from_numpy(host.view(np.int32)).cuda()
    out = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    any4.any4_read_probe(buf, out)
    torch.cuda.synchronize()
    assert int(out.item()) == 1 << 7


def test_read_probe_empty_buffer_gives_zero():
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    any4.any4_read_probe(torch.empty(0, dtype=torch.uint8, device="cuda"), out)
    torch.cuda.synchronize()
    assert int(out.item()) == 0
