"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import oracle
import learned_bit_lut_any4_b200 as any4
from learned_bit_lut_any4_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            names += re.findall(r"^ANY4_API\s+[\w\s\*]+?\b(any4_\w+)\s*\(", text, re.M)
    return names


def test_header_declares_entry_points():
    names = declared_symbols()
    for required in ("any4_pack", "any4_dequant", "any4_matmul"):
        assert required in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(any4.library_path())
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_version_and_strings():
    assert any4.any4_version() >= 10000
    for s in (0, -1, -2, -3, -4, -5, -6, -7, -8, -12345):
        assert isinstance(any4.any4_status_string(s), str) and any4.any4_status_string(s)


@pytest.mark.parametrize("K,G", [(4096, 128), (4096, 64), (1024, 128), (14336, 128),
                                 (28672, 128), (96, 32)])
def test_bits_per_weight_matches_oracle(K, G):
    # the oracle's accounting is pinned to the worked example of the paper (§2.4.1)
    assert any4.any4_bits_per_weight(K, G) == pytest.approx(oracle.bits_per_weight(K, G), abs=0)


FAKE = 0x10000  # an aligned, never dereferenced address (validation runs first)


def _matmul(M=1, N=64, K=128, G=32, x=FAKE, packed=FAKE, lut=FAKE, stride=16, scale=FAKE,
            offset=FAKE, y=FAKE, ws=None, ws_bytes=0, status=None, path=0, flags=0):
    return _native.library().any4_matmul_ex(x, packed, lut, stride, scale, offset, y, M, N, K,
                                            G, ws, ws_bytes, status, path, flags, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=None), any4.ANY4_ERR_NULL),
    (dict(packed=None), any4.ANY4_ERR_NULL),
    (dict(lut=None), any4.ANY4_ERR_NULL),
    (dict(scale=None), any4.ANY4_ERR_NULL),
    (dict(offset=None), any4.ANY4_ERR_NULL),
    (dict(y=None), any4.ANY4_ERR_NULL),
    (dict(M=0), any4.ANY4_ERR_SHAPE),
    (dict(N=0), any4.ANY4_ERR_SHAPE),
    (dict(K=0), any4.ANY4_ERR_SHAPE),
    (dict(K=48, G=48), any4.ANY4_ERR_SHAPE),
    (dict(K=128, G=48), any4.ANY4_ERR_SHAPE),
    (dict(K=96, G=64), any4.ANY4_ERR_SHAPE),
    (dict(K=16, G=16), any4.ANY4_ERR_SHAPE),
    (dict(stride=8), any4.ANY4_ERR_SHAPE),
    (dict(x=FAKE + 2), any4.ANY4_ERR_ALIGN),
    (dict(packed=FAKE + 8), any4.ANY4_ERR_ALIGN),
    (dict(y=FAKE + 4), any4.ANY4_ERR_ALIGN),
    (dict(status=FAKE + 2), any4.ANY4_ERR_ALIGN),
    (dict(M=17, path=1), any4.ANY4_ERR_UNSUPPORTED),
    (dict(path=7), any4.ANY4_ERR_UNSUPPORTED),
    (dict(flags=32), any4.ANY4_ERR_UNSUPPORTED),
    (dict(flags=64), any4.ANY4_ERR_UNSUPPORTED),
    # the decode layout: only M = 1, G = 128, K a multiple of 1024, decode path
    (dict(flags=16), any4.ANY4_ERR_UNSUPPORTED),
    (dict(M=2, K=4096, G=128, flags=16), any4.ANY4_ERR_UNSUPPORTED),
    (dict(K=4096, G=64, flags=16), any4.ANY4_ERR_UNSUPPORTED),
    (dict(K=3072 - 1024 + 512, G=128, flags=16), any4.ANY4_ERR_UNSUPPORTED),
    (dict(K=4096, G=128, path=2, flags=16), any4.ANY4_ERR_UNSUPPORTED),
    (dict(K=4096, G=128, flags=16 | 8), any4.ANY4_ERR_UNSUPPORTED),
    (dict(ws=FAKE + 8, ws_bytes=1 << 20), any4.ANY4_ERR_ALIGN),
])
def test_matmul_rejects_bad_arguments(kw, expect):
    assert _matmul(**kw) == expect


def test_repack_rejects_bad_arguments():
    lib = _native.library()
    N, K = 4, 2048
    assert lib.any4_repack(None, FAKE, N, K, None) == any4.ANY4_ERR_NULL
    assert lib.any4_repack(FAKE, None, N, K, None) == any4.ANY4_ERR_NULL
    assert lib.any4_repack(FAKE, FAKE + (1 << 20), N, 1536, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_repack(FAKE, FAKE + (1 << 20), 0, K, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_repack(FAKE + 4, FAKE + (1 << 20), N, K, None) == any4.ANY4_ERR_ALIGN
    # in place, or overlapping, is refused (the layout is a gather)
    assert lib.any4_repack(FAKE, FAKE, N, K, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_repack(FAKE, FAKE + 1024, N, K, None) == any4.ANY4_ERR_SHAPE
    import torch
    with pytest.raises(ValueError, match="multiple of 1024"):
        any4.any4_repack(torch.zeros((4, 768), dtype=torch.uint8))


def test_read_probe_rejects_bad_arguments():
    lib = _native.library()
    assert lib.any4_read_probe(FAKE, 64, None, None) == any4.ANY4_ERR_NULL
    assert lib.any4_read_probe(None, 64, FAKE, None) == any4.ANY4_ERR_NULL
    assert lib.any4_read_probe(FAKE, 40, FAKE + 64, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_read_probe(FAKE, -16, FAKE + 64, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_read_probe(FAKE + 8, 64, FAKE + 4096, None) == any4.ANY4_ERR_ALIGN
    assert lib.any4_read_probe(FAKE, 64, FAKE + 4098, None) == any4.ANY4_ERR_ALIGN
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        any4.any4_read_probe(torch.zeros(16, dtype=torch.uint8))


def test_pack_and_dequant_reject_bad_arguments():
    lib = _native.library()
    assert lib.any4_pack(None, FAKE, 4, 64, None, None) == any4.ANY4_ERR_NULL
    assert lib.any4_pack(FAKE, FAKE, 4, 48, None, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_pack(FAKE, FAKE, 0, 64, None, None) == any4.ANY4_ERR_SHAPE
    assert lib.any4_pack(FAKE + 1, FAKE, 4, 64, None, None) == any4.ANY4_ERR_ALIGN
    assert lib.any4_dequant(FAKE, FAKE, 16, FAKE, FAKE, None, 4, 64, 32, None) == \
        any4.ANY4_ERR_NULL
    assert lib.any4_dequant(FAKE, FAKE, 16, FAKE, FAKE, FAKE, 4, 64, 48, None) == \
        any4.ANY4_ERR_SHAPE
    assert lib.any4_dequant(FAKE, FAKE, 3, FAKE, FAKE, FAKE, 4, 64, 32, None) == \
        any4.ANY4_ERR_SHAPE
    assert lib.any4_dequant(FAKE, FAKE + 6, 16, FAKE, FAKE, FAKE, 4, 64, 32, None) == \
        any4.ANY4_ERR_ALIGN


@pytest.mark.parametrize("kw,expect", [
    (dict(w=None), any4.ANY4_ERR_NULL),
    (dict(ex=None), any4.ANY4_ERR_NULL),
    (dict(offset=None), any4.ANY4_ERR_NULL),
    (dict(K=48), any4.ANY4_ERR_SHAPE),
    (dict(G=48), any4.ANY4_ERR_SHAPE),
    (dict(N=0), any4.ANY4_ERR_SHAPE),
    (dict(K=any4.ANY4_QUANTIZE_MAX_K + 32, G=32), any4.ANY4_ERR_SHAPE),
    (dict(max_iter=-1), any4.ANY4_ERR_SHAPE),
    (dict(max_iter=any4.ANY4_QUANTIZE_MAX_ITER + 1), any4.ANY4_ERR_SHAPE),
    (dict(ex=FAKE + 4), any4.ANY4_ERR_ALIGN),
    (dict(packed=FAKE + 8), any4.ANY4_ERR_ALIGN),
    (dict(iters=FAKE + 2), any4.ANY4_ERR_ALIGN),
])
def test_quantize_rejects_bad_arguments(kw, expect):
    a = dict(w=FAKE, ex=FAKE, N=4, K=256, G=64, max_iter=10, packed=FAKE, lut=FAKE, scale=FAKE,
             offset=FAKE, iters=None)
    a.update(kw)
    assert _native.library().any4_quantize(a["w"], a["ex"], a["N"], a["K"], a["G"],
                                           a["max_iter"], a["packed"], a["lut"], a["scale"],
                                           a["offset"], a["iters"], None) == expect


def test_nbit_calls_reject_bad_arguments():
    lib = _native.library()
    E = any4
    # pack: bits outside 2..4, shapes, alignment
    assert lib.any4_pack_bits(FAKE, FAKE, 4, 64, 5, None, None) == E.ANY4_ERR_SHAPE
    assert lib.any4_pack_bits(FAKE, FAKE, 4, 64, 1, None, None) == E.ANY4_ERR_SHAPE
    assert lib.any4_pack_bits(None, FAKE, 4, 64, 3, None, None) == E.ANY4_ERR_NULL
    assert lib.any4_pack_bits(FAKE, FAKE, 4, 48, 3, None, None) == E.ANY4_ERR_SHAPE
    assert lib.any4_pack_bits(FAKE, FAKE + 4, 4, 64, 2, None, None) == E.ANY4_ERR_ALIGN
    assert lib.any4_pack_bits(FAKE + 1, FAKE, 4, 64, 4, None, None) == E.ANY4_ERR_ALIGN
    # dequant: the table stride must be 2^bits or 0
    assert lib.any4_dequant_bits(FAKE, FAKE, 16, FAKE, FAKE, FAKE, 4, 64, 32, 3, None) == \
        E.ANY4_ERR_SHAPE
    assert lib.any4_dequant_bits(FAKE, FAKE, 8, FAKE, FAKE, FAKE, 4, 64, 48, 3, None) == \
        E.ANY4_ERR_SHAPE
    assert lib.any4_dequant_bits(FAKE, FAKE, 4, FAKE, FAKE, None, 4, 64, 32, 2, None) == \
        E.ANY4_ERR_NULL
    assert lib.any4_dequant_bits(FAKE, FAKE + 2, 4, FAKE, FAKE, FAKE, 4, 64, 32, 2, None) == \
        E.ANY4_ERR_ALIGN
    assert lib.any4_dequant_bits(FAKE, FAKE, 8, FAKE, FAKE, FAKE, 4, 64, 32, 6, None) == \
        E.ANY4_ERR_SHAPE
    # quantize: bits, and the any4 limits
    q = lib.any4_quantize_bits
    assert q(FAKE, FAKE, 4, 256, 64, 1, 10, FAKE, FAKE, FAKE, FAKE, None, None) == E.ANY4_ERR_SHAPE
    assert q(FAKE, FAKE, 4, 256, 64, 5, 10, FAKE, FAKE, FAKE, FAKE, None, None) == E.ANY4_ERR_SHAPE
    assert q(FAKE, FAKE, 4, 256, 48, 3, 10, FAKE, FAKE, FAKE, FAKE, None, None) == E.ANY4_ERR_SHAPE
    assert q(FAKE, None, 4, 256, 64, 2, 10, FAKE, FAKE, FAKE, FAKE, None, None) == E.ANY4_ERR_NULL
    assert q(FAKE, FAKE, 4, 256, 64, 3, -1, FAKE, FAKE, FAKE, FAKE, None, None) == E.ANY4_ERR_SHAPE
    assert q(FAKE, FAKE, 4, 256, 64, 2, 10, FAKE, FAKE + 8, FAKE, FAKE, None, None) == \
        E.ANY4_ERR_ALIGN


def test_workspace_size_of_bad_shapes_is_zero():
    assert any4.any4_matmul_workspace_size(1, 64, 48, 48) == 0
    assert any4.any4_matmul_workspace_size(0, 64, 64, 32) == 0


def _sm_count():
    import torch
    return (torch.cuda.get_device_properties(0).multi_processor_count
            if torch.cuda.is_available() else 160)


def test_workspace_sizes_by_path():
    """Decode at M <= 2 takes the pair-table kernel's stream-K exchange (one
    64 x M fp32 partial and one 8-byte flag per block of an SM-count grid,
    rounded to 256 bytes) where its shape rules hold, and nothing otherwise;
    prefill below M = 1024 needs the one-pass stream-K scratch (independent of
    the shape); from M = 1024 the size adds room for the dequantised bf16
    weights, N * K * 2 bytes rounded to 256."""
    N, K, G = 1100, 2048, 128
    sms = _sm_count()
    for M in (1, 2):
        assert any4.any4_matmul_workspace_size(M, N, K, G) == \
            ((sms * M * 64 * 4 + sms * 8 + 255) // 256) * 256
    assert any4.any4_matmul_workspace_size(1, N, K, 256) == 0       # G outside {32, 64, 128}
    assert any4.any4_matmul_workspace_size(1, N, 1024 + 64, 64) == 0  # K not a multiple of 128
    for M in (3, 8, 16):
        assert any4.any4_matmul_workspace_size(M, N, K, G) == 0
    one = any4.any4_matmul_workspace_size(17, N, K, G)
    assert one > 0 and one == any4.any4_matmul_workspace_size(1023, N, K, G)
    assert one == any4.any4_matmul_workspace_size(300, 64, 64, 32)
    two = any4.any4_matmul_workspace_size(1024, N, K, G)
    assert two - one == ((N * K * 2 + 255) // 256) * 256
    # an explicit prefill path at small M still uses the one-pass size
    assert any4.any4_matmul_workspace_size(4, N, K, G, path="prefill") == one


def test_path_choice():
    assert any4.any4_matmul_choose_path(1, 4096, 4096, 128) == "decode"
    assert any4.any4_matmul_choose_path(16, 4096, 4096, 128) == "decode"
    assert any4.any4_matmul_choose_path(2048, 4096, 4096, 128) == "prefill"


def test_product_does_not_import_the_oracle():
    pkg = os.path.dirname(any4.__file__)
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "any4_oracle" not in text, fn


def test_bindings_refuse_host_tensors_and_wrong_dtypes():
    """The Python binding checks dtype and device before any library call; a
    host tensor is refused (there is no CPU path)."""
    import torch
    w = torch.zeros((4, 256), dtype=torch.bfloat16)
    ex = torch.zeros(256, dtype=torch.float32)
    idx = torch.zeros((4, 256), dtype=torch.uint8)
    for call in (lambda: any4.any4_quantize(w, ex, 64),
                 lambda: any4.any4_quantize_bits(w, ex, 64, 3),
                 lambda: any4.any4_pack_bits(idx, 3),
                 lambda: any4.any4_pack(idx)):
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
    with pytest.raises(TypeError):
        any4.any4_quantize(w.float(), ex, 64)
    with pytest.raises(TypeError):
        any4.any4_pack_bits(idx.to(torch.int32), 2)
    with pytest.raises(TypeError):
        any4.any4_dequant_bits(idx.float(), w, w, w, 64, 3)


def test_matmul_bindings_check_sizes_before_launch():
    """The C ABI sees bare pointers and cannot tell a short buffer; the Python
    matmul wrappers check every size against M, N, K and G before any library
    call, so an undersized y, scale, offset or dev_status never reaches a
    kernel (sizes are checked before the device, so host tensors show it)."""
    import torch
    M, N, K, G = 2, 16, 256, 64
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    packed = torch.zeros((N, K // 2), dtype=torch.uint8)
    lut = torch.zeros((N, 16), dtype=torch.bfloat16)
    so = torch.zeros((N, K // G), dtype=torch.bfloat16)
    short = torch.zeros((N, K // G - 1), dtype=torch.bfloat16)
    for fn in (any4.any4_matmul, any4.any4_matmul_static_scratch):
        with pytest.raises(ValueError, match="y must have shape"):
            fn(x, packed, lut, so, so, G, y=torch.zeros((M, N - 1), dtype=torch.bfloat16))
        with pytest.raises(ValueError, match="y must have shape"):
            fn(x, packed, lut, so, so, G, y=torch.zeros((M * N,), dtype=torch.bfloat16))
        with pytest.raises(ValueError, match="scale and offset"):
            fn(x, packed, lut, short, so, G)
        with pytest.raises(ValueError, match="scale and offset"):
            fn(x, packed, lut, so, short, G)
        with pytest.raises(ValueError, match="divide K"):
            fn(x, packed, lut, so, so, 96)
        with pytest.raises(ValueError, match="packed holds"):
            fn(x, packed[:, :64], lut, so, so, G)
        with pytest.raises(ValueError, match="lut must be"):
            fn(x, packed, lut[:8], so, so, G)
        with pytest.raises(ValueError, match="dev_status"):
            fn(x, packed, lut, so, so, G, y=torch.zeros((M, N), dtype=torch.bfloat16),
               dev_status=torch.zeros(0, dtype=torch.int32))
        # right sizes on host tensors: refused for the device, not the sizes
        with pytest.raises(ValueError, match="CUDA tensor"):
            fn(x, packed, lut, so, so, G)
    with pytest.raises(ValueError, match="packed must have shape"):
        any4.any4_pack(torch.zeros((N, K), dtype=torch.uint8),
                       packed=torch.zeros((N, K // 2 - 16), dtype=torch.uint8))


def _prefill_one_pass_bytes(slots):
    """The one-pass prefill workspace: one fp32 256 x 256 partial tile per
    block of the stream-K grid, then one flag word per block rounded up to
    256 bytes."""
    return slots * 256 * 256 * 4 + (slots * 4 + 255) // 256 * 256


def test_static_scratch_holds_a_148_sm_grid_and_no_more():
    """ANY4_STATIC_SCRATCH_BYTES covers the one-pass prefill workspace of a
    148-SM B200 and refuses a grid of one more block (the entry point then
    returns ANY4_ERR_WORKSPACE).  The library's own size (the SM count of the
    current device, or 160 blocks where there is no device) pins the formula."""
    import torch
    slots = (torch.cuda.get_device_properties(0).multi_processor_count
             if torch.cuda.is_available() else 160)
    assert any4.any4_matmul_workspace_size(16, 1024, 1024, 128, path="prefill") == \
        _prefill_one_pass_bytes(slots)
    assert _prefill_one_pass_bytes(148) <= any4.ANY4_STATIC_SCRATCH_BYTES
    assert _prefill_one_pass_bytes(149) > any4.ANY4_STATIC_SCRATCH_BYTES


def _grouped(items, M=1, K=128, G=32, x=FAKE, status=None, flags=0):
    arr = (_native.Any4Weight * max(1, len(items)))()
    for i, it in enumerate(items):
        arr[i] = _native.Any4Weight(**it)
    return _native.library().any4_matmul_grouped(x, arr, len(items), M, K, G, None, 0, status, 0,
                                                 flags, None)


def _item(**kw):
    d = dict(packed=FAKE, lut=FAKE, lut_row_stride=16, scale=FAKE, offset=FAKE, y=FAKE, N=64)
    d.update(kw)
    return d


def test_grouped_descriptor_layout_matches_header():
    # seven 8-byte fields, no padding: pointers, an int64 stride, pointers, int64 N
    assert ctypes.sizeof(_native.Any4Weight) == 56
    assert _native.Any4Weight.N.offset == 48
    text = open(os.path.join(HEADER_DIR, "any4.h")).read()
    assert f"#define ANY4_GROUP_MAX {any4.ANY4_GROUP_MAX}" in text


@pytest.mark.parametrize("items,kw,expect", [
    ([], {}, any4.ANY4_ERR_SHAPE),                                   # count 0
    ([_item()] * 5, {}, any4.ANY4_ERR_SHAPE),                        # above ANY4_GROUP_MAX
    ([_item(), _item(y=None)], {}, any4.ANY4_ERR_NULL),
    ([_item(), _item(N=0)], {}, any4.ANY4_ERR_SHAPE),
    ([_item(lut_row_stride=8)], {}, any4.ANY4_ERR_SHAPE),
    ([_item()], dict(K=100), any4.ANY4_ERR_SHAPE),
    ([_item(), _item(scale=FAKE + 2)], {}, any4.ANY4_ERR_ALIGN),
    ([_item()], dict(x=FAKE + 8), any4.ANY4_ERR_ALIGN),
    ([_item()], dict(x=None), any4.ANY4_ERR_NULL),
    ([_item()], dict(M=0), any4.ANY4_ERR_SHAPE),
    ([_item()], dict(flags=64), any4.ANY4_ERR_UNSUPPORTED),
    ([_item()], dict(status=FAKE + 2), any4.ANY4_ERR_ALIGN),
])
def test_grouped_rejects_bad_arguments(items, kw, expect):
    assert _grouped(items, **kw) == expect


def test_grouped_binding_checks_before_launch():
    import torch
    x = torch.zeros((1, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        any4.any4_matmul_grouped(x, [], 32)
    with pytest.raises((TypeError, ValueError)):
        any4.any4_matmul_grouped(x, [(torch.zeros((64, 64), dtype=torch.uint8),
                                      torch.zeros((64, 16), dtype=torch.bfloat16),
                                      torch.zeros((64, 4), dtype=torch.bfloat16),
                                      torch.zeros((64, 4), dtype=torch.bfloat16))], 32)


def _mbits(M=1, N=64, K=128, G=32, bits=3, x=FAKE, packed=FAKE, lut=FAKE, stride=8, scale=FAKE,
           offset=FAKE, y=FAKE, ws=None, ws_bytes=0, status=None, flags=0):
    return _native.library().any4_matmul_bits(x, packed, lut, stride, scale, offset, y, M, N, K,
                                              G, bits, ws, ws_bytes, status, flags, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(bits=1), any4.ANY4_ERR_SHAPE),
    (dict(bits=5), any4.ANY4_ERR_SHAPE),
    (dict(stride=16), any4.ANY4_ERR_SHAPE),          # 3 bits: 8 entries a row or 0
    (dict(bits=2, stride=8), any4.ANY4_ERR_SHAPE),   # 2 bits: 4 entries a row or 0
    (dict(K=100), any4.ANY4_ERR_SHAPE),
    (dict(M=0), any4.ANY4_ERR_SHAPE),
    (dict(x=None), any4.ANY4_ERR_NULL),
    (dict(y=FAKE + 4), any4.ANY4_ERR_ALIGN),
    (dict(flags=8), any4.ANY4_ERR_UNSUPPORTED),      # the pair-table flag is any4-only
    (dict(M=2), any4.ANY4_ERR_WORKSPACE),            # two passes need the workspace
    (dict(M=1, K=1056, G=32), any4.ANY4_ERR_WORKSPACE),
])
def test_matmul_bits_rejects_bad_arguments(kw, expect):
    assert _mbits(**kw) == expect


def test_matmul_bits_workspace_sizes():
    ws = any4.any4_matmul_bits_workspace_size
    # M = 1 on the weight-streaming kernel's shapes: none
    assert ws(1, 4096, 4096, 128, 3) == 0 and ws(1, 4096, 4096, 64, 2) == 0
    # otherwise the two-pass workspace, the same as any4's large-M path
    two = any4.any4_matmul_workspace_size(2048, 4096, 4096, 128)
    assert ws(2, 4096, 4096, 128, 3) == two and ws(2048, 4096, 4096, 128, 2) == two
    assert ws(1, 4096, 1056, 32, 3) == any4.any4_matmul_workspace_size(2048, 4096, 1056, 32)
    assert ws(1, 4096, 4096, 256, 3) > 0
    assert ws(1, 4096, 4096, 128, 4) == any4.any4_matmul_workspace_size(1, 4096, 4096, 128)
    assert ws(1, 4096, 4096, 128, 5) == 0 and ws(0, 4096, 4096, 128, 3) == 0


def test_prepare_checks_the_weights_once():
    """any4_prepare checks a matrix's sizes, dtypes and device up front (sizes
    first, so host tensors show them); a host matrix is refused."""
    import torch
    N, K, G = 16, 256, 64
    packed = torch.zeros((N, K // 2), dtype=torch.uint8)
    lut = torch.zeros((N, 16), dtype=torch.bfloat16)
    so = torch.zeros((N, K // G), dtype=torch.bfloat16)
    short = torch.zeros((N, K // G - 1), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="scale and offset"):
        any4.any4_prepare(packed, lut, short, so, G)
    with pytest.raises(ValueError, match="divide K"):
        any4.any4_prepare(packed, lut, so, so, 96)
    with pytest.raises(ValueError, match="lut must be"):
        any4.any4_prepare(packed, lut[:8], so, so, G)
    with pytest.raises(TypeError):
        any4.any4_prepare(packed.to(torch.int32), lut, so, so, G)
    with pytest.raises(TypeError):
        any4.any4_prepare(packed, lut.float(), so, so, G)
    with pytest.raises(ValueError, match="CUDA tensor"):
        any4.any4_prepare(packed, lut, so, so, G)


def test_prepared_group_cache_keeps_no_weights_alive():
    """The binding caches each group of prepared weights' descriptor array,
    but must not keep the weights (and their device tensors) alive."""
    import gc
    import weakref
    import torch
    ws = []
    for n in (8, 16):
        w = object.__new__(_native.Any4Prepared)   # host stand-ins: no CUDA needed
        w.packed = torch.zeros((n, 512), dtype=torch.uint8)
        w.lut = w.scale = w.offset = None
        w.G, w.N, w.K, w.lut_row_stride = 128, n, 1024, 16
        w.device, w.decode_layout, w._ptrs = w.packed.device, False, (0, 0, 0, 0)
        ws.append(w)
    g = _native._prepared_group(ws)
    assert g is _native._prepared_group(ws)          # a hit the second time
    refs = [weakref.ref(w) for w in ws]
    del ws, g, w  # (w: the loop variable still names the last one)
    gc.collect()
    assert all(r() is None for r in refs)
