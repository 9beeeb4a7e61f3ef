"""ctypes binding of libany4.so (argument marshalling only).

Each wrapper checks tensor dtypes/devices/contiguity, passes raw pointers and
sizes to the C entry point of the same name, on torch's current CUDA stream,
and raises Any4Error on a non-zero status.  Outputs are allocated with torch
when not supplied.
"""
from __future__ import annotations

import ctypes
import os
import threading
import weakref

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libany4.so")

ANY4_OK = 0
ANY4_ERR_NULL = -1
ANY4_ERR_SHAPE = -2
ANY4_ERR_ALIGN = -3
ANY4_ERR_RANGE = -4
ANY4_ERR_CUDA = -5
ANY4_ERR_TIMEOUT = -6
ANY4_ERR_UNSUPPORTED = -7
ANY4_ERR_WORKSPACE = -8

PATHS = {"auto": 0, "decode": 1, "prefill": 2}
# Bytes of the library's fixed scratch array (any4_matmul_static_scratch).
ANY4_STATIC_SCRATCH_BYTES = 148 * 262144 + 1024
ANY4_FLAG_OVERLAP_PRIOR = 1
ANY4_FLAG_FP32_OUT = 2
ANY4_FLAG_TEST_STALL = 4
ANY4_FLAG_PAIR_TABLE = 8
ANY4_FLAG_DECODE_LAYOUT = 16
# Limits of any4_quantize (the row lives in one block's shared memory).
ANY4_QUANTIZE_MAX_K = 16384
ANY4_QUANTIZE_MAX_ITER = 100000

_lib = None


class Any4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: any4 status {status} ({any4_status_string(status)})")


class Any4Weight(ctypes.Structure):
    """any4_weight of include/any4.h: one matrix of any4_matmul_grouped."""
    _fields_ = [("packed", ctypes.c_void_p), ("lut", ctypes.c_void_p),
                ("lut_row_stride", ctypes.c_int64), ("scale", ctypes.c_void_p),
                ("offset", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int64)]


ANY4_GROUP_MAX = 4


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """Load libany4.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m learned_bit_lut_any4_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.any4_pack.argtypes = [vp, vp, i64, i64, vp, vp]
    lib.any4_pack.restype = i32
    lib.any4_repack.argtypes = [vp, vp, i64, i64, vp]
    lib.any4_repack.restype = i32
    lib.any4_quantize.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp]
    lib.any4_quantize.restype = i32
    lib.any4_quantize_bits.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.any4_quantize_bits.restype = i32
    lib.any4_pack_bits.argtypes = [vp, vp, i64, i64, i32, vp, vp]
    lib.any4_pack_bits.restype = i32
    lib.any4_dequant_bits.argtypes = [vp, vp, i64, vp, vp, vp, i64, i64, i64, i32, vp]
    lib.any4_dequant_bits.restype = i32
    lib.any4_dequant.argtypes = [vp, vp, i64, vp, vp, vp, i64, i64, i64, vp]
    lib.any4_dequant.restype = i32
    lib.any4_matmul.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64, vp, sz, vp, vp]
    lib.any4_matmul.restype = i32
    lib.any4_matmul_ex.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64, vp, sz, vp,
                                   i32, ctypes.c_uint32, vp]
    lib.any4_matmul_ex.restype = i32
    lib.any4_matmul_static_scratch.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64,
                                               vp, vp]
    lib.any4_matmul_static_scratch.restype = i32
    lib.any4_matmul_workspace_size.argtypes = [i64, i64, i64, i64]
    lib.any4_matmul_workspace_size.restype = sz
    lib.any4_matmul_workspace_size_ex.argtypes = [i64, i64, i64, i64, i32]
    lib.any4_matmul_workspace_size_ex.restype = sz
    lib.any4_matmul_choose_path.argtypes = [i64, i64, i64, i64]
    lib.any4_matmul_choose_path.restype = i32
    lib.any4_status_string.argtypes = [i32]
    lib.any4_status_string.restype = ctypes.c_char_p
    lib.any4_matmul_grouped.argtypes = [vp, ctypes.POINTER(Any4Weight), i32, i64, i64, i64, vp,
                                        sz, vp, i32, ctypes.c_uint32, vp]
    lib.any4_matmul_grouped.restype = i32
    lib.any4_matmul_bits.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64, i32, vp,
                                     sz, vp, ctypes.c_uint32, vp]
    lib.any4_matmul_bits.restype = i32
    lib.any4_matmul_bits_workspace_size.argtypes = [i64, i64, i64, i64, i32]
    lib.any4_matmul_bits_workspace_size.restype = sz
    lib.any4_group_sums.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.any4_group_sums.restype = i32
    lib.any4_read_probe.argtypes = [vp, i64, vp, vp]
    lib.any4_read_probe.restype = i32
    lib.any4_bits_per_weight.argtypes = [i64, i64]
    lib.any4_bits_per_weight.restype = ctypes.c_double
    lib.any4_version.argtypes = []
    lib.any4_version.restype = i32
    _lib = lib
    return lib


def any4_status_string(status: int) -> str:
    return library().any4_status_string(int(status)).decode()


def any4_version() -> int:
    return int(library().any4_version())


def any4_bits_per_weight(K: int, G: int) -> float:
    return float(library().any4_bits_per_weight(K, G))


# workspace bytes per (device, M, N, K, G, path), asked of the library once
_WS_NEED: dict = {}


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_NULL_CTX = _NullCtx()


def _on_device(dev: torch.device):
    """torch.cuda.device(dev), skipped when dev is already the current device
    (the C entry points act on the current device)."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return _NULL_CTX
    return torch.cuda.device(dev)


def _check(status: int, where: str):
    if status != ANY4_OK:
        raise Any4Error(status, where)


_RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _stream_index(index: int) -> int:
    """The current stream's handle on device `index` (torch's raw-handle
    accessor where it has one: no Stream object per call)."""
    if _RAW_STREAM is not None:
        return _RAW_STREAM(index)
    return torch.cuda.current_stream(index).cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtypes, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def any4_pack(idx: torch.Tensor, packed: torch.Tensor | None = None,
              dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """uint8 codes [N, K] (values 0..15) -> uint8 packed [N, K/2] (low nibble = even k).

    A code above 15 sets ANY4_ERR_RANGE in dev_status (int32 CUDA tensor of one
    element, zeroed by the caller) once the stream has run."""
    if not isinstance(idx, torch.Tensor) or idx.dim() != 2:
        raise ValueError("idx must be a [N, K] tensor")
    N, K = idx.shape
    if packed is not None:
        _need_shape(packed, "packed", (N, K // 2))
    _need(idx, "idx", (torch.uint8,))
    if packed is None:
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device=idx.device)
    _need(packed, "packed", (torch.uint8,), idx.device)
    _need_status(dev_status, idx.device)
    with torch.cuda.device(idx.device):
        _check(library().any4_pack(_ptr(idx), _ptr(packed), N, K, _ptr(dev_status),
                                   _stream(idx.device)), "any4_pack")
    return packed


def any4_repack(packed: torch.Tensor, repacked: torch.Tensor | None = None) -> torch.Tensor:
    """uint8 packed [N, K/2] (any4_pack's layout) -> the same codes in the M = 1
    decode kernel's layout (see any4_repack in include/any4.h); K a multiple of
    1024.  Use the result with decode_layout=True (M = 1, G = 128 only)."""
    if not isinstance(packed, torch.Tensor) or packed.dim() != 2:
        raise ValueError("packed must be a [N, K/2] tensor")
    N, Kh = packed.shape
    if (2 * Kh) % 1024 != 0 or Kh == 0:
        raise ValueError(f"K = {2 * Kh} must be a positive multiple of 1024")
    if repacked is not None:
        _need_shape(repacked, "repacked", (N, Kh))
    _need(packed, "packed", (torch.uint8,))
    if repacked is None:
        repacked = torch.empty_like(packed)
    _need(repacked, "repacked", (torch.uint8,), packed.device)
    with torch.cuda.device(packed.device):
        _check(library().any4_repack(_ptr(packed), _ptr(repacked), N, 2 * Kh,
                                     _stream(packed.device)), "any4_repack")
    return repacked


def any4_quantize(w: torch.Tensor, ex_abs: torch.Tensor, G: int, max_iter: int = 100,
                  return_iters: bool = False):
    """Learn the any4 representation of a bf16 weight w [N, K]: group scaling,
    then a weighted k-means per row with sample weight alpha * E|x| (ex_abs,
    fp32 [K], finite and >= 0).  Returns (packed [N, K/2] uint8, lut [N, 16],
    scale [N, K/G], offset [N, K/G]) in bf16, plus the int32 M-steps per row
    when return_iters."""
    _need(w, "w", _BF16)
    dev = w.device
    _need(ex_abs, "ex_abs", (torch.float32,), dev)
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    if ex_abs.numel() != K:
        raise ValueError(f"ex_abs must hold K={K} values")
    ng = K // G if G > 0 else 0
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    lut = torch.empty((N, 16), dtype=torch.bfloat16, device=dev)
    scale = torch.empty((N, ng), dtype=torch.bfloat16, device=dev)
    offset = torch.empty((N, ng), dtype=torch.bfloat16, device=dev)
    iters = torch.empty(N, dtype=torch.int32, device=dev) if return_iters else None
    with _on_device(dev):
        _check(library().any4_quantize(_ptr(w), _ptr(ex_abs), N, K, G, int(max_iter),
                                       _ptr(packed), _ptr(lut), _ptr(scale), _ptr(offset),
                                       _ptr(iters), _stream(dev)), "any4_quantize")
    if return_iters:
        return packed, lut, scale, offset, iters
    return packed, lut, scale, offset


def any4_quantize_bits(w: torch.Tensor, ex_abs: torch.Tensor, G: int, bits: int,
                       max_iter: int = 100, return_iters: bool = False):
    """any4_quantize with 2^bits table entries (bits 2, 3 or 4): packed
    [N, bits*K/8] uint8 (one little-endian bit stream per row), lut [N, 2^bits],
    scale and offset [N, K/G] in bf16 (+ int32 M-steps per row)."""
    _need(w, "w", _BF16)
    dev = w.device
    _need(ex_abs, "ex_abs", (torch.float32,), dev)
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    if ex_abs.numel() != K:
        raise ValueError(f"ex_abs must hold K={K} values")
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    ng = K // G if G > 0 else 0
    packed = torch.empty((N, bits * K // 8), dtype=torch.uint8, device=dev)
    lut = torch.empty((N, 1 << bits), dtype=torch.bfloat16, device=dev)
    scale = torch.empty((N, ng), dtype=torch.bfloat16, device=dev)
    offset = torch.empty((N, ng), dtype=torch.bfloat16, device=dev)
    iters = torch.empty(N, dtype=torch.int32, device=dev) if return_iters else None
    with _on_device(dev):
        _check(library().any4_quantize_bits(_ptr(w), _ptr(ex_abs), N, K, G, bits, int(max_iter),
                                            _ptr(packed), _ptr(lut), _ptr(scale), _ptr(offset),
                                            _ptr(iters), _stream(dev)), "any4_quantize_bits")
    if return_iters:
        return packed, lut, scale, offset, iters
    return packed, lut, scale, offset


def any4_pack_bits(idx: torch.Tensor, bits: int, packed: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """uint8 codes [N, K] (0 .. 2^bits - 1) -> packed [N, bits*K/8]: one
    little-endian bit stream per row, code k in bits [bits*k, bits*k + bits)."""
    _need(idx, "idx", (torch.uint8,))
    N, K = idx.shape
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    if packed is None:
        packed = torch.empty((N, bits * K // 8), dtype=torch.uint8, device=idx.device)
    _need(packed, "packed", (torch.uint8,), idx.device)
    _need_shape(packed, "packed", (N, bits * K // 8))
    _need_status(dev_status, idx.device)
    with _on_device(idx.device):
        _check(library().any4_pack_bits(_ptr(idx), _ptr(packed), N, K, bits, _ptr(dev_status),
                                        _stream(idx.device)), "any4_pack_bits")
    return packed


def any4_dequant_bits(packed: torch.Tensor, lut: torch.Tensor, scale: torch.Tensor,
                      offset: torch.Tensor, G: int, bits: int,
                      W: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 W[N, K] from n-bit codes; lut is [N, 2^bits] or [2^bits] (one table)."""
    _need(packed, "packed", (torch.uint8,))
    dev = packed.device
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    N, nb = packed.shape
    K = nb * 8 // bits
    nq = 1 << bits
    for t, nm in ((lut, "lut"), (scale, "scale"), (offset, "offset")):
        _need(t, nm, _BF16, dev)
    if lut.dim() == 1 and lut.numel() == nq:
        stride = 0
    elif lut.dim() == 2 and tuple(lut.shape) == (N, nq):
        stride = nq
    else:
        raise ValueError(f"lut must be [N, {nq}] or [{nq}], got {tuple(lut.shape)}")
    if W is None:
        W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    _need(W, "W", _BF16, dev)
    _need_shape(W, "W", (N, K))
    if scale.numel() != N * (K // G if G else 0) or offset.numel() != scale.numel():
        raise ValueError("scale and offset must hold N * K/G values")
    with _on_device(dev):
        _check(library().any4_dequant_bits(_ptr(packed), _ptr(lut), stride, _ptr(scale),
                                           _ptr(offset), _ptr(W), N, K, G, bits, _stream(dev)),
               "any4_dequant_bits")
    return W


def _need_shape(t: torch.Tensor, name: str, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_status(dev_status, dev):
    """dev_status: None, or an int32 CUDA tensor of at least one element."""
    if dev_status is None:
        return
    if isinstance(dev_status, torch.Tensor) and dev_status.numel() < 1:
        raise ValueError("dev_status must hold at least one int32")
    _need(dev_status, "dev_status", (torch.int32,), dev)


def _weight_operands(packed, lut, scale, offset, G, K=None, bits=4):
    """Check one matrix's packed codes, table, scales and offsets (types and
    sizes; devices and layout by the caller).  Returns (N, K, lut_row_stride)."""
    for t, nm, dts in ((packed, "packed", (torch.uint8,)), (lut, "lut", _BF16),
                       (scale, "scale", _BF16), (offset, "offset", _BF16)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{nm} must be a torch.Tensor")
        if t.dtype not in dts:
            raise TypeError(f"{nm} must have dtype in {dts}, got {t.dtype}")
    if packed.dim() != 2:
        raise ValueError(f"packed must be [N, {bits} K / 8]")
    N, Kh = packed.shape
    if K is None:
        if (Kh * 8) % bits != 0:
            raise ValueError(f"packed rows of {Kh} bytes do not hold whole {bits}-bit codes")
        K = Kh * 8 // bits
    elif Kh * 8 != K * bits:
        raise ValueError(f"x has K={K} but packed holds {Kh * 8 // bits} {bits}-bit columns")
    if G <= 0 or K % G != 0:
        raise ValueError(f"G={G} must be positive and divide K={K}")
    stride = _lut_stride(lut, N, 1 << bits)
    if scale.numel() != N * (K // G) or offset.numel() != N * (K // G):
        raise ValueError(f"scale and offset must hold N * K/G = {N * (K // G)} values")
    return N, K, stride


def _matmul_operands(x, packed, lut, scale, offset, G, y, dev_status=None, fp32_out=False,
                     bits=4):
    """Validate the operands of a matmul call on the host, before any launch:
    the C ABI sees bare pointers and cannot check that a buffer is large
    enough, so a short y, scale or offset is caught here.  Sizes are checked
    before devices, so the checks hold for any tensor.  Returns
    (M, N, K, lut_row_stride, y), allocating y when it is None."""
    if not isinstance(x, torch.Tensor):
        raise TypeError("x must be a torch.Tensor")
    if x.dtype not in _BF16:
        raise TypeError(f"x must have dtype in {_BF16}, got {x.dtype}")
    if x.dim() != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    N, K, stride = _weight_operands(packed, lut, scale, offset, G, K, bits)
    if y is not None:
        _need_shape(y, "y", (M, N))
    if isinstance(dev_status, torch.Tensor) and dev_status.numel() < 1:
        raise ValueError("dev_status must hold at least one int32")
    dev = x.device
    _need(x, "x", _BF16)
    _need(packed, "packed", (torch.uint8,), dev)
    for t, nm in ((lut, "lut"), (scale, "scale"), (offset, "offset")):
        _need(t, nm, _BF16, dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32 if fp32_out else torch.bfloat16, device=dev)
    _need(y, "y", (torch.float32,) if fp32_out else _BF16, dev)
    return M, N, K, stride, y


class Any4Prepared:
    """One any4 matrix checked once, for repeated matmul calls (a decode loop).

    any4_prepare checks the packed codes, table, scales and offsets (dtypes,
    sizes, device, contiguity) and keeps them; any4_matmul and
    any4_matmul_grouped take it in place of those four tensors and then check
    only x, y and the workspace, which keeps the host cost of a call small.
    The tensors must stay as they are (not resized, not moved) while it is in
    use."""
    __slots__ = ("packed", "lut", "scale", "offset", "G", "N", "K", "lut_row_stride",
                 "device", "decode_layout", "_ptrs", "__weakref__")

    def __init__(self, packed, lut, scale, offset, G, decode_layout=False):
        N, K, stride = _weight_operands(packed, lut, scale, offset, G)
        if decode_layout and (G != 128 or K % 1024 != 0):
            raise ValueError("the decode layout needs G = 128 and K a multiple of 1024")
        dev = packed.device
        _need(packed, "packed", (torch.uint8,))
        for t, nm in ((lut, "lut"), (scale, "scale"), (offset, "offset")):
            _need(t, nm, _BF16, dev)
        self.packed, self.lut, self.scale, self.offset = packed, lut, scale, offset
        self.G, self.N, self.K, self.lut_row_stride = int(G), int(N), int(K), stride
        self.device = dev
        self.decode_layout = bool(decode_layout)
        self._ptrs = (packed.data_ptr(), lut.data_ptr(), scale.data_ptr(), offset.data_ptr())

    def __repr__(self):
        return f"Any4Prepared(N={self.N}, K={self.K}, G={self.G}, device={self.device})"


def any4_prepare(packed: torch.Tensor, lut: torch.Tensor, scale: torch.Tensor,
                 offset: torch.Tensor, G: int, decode_layout: bool = False) -> Any4Prepared:
    """Check an any4 matrix once for repeated calls (see Any4Prepared);
    decode_layout: packed comes from any4_repack."""
    return Any4Prepared(packed, lut, scale, offset, G, decode_layout)


# Per thread: the ctypes descriptor array of each group of prepared weights
# used in a call (only the y pointers change from call to call), and the
# workspace each needs per M.  Entries are keyed by the objects' ids and hold
# only weak references to them, so the cache keeps no weights alive; an entry
# whose objects are gone (an id reused by a new object) is rebuilt.
_PREPARED_GROUPS = threading.local()
_PREPARED_GROUPS_MAX = 4096


def _prepared_group(weights):
    cache = getattr(_PREPARED_GROUPS, "d", None)
    if cache is None:
        cache = _PREPARED_GROUPS.d = {}
    key = tuple(map(id, weights))
    g = cache.get(key)
    if g is not None:
        for r, w in zip(g[7], weights):
            if r() is not w:
                break
        else:
            return g
    w0 = weights[0]
    for w in weights:
        if not isinstance(w, Any4Prepared):
            raise TypeError("mix of prepared and plain weights in one call")
        if (w.device != w0.device or w.K != w0.K or w.G != w0.G
                or w.decode_layout != w0.decode_layout):
            raise ValueError("prepared weights of one call must share device, K, G and "
                             "code layout")
    descs = (Any4Weight * len(weights))()
    for i, w in enumerate(weights):
        pk, lt, sc, of = w._ptrs
        descs[i] = Any4Weight(pk, lt, w.lut_row_stride, sc, of, 0, w.N)
    if len(cache) >= _PREPARED_GROUPS_MAX:
        cache.clear()
    di = w0.device.index if w0.device.index is not None else -1
    g = cache[key] = [descs, w0.K, w0.G, w0.device, di, {}, w0.decode_layout,
                      tuple(weakref.ref(w) for w in weights)]
    return g


def _prepared_x(x, K, dev_index):
    """Check x of a call on prepared weights (K columns, on device dev_index);
    returns M."""
    if not isinstance(x, torch.Tensor) or x.dtype not in _BF16:
        raise TypeError("x must be a bf16 torch.Tensor")
    if x.get_device() != dev_index:
        raise ValueError(f"x must be on cuda:{dev_index}, the device of the weights")
    shape = x.shape
    if len(shape) != 2 or shape[1] != K:
        raise ValueError(f"x must be [M, {K}], got {tuple(shape)}")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    return shape[0]


def _prepared_y(y, M, N, dev_index, fp32_out):
    dts = (torch.float32,) if fp32_out else _BF16
    if not isinstance(y, torch.Tensor) or y.dtype not in dts:
        raise TypeError(f"y must be a torch.Tensor with dtype in {dts}")
    if y.get_device() != dev_index:
        raise ValueError(f"y must be on cuda:{dev_index}, the device of the weights")
    if tuple(y.shape) != (M, N):
        raise ValueError(f"y must have shape {(M, N)}, got {tuple(y.shape)}")
    if not y.is_contiguous():
        raise ValueError("y must be contiguous")


def _lut_stride(lut: torch.Tensor, N: int, entries: int = 16) -> int:
    if lut.dim() == 1 and lut.numel() == entries:
        return 0
    if lut.dim() == 2 and tuple(lut.shape) == (N, entries):
        return entries
    raise ValueError(f"lut must be [N, {entries}] or [{entries}], got {tuple(lut.shape)}")


def any4_dequant(packed: torch.Tensor, lut: torch.Tensor, scale: torch.Tensor,
                 offset: torch.Tensor, G: int, W: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 W[N, K] = bf16(fmaf(LUT[n][code], scale[n][k/G], offset[n][k/G]))."""
    _need(packed, "packed", (torch.uint8,))
    dev = packed.device
    N, Kh = packed.shape
    K = 2 * Kh
    for t, nm in ((lut, "lut"), (scale, "scale"), (offset, "offset")):
        _need(t, nm, _BF16, dev)
    stride = _lut_stride(lut, N)
    if W is None:
        W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    _need(W, "W", _BF16, dev)
    _need_shape(W, "W", (N, K))
    if scale.numel() != N * (K // G if G else 0) or offset.numel() != scale.numel():
        raise ValueError("scale and offset must hold N * K/G values")
    with _on_device(dev):
        _check(library().any4_dequant(_ptr(packed), _ptr(lut), stride, _ptr(scale),
                                      _ptr(offset), _ptr(W), N, K, G, _stream(dev)),
               "any4_dequant")
    return W


def any4_group_sums(x: torch.Tensor, G: int, xsum: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 xsum[M, K/G]: the sum of x[m, k] over each group of G columns."""
    _need(x, "x", _BF16)
    if x.dim() != 2:
        raise ValueError("x must be [M, K]")
    dev = x.device
    M, K = x.shape
    if G < 1 or K % G:
        raise ValueError("K must be a multiple of G")
    if xsum is None:
        xsum = torch.empty((M, K // G), dtype=torch.float32, device=dev)
    _need(xsum, "xsum", (torch.float32,), dev)
    _need_shape(xsum, "xsum", (M, K // G))
    with _on_device(dev):
        _check(library().any4_group_sums(_ptr(x), _ptr(xsum), M, K, G, _stream(dev)),
               "any4_group_sums")
    return xsum


def any4_read_probe(buf: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """A read-only stream over buf (a contiguous CUDA tensor of a multiple of
    16 bytes): returns a one-element int32 tensor holding the XOR of its 32-bit
    words.  Timed, it measures the HBM read bandwidth that bounds the decode
    matmuls."""
    if not isinstance(buf, torch.Tensor) or not buf.is_cuda:
        raise ValueError("buf must be a CUDA tensor")
    if not buf.is_contiguous():
        raise ValueError("buf must be contiguous")
    dev = buf.device
    nbytes = buf.numel() * buf.element_size()
    if nbytes % 16:
        raise ValueError(f"buf holds {nbytes} bytes, not a multiple of 16")
    if out is None:
        out = torch.empty(1, dtype=torch.int32, device=dev)
    _need(out, "out", (torch.int32,), dev)
    if out.numel() < 1:
        raise ValueError("out must hold one int32")
    with _on_device(dev):
        _check(library().any4_read_probe(_ptr(buf) if nbytes else None, nbytes, _ptr(out),
                                         _stream(dev)), "any4_read_probe")
    return out


def any4_matmul_workspace_size(M: int, N: int, K: int, G: int, path: str = "auto") -> int:
    return int(library().any4_matmul_workspace_size_ex(M, N, K, G, PATHS[path]))


def any4_matmul_choose_path(M: int, N: int, K: int, G: int) -> str:
    code = int(library().any4_matmul_choose_path(M, N, K, G))
    return {v: k for k, v in PATHS.items()}[code]


def any4_matmul(x: torch.Tensor, packed: torch.Tensor, lut: torch.Tensor,
                scale: torch.Tensor, offset: torch.Tensor, G: int,
                y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                path: str = "auto", dev_status: torch.Tensor | None = None,
                overlap_prior: bool = False, fp32_out: bool = False,
                test_stall: bool = False, pair_table: bool = False,
                decode_layout: bool = False) -> torch.Tensor:
    """bf16 y[M, N] = x[M, K] * dequant(W)^T, fp32 accumulation.

    workspace: a CUDA tensor of at least any4_matmul_workspace_size() bytes, or
    None to have one allocated here when the path needs it (an empty tensor
    passes none: the decode path then runs its kernels that need none).
    overlap_prior: ANY4_FLAG_OVERLAP_PRIOR (the weights are not written by
    work still running on the stream; the decode kernel may then overlap it).
    fp32_out: ANY4_FLAG_FP32_OUT, y is fp32 and holds the sums unrounded.
    test_stall: ANY4_FLAG_TEST_STALL, a test of the failure handling (one
    block's stream stops, the call ends with ANY4_ERR_TIMEOUT in dev_status).
    pair_table: ANY4_FLAG_PAIR_TABLE, M = 1 on the pair-table kernel (needs
    the workspace) instead of the weight-streaming kernel.
    decode_layout: ANY4_FLAG_DECODE_LAYOUT, packed comes from any4_repack
    (M = 1, G = 128 only)."""
    M, N, K, stride, y = _matmul_operands(x, packed, lut, scale, offset, G, y,
                                             dev_status, fp32_out)
    dev = x.device
    lib = library()
    p = PATHS[path]
    key = (dev.index, M, N, K, G, p)
    need = _WS_NEED.get(key)
    if need is None:
        need = _WS_NEED[key] = int(lib.any4_matmul_workspace_size_ex(M, N, K, G, p))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", (torch.uint8,), dev)
        ws_bytes = workspace.numel()
        if ws_bytes == 0:
            workspace = None
    _need_status(dev_status, dev)
    with _on_device(dev):
        _check(lib.any4_matmul_ex(_ptr(x), _ptr(packed), _ptr(lut), stride, _ptr(scale),
                                  _ptr(offset), _ptr(y), M, N, K, G, _ptr(workspace), ws_bytes,
                                  _ptr(dev_status), p,
                                  (ANY4_FLAG_OVERLAP_PRIOR if overlap_prior else 0)
                                  | (ANY4_FLAG_FP32_OUT if fp32_out else 0)
                                  | (ANY4_FLAG_TEST_STALL if test_stall else 0)
                                  | (ANY4_FLAG_PAIR_TABLE if pair_table else 0)
                                  | (ANY4_FLAG_DECODE_LAYOUT if decode_layout else 0),
                                  _stream(dev)), "any4_matmul")
    return y


def any4_matmul_bits_workspace_size(M: int, N: int, K: int, G: int, bits: int) -> int:
    return int(library().any4_matmul_bits_workspace_size(M, N, K, G, bits))


def any4_matmul_bits(x: torch.Tensor, packed: torch.Tensor, lut: torch.Tensor,
                     scale: torch.Tensor, offset: torch.Tensor, G: int, bits: int,
                     y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None, overlap_prior: bool = False,
                     fp32_out: bool = False, test_stall: bool = False) -> torch.Tensor:
    """y[M, N] = x * dequant(W)^T for n-bit codes (any4_pack_bits layout; lut
    [N, 2^bits] or [2^bits]).  bits = 4 is any4_matmul."""
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    M, N, K, stride, y = _matmul_operands(x, packed, lut, scale, offset, G, y, dev_status,
                                          fp32_out, bits)
    dev = x.device
    lib = library()
    need = int(lib.any4_matmul_bits_workspace_size(M, N, K, G, bits))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", (torch.uint8,), dev)
        ws_bytes = workspace.numel()
        if ws_bytes == 0:
            workspace = None
    _need_status(dev_status, dev)
    with _on_device(dev):
        _check(lib.any4_matmul_bits(_ptr(x), _ptr(packed), _ptr(lut), stride, _ptr(scale),
                                    _ptr(offset), _ptr(y), M, N, K, G, bits, _ptr(workspace),
                                    ws_bytes, _ptr(dev_status),
                                    (ANY4_FLAG_OVERLAP_PRIOR if overlap_prior else 0)
                                    | (ANY4_FLAG_FP32_OUT if fp32_out else 0)
                                    | (ANY4_FLAG_TEST_STALL if test_stall else 0),
                                    _stream(dev)), "any4_matmul_bits")
    return y


def any4_matmul_grouped(x: torch.Tensor, weights, G: int, ys=None,
                        workspace: torch.Tensor | None = None, path: str = "auto",
                        dev_status: torch.Tensor | None = None, overlap_prior: bool = False,
                        fp32_out: bool = False, test_stall: bool = False,
                        pair_table: bool = False, decode_layout: bool = False):
    """[y_i = x * dequant(W_i)^T for each (packed, lut, scale, offset) in
    weights]: matrices that share x, in one launch at M = 1 (see
    any4_matmul_grouped in include/any4.h).  Returns the list of y_i.  The
    entries may instead all be Any4Prepared (any4_prepare): then only x, the
    y's and the workspace are checked per call, and their decode_layout
    (any4_repack'd codes) applies.  decode_layout: the plain entries' packed
    come from any4_repack (M = 1, G = 128 only)."""
    weights = list(weights)
    if not 1 <= len(weights) <= ANY4_GROUP_MAX:
        raise ValueError(f"between 1 and {ANY4_GROUP_MAX} matrices")
    if ys is not None and len(ys) != len(weights):
        raise ValueError("one y per matrix")
    outs = []
    M = K = None
    need_ws = 0
    lib = library()
    p = PATHS[path]
    if isinstance(weights[0], Any4Prepared):
        # prepared weights: only x, the y's and the workspace are checked here
        descs, K, Gp, dev, di, ws_need, dl, _refs = _prepared_group(weights)
        if G != Gp:
            raise ValueError(f"G={G} but the weights were prepared with G={Gp}")
        M = _prepared_x(x, K, di)
        for i, w in enumerate(weights):
            if ys is None:
                y = torch.empty((M, w.N), dtype=torch.float32 if fp32_out else torch.bfloat16,
                                device=dev)
            else:
                y = ys[i]
                _prepared_y(y, M, w.N, di, fp32_out)
            outs.append(y)
            descs[i].y = y.data_ptr()
        need_ws = ws_need.get((M, p))
        if need_ws is None:
            need_ws = ws_need[(M, p)] = max(
                int(lib.any4_matmul_workspace_size_ex(M, w.N, K, G, p)) for w in weights)
        if workspace is None and need_ws > 0:
            workspace = torch.empty(need_ws, dtype=torch.uint8, device=dev)
        ws_bytes = 0
        if workspace is not None:
            if (not isinstance(workspace, torch.Tensor) or workspace.dtype != torch.uint8
                    or workspace.get_device() != di or not workspace.is_contiguous()):
                raise ValueError(f"workspace must be a contiguous uint8 tensor on cuda:{di}")
            ws_bytes = workspace.numel()
            if ws_bytes == 0:
                workspace = None
        _need_status(dev_status, dev)
        st = _stream_index(di)
        with _on_device(dev):
            _check(lib.any4_matmul_grouped(x.data_ptr(), descs, len(weights), M, K, G,
                                           _ptr(workspace), ws_bytes, _ptr(dev_status), p,
                                           (ANY4_FLAG_OVERLAP_PRIOR if overlap_prior else 0)
                                           | (ANY4_FLAG_FP32_OUT if fp32_out else 0)
                                           | (ANY4_FLAG_TEST_STALL if test_stall else 0)
                                           | (ANY4_FLAG_PAIR_TABLE if pair_table else 0)
                                           | (ANY4_FLAG_DECODE_LAYOUT if dl else 0),
                                           st), "any4_matmul_grouped")
        return outs
    descs = (Any4Weight * len(weights))()
    for i, wt in enumerate(weights):
        if isinstance(wt, Any4Prepared):
            raise TypeError("mix of prepared and plain weights in one call")
        packed, lut, scale, offset = wt
        y = None if ys is None else ys[i]
        M, N, K, stride, y = _matmul_operands(x, packed, lut, scale, offset, G, y,
                                              dev_status, fp32_out)
        outs.append(y)
        descs[i] = Any4Weight(_ptr(packed), _ptr(lut), stride, _ptr(scale), _ptr(offset),
                              _ptr(y), N)
        need_ws = max(need_ws, int(lib.any4_matmul_workspace_size_ex(M, N, K, G, p)))
    dev = x.device
    if workspace is None and need_ws > 0:
        workspace = torch.empty(need_ws, dtype=torch.uint8, device=dev)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", (torch.uint8,), dev)
        ws_bytes = workspace.numel()
        if ws_bytes == 0:
            workspace = None
    _need_status(dev_status, dev)
    with _on_device(dev):
        _check(lib.any4_matmul_grouped(_ptr(x), descs, len(weights), M, K, G, _ptr(workspace),
                                       ws_bytes, _ptr(dev_status), p,
                                       (ANY4_FLAG_OVERLAP_PRIOR if overlap_prior else 0)
                                       | (ANY4_FLAG_FP32_OUT if fp32_out else 0)
                                       | (ANY4_FLAG_TEST_STALL if test_stall else 0)
                                       | (ANY4_FLAG_PAIR_TABLE if pair_table else 0)
                                       | (ANY4_FLAG_DECODE_LAYOUT if decode_layout else 0),
                                       _stream(dev)), "any4_matmul_grouped")
    return outs


def any4_matmul_static_scratch(x: torch.Tensor, packed: torch.Tensor, lut: torch.Tensor,
                               scale: torch.Tensor, offset: torch.Tensor, G: int,
                               y: torch.Tensor | None = None,
                               dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """any4_matmul on the prefill kernel with the library's fixed scratch
    array instead of a workspace (the C entry point allocates nothing).

    For a call that allocates nothing at all, pass y (and dev_status if
    wanted): only a missing y is allocated here, with torch.  The first call on
    a device looks up the array's address; make it before any stream capture.
    Calls whose kernels overlap on the GPU share the array and race."""
    M, N, K, stride, y = _matmul_operands(x, packed, lut, scale, offset, G, y,
                                             dev_status)
    dev = x.device
    _need_status(dev_status, dev)
    lib = library()
    with _on_device(dev):
        _check(lib.any4_matmul_static_scratch(_ptr(x), _ptr(packed), _ptr(lut), stride,
                                              _ptr(scale), _ptr(offset), _ptr(y), M, N, K, G,
                                              _ptr(dev_status), _stream(dev)),
               "any4_matmul_static_scratch")
    return y
