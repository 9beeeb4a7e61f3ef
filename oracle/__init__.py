"""any4 oracle: plain fp64 CPU implementation of the any4 W4A16 path.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg (and its ``--impl reference`` arm) may import this package.  The
product path (learned_bit_lut_any4_b200) never imports it and shares no code
with it.

Every function follows "any4: Learned 4-bit Numeric Representation for LLMs"
(Elhoushi & Johnson, arXiv 2507.04610):
  pack / unpack      §2.4.1 and §4.2 (two 4-bit codes per byte; low nibble =
                     even column is the reading used here, the pages are silent)
  dequant            §2.5.2 dequant(w_Q) = alpha*w_Q + beta with w_Q = LUT[code];
                     §2.5.1 group k covers columns k*G .. (k+1)*G-1
  matmul             §4.1 Eq. 8 and §4.2 (y = x W^T, x is M x K, W is N x K)
  repack_decode_layout  §4.2's pre-permuted weight order, for the library's
                     M = 1 kernel: which 8 columns a thread reads at a step
  group_sums         per-group activation sums, the factor of the group offset
                     when Eq. 8 is expanded with the group-affine weights of
                     §2.5.2 (the pages do not name it; this is that reading)
  bits_per_weight    §2.4.1 storage accounting (4.3125 bits at G=128, K=4096)
  group_scale        §2.5.1 Eq. 1-2 (alpha = (max - min) / 15, beta = min)
  scaled_weights     §2.5.1 Eq. 1 (w_S = (w - beta) / alpha)
  kmeans_row         §4.1 E-step (Eq. 18) and M-step (Eq. 23), weighted Lloyd
                     iteration from a quantile initialisation
  quantize           §4.1 and Appendix A.1 (Alg. 1): scaling, then k-means per
                     row with sample weight alpha * E|x|; bf16 table and codes
  *_bits             the same for n-bit codes, n in {2, 3, 4} (§4.1 Eq. 9: 2^n
                     values per row; §5: any3, any2), with the storage reading
                     "one little-endian bit stream per row" (the pages give no
                     layout below 4 bits)

bf16 values cross this interface as their raw uint16 bit patterns.  The
arithmetic lives in any4_oracle.c (fp32 fmaf + IEEE round-to-nearest-even to
bf16 for the dequant, fp64 ascending-k sums for the matmul).

Parity status: every function here is pinned by tests/test_oracle_pins.py.
The nf4 constant table itself is not printed on the pages; the nf4 pin checks
the one-table-per-matrix structure for an arbitrary table (parity of the
table's VALUES with a published nf4 table is unpinned).
"""
import contextlib
import ctypes

import numpy as np

from . import build as _build

_lib = None


def _bind(lib):
    """Declare the C signatures on a loaded oracle library."""
    u8p = ctypes.POINTER(ctypes.c_uint8)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i64 = ctypes.c_int64
    lib.oracle_bf16_rne.argtypes = [ctypes.c_float]
    lib.oracle_bf16_rne.restype = ctypes.c_uint16
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = ctypes.c_float
    f32p = ctypes.POINTER(ctypes.c_float)
    lib.oracle_bf16_rne_array.argtypes = [f32p, u16p, i64]
    lib.oracle_bf16_rne_array.restype = None
    lib.oracle_bf16_to_f32_array.argtypes = [u16p, f32p, i64]
    lib.oracle_bf16_to_f32_array.restype = None
    lib.oracle_pack.argtypes = [u8p, u8p, i64, i64]
    lib.oracle_pack.restype = i64
    lib.oracle_unpack.argtypes = [u8p, u8p, i64, i64]
    lib.oracle_unpack.restype = None
    lib.oracle_repack_decode_layout.argtypes = [u8p, u8p, i64, i64]
    lib.oracle_repack_decode_layout.restype = ctypes.c_int
    lib.oracle_bits_per_weight.argtypes = [i64, i64, i64, i64]
    lib.oracle_bits_per_weight.restype = ctypes.c_double
    lib.oracle_dequant_one.argtypes = [ctypes.c_uint16] * 3
    lib.oracle_dequant_one.restype = ctypes.c_uint16
    lib.oracle_dequant.argtypes = [u8p, u16p, i64, u16p, u16p, u16p, i64, i64, i64]
    lib.oracle_dequant.restype = None
    lib.oracle_matmul.argtypes = [u16p, u16p, f64p, i64, i64, i64]
    lib.oracle_matmul.restype = None
    lib.oracle_matmul_rows.argtypes = [u16p, u8p, u16p, i64, u16p, u16p, i64p, i64,
                                       f64p, u16p, i64, i64, i64, i64]
    lib.oracle_matmul_rows.restype = None
    lib.oracle_group_scale.argtypes = [u16p, i64, i64, i64, u16p, u16p]
    lib.oracle_group_scale.restype = None
    lib.oracle_scaled_weights.argtypes = [u16p, u16p, u16p, i64, i64, i64, f64p]
    lib.oracle_scaled_weights.restype = None
    lib.oracle_kmeans_row.argtypes = [f64p, f64p, i64, i64, f64p, u8p]
    lib.oracle_kmeans_row.restype = i64
    lib.oracle_any4_quantize.argtypes = [u16p, f32p, i64, i64, i64, i64, u8p, u16p, u16p, u16p,
                                         i64p]
    lib.oracle_any4_quantize.restype = None
    ci = ctypes.c_int
    lib.oracle_group_scale_bits.argtypes = [u16p, i64, i64, i64, ci, u16p, u16p]
    lib.oracle_group_scale_bits.restype = None
    lib.oracle_kmeans_row_bits.argtypes = [f64p, f64p, i64, ci, i64, f64p, u8p]
    lib.oracle_kmeans_row_bits.restype = i64
    lib.oracle_quantize_bits.argtypes = [u16p, f32p, i64, i64, i64, ci, i64, u8p, u16p, u16p,
                                         u16p, i64p]
    lib.oracle_quantize_bits.restype = None
    lib.oracle_pack_bits.argtypes = [u8p, u8p, i64, i64, ci]
    lib.oracle_pack_bits.restype = i64
    lib.oracle_unpack_bits.argtypes = [u8p, u8p, i64, i64, ci]
    lib.oracle_unpack_bits.restype = None
    lib.oracle_dequant_bits.argtypes = [u8p, u16p, i64, u16p, u16p, u16p, i64, i64, i64, ci]
    lib.oracle_dequant_bits.restype = None
    lib.oracle_bits_per_weight_n.argtypes = [i64, i64, ci]
    lib.oracle_bits_per_weight_n.restype = ctypes.c_double
    lib.oracle_group_sums.argtypes = [u16p, f64p, i64, i64, i64]
    lib.oracle_group_sums.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


@contextlib.contextmanager
def swapped_library(path: str):
    """Test hook: run the wrappers against another build of the oracle source
    (the mutation tests plant a mistake in a copy and check that a pin fails)."""
    global _lib
    saved = _lib
    _lib = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(t: int) -> None:
    _load().oracle_set_num_threads(int(t))


def bf16_rne(f32: np.ndarray) -> np.ndarray:
    """Round binary32 values to bfloat16 bit patterns (ties to even)."""
    f = np.ascontiguousarray(f32, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    _load().oracle_bf16_rne_array(_ptr(f, ctypes.c_float), _ptr(out, ctypes.c_uint16), f.size)
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to binary32 (exact)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    _load().oracle_bf16_to_f32_array(_ptr(h, ctypes.c_uint16), _ptr(out, ctypes.c_float), h.size)
    return out


def pack(idx: np.ndarray) -> np.ndarray:
    """idx uint8 [N, K] (codes 0..15) -> packed uint8 [N, K/2], low nibble = even k.

    Raises ValueError if any code is outside 0..15 or K is odd."""
    idx = _c(idx, np.uint8)
    N, K = idx.shape
    if K % 2:
        raise ValueError("K must be even")
    packed = np.empty((N, K // 2), dtype=np.uint8)
    bad = _load().oracle_pack(_ptr(idx, ctypes.c_uint8), _ptr(packed, ctypes.c_uint8), N, K)
    if bad:
        raise ValueError(f"{bad} codes outside 0..15")
    return packed


def unpack(packed: np.ndarray) -> np.ndarray:
    packed = _c(packed, np.uint8)
    N, Kh = packed.shape
    idx = np.empty((N, 2 * Kh), dtype=np.uint8)
    _load().oracle_unpack(_ptr(packed, ctypes.c_uint8), _ptr(idx, ctypes.c_uint8), N, 2 * Kh)
    return idx


def repack_decode_layout(packed: np.ndarray) -> np.ndarray:
    """packed uint8 [N, K/2] (pack's layout) -> the same codes in the order the
    library's M = 1 decode kernel reads them (any4_repack); K a multiple of
    1024.  The statement is oracle_repack_decode_layout in any4_oracle.c."""
    packed = _c(packed, np.uint8)
    N, Kh = packed.shape
    out = np.empty_like(packed)
    if _load().oracle_repack_decode_layout(_ptr(packed, ctypes.c_uint8),
                                           _ptr(out, ctypes.c_uint8), N, 2 * Kh) != 0:
        raise ValueError("K must be a positive multiple of 1024")
    return out


def bits_per_weight(K: int, G: int, lut_bits: int = 16, group_param_bits: int = 16) -> float:
    return _load().oracle_bits_per_weight(K, G, lut_bits, group_param_bits)


def dequant_one(lut_c: int, scale: int, offset: int) -> int:
    """bf16 bits of bf16_rne(fmaf(LUT[c], scale, offset)) for one weight."""
    return int(_load().oracle_dequant_one(lut_c, scale, offset))


def dequant(packed, lut, scale, offset, G: int, per_tensor_lut: bool = False) -> np.ndarray:
    """W[n][k] = bf16(fmaf(LUT[n][code], scale[n][k/G], offset[n][k/G])) as uint16 [N, K].

    lut is uint16 [N, 16] (one table per row) or, with per_tensor_lut, [16]
    (one table for the whole matrix, the nf4/af4 mode)."""
    packed = _c(packed, np.uint8)
    lut = _c(lut, np.uint16)
    scale = _c(scale, np.uint16)
    offset = _c(offset, np.uint16)
    N, Kh = packed.shape
    K = 2 * Kh
    if K % G:
        raise ValueError("K must be a multiple of G")
    if scale.shape != (N, K // G) or offset.shape != (N, K // G):
        raise ValueError("scale/offset must be [N, K/G]")
    if per_tensor_lut:
        if lut.size != 16:
            raise ValueError("per-tensor LUT must have 16 entries")
        stride = 0
    else:
        if lut.shape != (N, 16):
            raise ValueError("LUT must be [N, 16]")
        stride = 16
    W = np.empty((N, K), dtype=np.uint16)
    _load().oracle_dequant(_ptr(packed, ctypes.c_uint8), _ptr(lut, ctypes.c_uint16), stride,
                           _ptr(scale, ctypes.c_uint16), _ptr(offset, ctypes.c_uint16),
                           _ptr(W, ctypes.c_uint16), N, K, G)
    return W


def matmul(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = x W^T in fp64 (ascending-k sums).  x uint16 [M, K], W uint16 [N, K]."""
    x = _c(x, np.uint16)
    W = _c(W, np.uint16)
    M, K = x.shape
    N, K2 = W.shape
    if K != K2:
        raise ValueError("K mismatch")
    y = np.empty((M, N), dtype=np.float64)
    _load().oracle_matmul(_ptr(x, ctypes.c_uint16), _ptr(W, ctypes.c_uint16),
                          _ptr(y, ctypes.c_double), M, N, K)
    return y


def matmul_rows(x, packed, lut, scale, offset, G: int, rows, per_tensor_lut: bool = False):
    """fp64 y[:, rows] of y = x dequant(W)^T, dequantising only the chosen rows."""
    x = _c(x, np.uint16)
    packed = _c(packed, np.uint8)
    lut = _c(lut, np.uint16)
    scale = _c(scale, np.uint16)
    offset = _c(offset, np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K:
        raise ValueError("K mismatch")
    if rows.size and (rows.min() < 0 or rows.max() >= N):
        raise ValueError("row index out of range")
    stride = 0 if per_tensor_lut else 16
    y = np.empty((M, rows.size), dtype=np.float64)
    wrow = np.empty((rows.size, K), dtype=np.uint16)
    _load().oracle_matmul_rows(_ptr(x, ctypes.c_uint16), _ptr(packed, ctypes.c_uint8),
                               _ptr(lut, ctypes.c_uint16), stride,
                               _ptr(scale, ctypes.c_uint16), _ptr(offset, ctypes.c_uint16),
                               _ptr(rows, ctypes.c_int64), rows.size,
                               _ptr(y, ctypes.c_double), _ptr(wrow, ctypes.c_uint16),
                               M, N, K, G)
    return y


def group_sums(x: np.ndarray, G: int) -> np.ndarray:
    """xsum[m][g] = sum of x[m][k] over the G columns of group g, fp64 [M, K/G].

    x is uint16 (bf16 bits) [M, K]; K must be a multiple of G."""
    x = _c(x, np.uint16)
    if x.ndim != 2 or G < 1 or x.shape[1] % G:
        raise ValueError("x must be [M, K] with K a multiple of G")
    M, K = x.shape
    out = np.empty((M, K // G), dtype=np.float64)
    _load().oracle_group_sums(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_double), M, K, G)
    return out


def any4_matmul(x, packed, lut, scale, offset, G: int, per_tensor_lut: bool = False):
    """Dequant-then-matmul, the full definition: fp64 y [M, N]."""
    return matmul(x, dequant(packed, lut, scale, offset, G, per_tensor_lut))


def _check_weight(w, G):
    w = _c(w, np.uint16)
    if w.ndim != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    if N < 1 or K < 1 or G < 1 or K % G:
        raise ValueError("need N, K, G >= 1 and K a multiple of G")
    return w, N, K


def group_scale(w, G: int):
    """§2.5.1 Eq. 1-2 per group of G columns: (scale, offset) as bf16 bits [N, K/G],
    scale = bf16((max - min) / 15 in fp32), offset = min."""
    w, N, K = _check_weight(w, G)
    scale = np.empty((N, K // G), dtype=np.uint16)
    offset = np.empty((N, K // G), dtype=np.uint16)
    _load().oracle_group_scale(_ptr(w, ctypes.c_uint16), N, K, G, _ptr(scale, ctypes.c_uint16),
                               _ptr(offset, ctypes.c_uint16))
    return scale, offset


def scaled_weights(w, scale, offset, G: int):
    """fp64 w_S = (w - offset) / scale [N, K] (0 in a group whose scale is 0)."""
    w, N, K = _check_weight(w, G)
    scale = _c(scale, np.uint16)
    offset = _c(offset, np.uint16)
    if scale.shape != (N, K // G) or offset.shape != (N, K // G):
        raise ValueError("scale/offset must be [N, K/G]")
    ws = np.empty((N, K), dtype=np.float64)
    _load().oracle_scaled_weights(_ptr(w, ctypes.c_uint16), _ptr(scale, ctypes.c_uint16),
                                  _ptr(offset, ctypes.c_uint16), N, K, G,
                                  _ptr(ws, ctypes.c_double))
    return ws


def kmeans_row(xs, u, max_iter: int):
    """Weighted Lloyd iteration (§4.1 Eq. 18 / Eq. 23) on one row from the
    quantile initialisation: (fp64 centroids [16], codes uint8 [K], M-steps run)."""
    xs = _c(xs, np.float64)
    u = _c(u, np.float64)
    if xs.ndim != 1 or u.shape != xs.shape or xs.size < 1:
        raise ValueError("xs and u must be equal-length non-empty vectors")
    if max_iter < 0:
        raise ValueError("max_iter must be >= 0")
    c = np.empty(16, dtype=np.float64)
    code = np.empty(xs.size, dtype=np.uint8)
    it = _load().oracle_kmeans_row(_ptr(xs, ctypes.c_double), _ptr(u, ctypes.c_double), xs.size,
                                   int(max_iter), _ptr(c, ctypes.c_double),
                                   _ptr(code, ctypes.c_uint8))
    return c, code, int(it)


def quantize(w, ex, G: int, max_iter: int):
    """The whole any4 quantiser (§2.5.1 scaling, then §4.1 weighted k-means per
    row): w bf16 bits [N, K], ex = E|x| fp32 [K] (finite, >= 0).

    Returns (codes uint8 [N, K], lut bf16 bits [N, 16], scale [N, K/G],
    offset [N, K/G], iters int64 [N])."""
    w, N, K = _check_weight(w, G)
    ex = _c(ex, np.float32)
    if ex.shape != (K,):
        raise ValueError("ex must be [K]")
    if not np.all(np.isfinite(ex)) or np.any(ex < 0):
        raise ValueError("ex must be finite and >= 0")
    if max_iter < 0:
        raise ValueError("max_iter must be >= 0")
    codes = np.empty((N, K), dtype=np.uint8)
    lut = np.empty((N, 16), dtype=np.uint16)
    scale = np.empty((N, K // G), dtype=np.uint16)
    offset = np.empty((N, K // G), dtype=np.uint16)
    iters = np.empty(N, dtype=np.int64)
    _load().oracle_any4_quantize(_ptr(w, ctypes.c_uint16), _ptr(ex, ctypes.c_float), N, K, G,
                                 int(max_iter), _ptr(codes, ctypes.c_uint8),
                                 _ptr(lut, ctypes.c_uint16), _ptr(scale, ctypes.c_uint16),
                                 _ptr(offset, ctypes.c_uint16), _ptr(iters, ctypes.c_int64))
    return codes, lut, scale, offset, iters


# --------------------------------------------------------------------------
# n-bit variants (any3, any2; n = 4 is any4): §4.1 Eq. 9 (2^n values per row),
# §5 (any3 / any2 evaluated).  Storage reading: a row's codes form one
# little-endian bit stream, code k in bits [n k, n k + n).
# --------------------------------------------------------------------------

_BITS = (2, 3, 4)


def _check_bits(bits):
    if bits not in _BITS:
        raise ValueError(f"bits must be one of {_BITS}")
    return int(bits)


def pack_bits(idx: np.ndarray, bits: int) -> np.ndarray:
    """idx uint8 [N, K] (codes 0 .. 2^bits - 1) -> packed uint8 [N, bits*K/8]."""
    bits = _check_bits(bits)
    idx = _c(idx, np.uint8)
    N, K = idx.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    packed = np.empty((N, bits * K // 8), dtype=np.uint8)
    bad = _load().oracle_pack_bits(_ptr(idx, ctypes.c_uint8), _ptr(packed, ctypes.c_uint8), N, K,
                                   bits)
    if bad:
        raise ValueError(f"{bad} codes outside 0..{(1 << bits) - 1}")
    return packed


def unpack_bits(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    bits = _check_bits(bits)
    packed = _c(packed, np.uint8)
    N = packed.shape[0]
    if K % 8 or packed.shape[1] != bits * K // 8:
        raise ValueError("packed must be [N, bits*K/8] with K a multiple of 8")
    idx = np.empty((N, K), dtype=np.uint8)
    _load().oracle_unpack_bits(_ptr(packed, ctypes.c_uint8), _ptr(idx, ctypes.c_uint8), N, K, bits)
    return idx


def dequant_bits(packed, lut, scale, offset, G: int, bits: int, K: int,
                 per_tensor_lut: bool = False) -> np.ndarray:
    """W[n][k] = bf16(fmaf(LUT[n][code], scale[n][k/G], offset[n][k/G])) for
    n-bit codes; lut is [N, 2^bits] or, with per_tensor_lut, [2^bits]."""
    bits = _check_bits(bits)
    packed = _c(packed, np.uint8)
    lut = _c(lut, np.uint16)
    scale = _c(scale, np.uint16)
    offset = _c(offset, np.uint16)
    N = packed.shape[0]
    nq = 1 << bits
    if K % 8 or K % G or packed.shape[1] != bits * K // 8:
        raise ValueError("bad K, G or packed shape")
    if scale.shape != (N, K // G) or offset.shape != (N, K // G):
        raise ValueError("scale/offset must be [N, K/G]")
    if per_tensor_lut:
        if lut.size != nq:
            raise ValueError(f"per-tensor LUT must have {nq} entries")
        stride = 0
    else:
        if lut.shape != (N, nq):
            raise ValueError(f"LUT must be [N, {nq}]")
        stride = nq
    W = np.empty((N, K), dtype=np.uint16)
    _load().oracle_dequant_bits(_ptr(packed, ctypes.c_uint8), _ptr(lut, ctypes.c_uint16), stride,
                                _ptr(scale, ctypes.c_uint16), _ptr(offset, ctypes.c_uint16),
                                _ptr(W, ctypes.c_uint16), N, K, G, bits)
    return W


def bits_per_weight_n(K: int, G: int, bits: int) -> float:
    return _load().oracle_bits_per_weight_n(K, G, _check_bits(bits))


def group_scale_bits(w, G: int, bits: int):
    """Eq. 1-2 with Qmax - Qmin = 2^bits - 1: (scale, offset) bf16 bits [N, K/G]."""
    bits = _check_bits(bits)
    w, N, K = _check_weight(w, G)
    scale = np.empty((N, K // G), dtype=np.uint16)
    offset = np.empty((N, K // G), dtype=np.uint16)
    _load().oracle_group_scale_bits(_ptr(w, ctypes.c_uint16), N, K, G, bits,
                                    _ptr(scale, ctypes.c_uint16), _ptr(offset, ctypes.c_uint16))
    return scale, offset


def kmeans_row_bits(xs, u, bits: int, max_iter: int):
    """kmeans_row with 2^bits entries."""
    bits = _check_bits(bits)
    xs = _c(xs, np.float64)
    u = _c(u, np.float64)
    if xs.ndim != 1 or u.shape != xs.shape or xs.size < 1 or max_iter < 0:
        raise ValueError("bad arguments")
    c = np.empty(1 << bits, dtype=np.float64)
    code = np.empty(xs.size, dtype=np.uint8)
    it = _load().oracle_kmeans_row_bits(_ptr(xs, ctypes.c_double), _ptr(u, ctypes.c_double),
                                        xs.size, bits, int(max_iter), _ptr(c, ctypes.c_double),
                                        _ptr(code, ctypes.c_uint8))
    return c, code, int(it)


def quantize_bits(w, ex, G: int, bits: int, max_iter: int):
    """quantize for n-bit codes: (codes [N, K], lut [N, 2^bits], scale, offset, iters)."""
    bits = _check_bits(bits)
    w, N, K = _check_weight(w, G)
    ex = _c(ex, np.float32)
    if ex.shape != (K,):
        raise ValueError("ex must be [K]")
    if not np.all(np.isfinite(ex)) or np.any(ex < 0):
        raise ValueError("ex must be finite and >= 0")
    if max_iter < 0:
        raise ValueError("max_iter must be >= 0")
    nq = 1 << bits
    codes = np.empty((N, K), dtype=np.uint8)
    lut = np.empty((N, nq), dtype=np.uint16)
    scale = np.empty((N, K // G), dtype=np.uint16)
    offset = np.empty((N, K // G), dtype=np.uint16)
    iters = np.empty(N, dtype=np.int64)
    _load().oracle_quantize_bits(_ptr(w, ctypes.c_uint16), _ptr(ex, ctypes.c_float), N, K, G,
                                 bits, int(max_iter), _ptr(codes, ctypes.c_uint8),
                                 _ptr(lut, ctypes.c_uint16), _ptr(scale, ctypes.c_uint16),
                                 _ptr(offset, ctypes.c_uint16), _ptr(iters, ctypes.c_int64))
    return codes, lut, scale, offset, iters


__all__ = ["bf16_rne", "bf16_to_f32", "pack", "unpack", "bits_per_weight", "dequant_one",
           "dequant", "matmul", "matmul_rows", "any4_matmul", "num_threads",
           "set_num_threads", "group_scale", "scaled_weights", "kmeans_row", "quantize",
           "pack_bits", "unpack_bits", "dequant_bits", "bits_per_weight_n", "group_scale_bits",
           "kmeans_row_bits", "quantize_bits"]
