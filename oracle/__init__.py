"""Test infrastructure: numpy-facing wrapper of the plain-C CPU oracle.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this
package. The product path (mxfp4_w4a4_post_b200 and its CUDA library) never does, and
the oracle imports nothing from it.

Every function here marshals numpy arrays into oracle/liboracle.so; the arithmetic is
in oracle/macaq_oracle.c (see its header for the pages it follows).
"""
import ctypes
import os

import numpy as np

from . import build_oracle

_libs = {}
_openmp = False


def set_openmp(flag):
    """Route every call below to the OpenMP build of the oracle (row loops on all host
    cores, same results) or back to the single-threaded one (the default). Used only to
    time the oracle."""
    global _openmp
    _openmp = bool(flag)


def lib():
    key = "omp" if _openmp else "serial"
    if key not in _libs:
        path = build_oracle.build_omp() if _openmp else build_oracle.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_hadamard_entry.argtypes = [ctypes.c_int, ctypes.c_int]
        L.oracle_hadamard_entry.restype = ctypes.c_int
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_fwht32_f32.argtypes = [P]
        L.oracle_fwht32_f32.restype = None
        L.oracle_e8m0_exponent.argtypes = [ctypes.c_float]
        L.oracle_e8m0_exponent.restype = ctypes.c_int
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode_array.argtypes = [P, I64, P]
        L.oracle_e2m1_encode_array.restype = None
        L.oracle_e8m0_exponent_array.argtypes = [P, I64, P]
        L.oracle_e8m0_exponent_array.restype = None
        L.oracle_quant_rows.argtypes = [P, I64, I64, I64, P, P, P]
        L.oracle_quant_rows.restype = None
        L.oracle_prepare_weight.argtypes = [P, I64, I64, I64, P, P, P, P]
        L.oracle_prepare_weight.restype = None
        L.oracle_scale_rows_padded.argtypes = [I64]
        L.oracle_scale_rows_padded.restype = I64
        L.oracle_scale_blocks_padded.argtypes = [I64]
        L.oracle_scale_blocks_padded.restype = I64
        L.oracle_scale_offset.argtypes = [I64, I64, I64]
        L.oracle_scale_offset.restype = I64
        L.oracle_swizzle_scales.argtypes = [P, I64, I64, P]
        L.oracle_swizzle_scales.restype = None
        L.oracle_unswizzle_scales.argtypes = [P, I64, I64, P]
        L.oracle_unswizzle_scales.restype = None
        L.oracle_gemm_fp64.argtypes = [P, P, I64, P, P, I64, I64, P, I64, P]
        L.oracle_gemm_fp64.restype = None
        L.oracle_dequant_rows.argtypes = [P, P, I64, I64, P]
        L.oracle_dequant_rows.restype = None
        L.oracle_transform_rows_f64.argtypes = [P, I64, I64, P, ctypes.c_double, P]
        L.oracle_transform_rows_f64.restype = None
        L.oracle_transform_block_f32.argtypes = [P, P, I64, P]
        L.oracle_transform_block_f32.restype = None
        L.oracle_hessian_blocks.argtypes = [P, I64, I64, I64, P, P]
        L.oracle_hessian_blocks.restype = None
        L.oracle_block_error.argtypes = [P, P]
        L.oracle_block_error.restype = ctypes.c_double
        L.oracle_block_error_at.argtypes = [P, ctypes.c_int, P, P]
        L.oracle_block_error_at.restype = ctypes.c_double
        L.oracle_search_block.argtypes = [P, P, P, P]
        L.oracle_search_block.restype = None
        L.oracle_prepare_weight_hessian.argtypes = [P, I64, I64, I64, P, P, P, P, P]
        L.oracle_prepare_weight_hessian.restype = None
        L.oracle_hessian_full.argtypes = [P, I64, I64, I64, P, P]
        L.oracle_hessian_full.restype = None
        L.oracle_flip_refine_row.argtypes = [P, P, I64, P, P, ctypes.c_int]
        L.oracle_flip_refine_row.restype = ctypes.c_int
        L.oracle_flip_refine.argtypes = [P, I64, I64, I64, P, P, P, P, ctypes.c_int, P]
        L.oracle_flip_refine.restype = None
        _libs[key] = L
    return _libs[key]


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ scalars ---

def hadamard_entry(i, j):
    return lib().oracle_hadamard_entry(int(i), int(j))


def bf16_to_f32(b):
    return np.float32(lib().oracle_bf16_to_f32(int(b)))


def fwht32(v):
    a = _c(v, np.float32).copy()
    assert a.shape == (32,)
    lib().oracle_fwht32_f32(_p(a))
    return a


def e8m0_exponent(amax):
    a = _c(np.atleast_1d(amax), np.float32)
    out = np.empty(a.shape, np.int32)
    lib().oracle_e8m0_exponent_array(_p(a), a.size, _p(out))
    return out if np.ndim(amax) else int(out[0])


def e2m1_encode(q):
    a = _c(np.atleast_1d(q), np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_p(a), a.size, _p(out))
    return out if np.ndim(q) else int(out[0])


def e2m1_decode(code):
    return lib().oracle_e2m1_decode(int(code))


# --------------------------------------------------------------------- rows ---

def quant_rows(x_bf16, mult):
    """x_bf16: uint16 [rows, K] bf16 bits; mult: float32 [K].
    Returns (codes uint8 [rows, K/2], scales uint8 [rows, K/32] row-major)."""
    x = _c(x_bf16, np.uint16)
    m = _c(mult, np.float32)
    rows, K = x.shape
    assert K % 32 == 0 and m.shape == (K,)
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    lib().oracle_quant_rows(_p(x), rows, K, K, _p(m), _p(codes), _p(scales))
    return codes, scales


def prepare_weight(W_bf16, s):
    """Returns (codes [N, K/2], scales [N, K/32] row-major, inv_s float32 [K])."""
    W = _c(W_bf16, np.uint16)
    s = _c(s, np.float32)
    N, K = W.shape
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    inv_s = np.empty(K, np.float32)
    lib().oracle_prepare_weight(_p(W), N, K, K, _p(s), _p(codes), _p(scales), _p(inv_s))
    return codes, scales, inv_s


def transform_block(x_row_bf16, mult, b):
    """The fp32 transformed block b of one row (fwht32 of x * mult)."""
    x = _c(x_row_bf16, np.uint16)
    m = _c(mult, np.float32)
    v = np.empty(32, np.float32)
    lib().oracle_transform_block_f32(_p(x), _p(m), int(b), _p(v))
    return v


def hessian_blocks(x_bf16, inv_s):
    """x_bf16: uint16 [T, K]; returns H float64 [K/32, 32, 32]."""
    x = _c(x_bf16, np.uint16)
    m = _c(inv_s, np.float32)
    T, K = x.shape
    H = np.empty((K // 32, 32, 32), np.float64)
    lib().oracle_hessian_blocks(_p(x), T, K, K, _p(m), _p(H))
    return H


def block_error(d, H):
    dd = _c(d, np.float64)
    Hh = _c(H, np.float64)
    return lib().oracle_block_error(_p(dd), _p(Hh))


def block_error_at(v, e, H):
    vv = _c(v, np.float32)
    Hh = _c(H, np.float64)
    codes = np.empty(16, np.uint8)
    err = lib().oracle_block_error_at(_p(vv), int(e), _p(Hh), _p(codes))
    return err, codes


def search_block(v, H):
    """Returns (codes uint8 [16], scale byte)."""
    vv = _c(v, np.float32)
    Hh = _c(H, np.float64)
    codes = np.empty(16, np.uint8)
    sc = np.empty(1, np.uint8)
    lib().oracle_search_block(_p(vv), _p(Hh), _p(codes), _p(sc))
    return codes, int(sc[0])


def prepare_weight_hessian(W_bf16, s, H):
    """Returns (codes [N, K/2], scales [N, K/32] row-major, inv_s float32 [K])."""
    W = _c(W_bf16, np.uint16)
    s = _c(s, np.float32)
    N, K = W.shape
    Hh = _c(H, np.float64)
    assert Hh.shape == (K // 32, 32, 32)
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    inv_s = np.empty(K, np.float32)
    lib().oracle_prepare_weight_hessian(_p(W), N, K, K, _p(s), _p(Hh), _p(codes), _p(scales), _p(inv_s))
    return codes, scales, inv_s


def hessian_full(x_bf16, inv_s):
    """Full K x K Gram matrix of the transformed rows of x (fp64)."""
    x = _c(x_bf16, np.uint16)
    m = _c(inv_s, np.float32)
    T, K = x.shape
    H = np.empty((K, K), np.float64)
    lib().oracle_hessian_full(_p(x), T, K, K, _p(m), _p(H))
    return H


def flip_refine_row(wv, H, codes_row, scales_row, max_rounds):
    """Returns (refined codes [K/2], number of moves)."""
    w = _c(wv, np.float32)
    Hh = _c(H, np.float64)
    c = np.array(codes_row, np.uint8, copy=True)
    sr = _c(scales_row, np.uint8)
    n = lib().oracle_flip_refine_row(_p(w), _p(Hh), w.size, _p(c), _p(sr), int(max_rounds))
    return c, n


def flip_refine(W_bf16, s, H, codes, scales_rowmajor, max_rounds):
    """Returns (refined codes [N, K/2], moves int32 [N])."""
    W = _c(W_bf16, np.uint16)
    s = _c(s, np.float32)
    N, K = W.shape
    Hh = _c(H, np.float64)
    assert Hh.shape == (K, K)
    c = np.array(codes, np.uint8, copy=True)
    sc = _c(scales_rowmajor, np.uint8)
    moves = np.empty(N, np.int32)
    lib().oracle_flip_refine(_p(W), N, K, K, _p(s), _p(Hh), _p(c), _p(sc), int(max_rounds), _p(moves))
    return c, moves


def scale_rows_padded(rows):
    return lib().oracle_scale_rows_padded(rows)


def scale_blocks_padded(K):
    return lib().oracle_scale_blocks_padded(K)


def scale_offset(r, j, K):
    return lib().oracle_scale_offset(r, j, K)


def swizzle_scales(rowmajor, K):
    rm = _c(rowmajor, np.uint8)
    rows = rm.shape[0]
    out = np.empty(scale_rows_padded(rows) * scale_blocks_padded(K), np.uint8)
    lib().oracle_swizzle_scales(_p(rm), rows, K, _p(out))
    return out


def unswizzle_scales(atom, rows, K):
    a = _c(atom, np.uint8).reshape(-1)
    assert a.size >= scale_rows_padded(rows) * scale_blocks_padded(K)
    out = np.empty((rows, K // 32), np.uint8)
    lib().oracle_unswizzle_scales(_p(a), rows, K, _p(out))
    return out


def dequant_rows(codes, scales, K):
    c = _c(codes, np.uint8)
    s = _c(scales, np.uint8)
    rows = c.shape[0]
    out = np.empty((rows, K), np.float64)
    lib().oracle_dequant_rows(_p(c), _p(s), rows, K, _p(out))
    return out


def gemm_fp64(a_codes, a_scales, w_codes, w_scales, K, rows=None):
    """fp64 sum of decoded products. rows: optional int64 row indices of A."""
    ac = _c(a_codes, np.uint8)
    as_ = _c(a_scales, np.uint8)
    wc = _c(w_codes, np.uint8)
    ws = _c(w_scales, np.uint8)
    M = ac.shape[0]
    N = wc.shape[0]
    if rows is None:
        y = np.empty((M, N), np.float64)
        lib().oracle_gemm_fp64(_p(ac), _p(as_), M, _p(wc), _p(ws), N, K, None, 0, _p(y))
    else:
        r = _c(rows, np.int64)
        assert r.min() >= 0 and r.max() < M
        y = np.empty((r.size, N), np.float64)
        lib().oracle_gemm_fp64(_p(ac), _p(as_), M, _p(wc), _p(ws), N, K, _p(r), r.size, _p(y))
    return y


def transform_rows_f64(x, mult, norm):
    xx = _c(x, np.float64)
    m = _c(mult, np.float64)
    rows, K = xx.shape
    out = np.empty_like(xx)
    lib().oracle_transform_rows_f64(_p(xx), rows, K, _p(m), float(norm), _p(out))
    return out


LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liboracle.so")


class use_library:
    """Temporarily route every oracle call to another build of the oracle source
    (used by the mutation tests, which compile deliberately broken copies to show
    that the pins catch them)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _openmp
        self._saved_mode = _openmp
        _openmp = False
        self._saved = lib()  # the default build, whose signatures are known
        L = ctypes.CDLL(self.path)
        for name in dir(self._saved):
            if name.startswith("oracle_"):
                f_src = getattr(self._saved, name)
                f = getattr(L, name)
                f.argtypes = f_src.argtypes
                f.restype = f_src.restype
        _libs["serial"] = L
        return L

    def __exit__(self, *exc):
        global _openmp
        _libs["serial"] = self._saved
        _openmp = self._saved_mode
        return False
