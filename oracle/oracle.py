"""numpy-facing wrappers of the C oracle (ctypes, no torch).

TEST INFRASTRUCTURE ONLY. See w4a16_oracle.c for the definitions and the passages they follow.
Arrays of 16-bit floats travel as uint16 bit patterns so that no library conversion sits
between the caller's bits and the oracle's own IEEE decoding.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

F16 = 0
BF16 = 1
OK = 0
EINVAL = -1
ENONFINITE = -4

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        lib.w4o_half_to_double.argtypes = [ctypes.c_uint16]
        lib.w4o_half_to_double.restype = ctypes.c_double
        lib.w4o_double_to_half.argtypes = [ctypes.c_double]
        lib.w4o_double_to_half.restype = ctypes.c_uint16
        lib.w4o_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.w4o_bf16_to_double.restype = ctypes.c_double
        lib.w4o_double_to_bf16.argtypes = [ctypes.c_double]
        lib.w4o_double_to_bf16.restype = ctypes.c_uint16
        lib.w4o_decode16.argtypes = [P, L, I, P]
        lib.w4o_decode16.restype = None
        lib.w4o_encode16.argtypes = [P, L, I, P]
        lib.w4o_encode16.restype = None
        lib.w4o_sizes.argtypes = [L, L, L, I, P]
        lib.w4o_sizes.restype = None
        lib.w4o_quantize.argtypes = [P, L, L, L, I, P, P, P, I]
        lib.w4o_quantize.restype = I
        lib.w4o_unpack_codes.argtypes = [P, L, L, I, P]
        lib.w4o_unpack_codes.restype = None
        lib.w4o_unpack_zeros.argtypes = [P, L, L, P]
        lib.w4o_unpack_zeros.restype = None
        lib.w4o_dequant.argtypes = [P, P, P, L, L, L, I, P]
        lib.w4o_dequant.restype = None
        lib.w4o_linear.argtypes = [P, I, L, L, P, P, P, L, L, I, P, L, P, P, I]
        lib.w4o_linear.restype = I
        lib.w4o_matmul.argtypes = [P, I, L, L, P, L, P]
        lib.w4o_matmul.restype = None
        lib.w4o_tiled_offsets.argtypes = [L, L, L, I, P]
        lib.w4o_tiled_offsets.restype = None
        lib.w4o_repack.argtypes = [P, P, P, L, L, L, I, P]
        lib.w4o_repack.restype = I
        lib.w4o_max_threads.argtypes = []
        lib.w4o_max_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    return int(_load().w4o_max_threads())


# ----------------------------------------------------------------------------- 16-bit formats
def decode16(bits, dtype=F16):
    """uint16 bit patterns -> float64, IEEE binary16 (dtype=F16) or bfloat16 (dtype=BF16)."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    _load().w4o_decode16(_ptr(b), b.size, dtype, _ptr(out))
    return out


def encode16(x, dtype=F16):
    """float64 -> uint16 bit patterns, round to nearest, ties to even."""
    v = _c(x, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().w4o_encode16(_ptr(v), v.size, dtype, _ptr(out))
    return out


# ----------------------------------------------------------------------------- format sizes
def sizes(K, N, group, sym):
    """(codes bytes, scale bytes, zero bytes) of the packed format."""
    out = np.zeros(3, dtype=np.int64)
    _load().w4o_sizes(K, N, group, int(sym), _ptr(out))
    return tuple(int(x) for x in out)


# ----------------------------------------------------------------------------- quantize
def quantize(W_bits, group, sym, nthreads=0):
    """RTN group quantization of fp16 W [K, N] (uint16 bits).

    Returns (status, codes int32 [K/8, N], scales uint16 fp16 bits [K/g, N],
    zeros int32 [K/g, N/8] or None when sym).
    """
    W = _c(W_bits, np.uint16)
    K, N = W.shape
    codes = np.zeros((K // 8, N), dtype=np.int32)
    scales = np.zeros((K // group, N), dtype=np.uint16)
    zeros = None if sym else np.zeros((K // group, N // 8), dtype=np.int32)
    st = _load().w4o_quantize(_ptr(W), K, N, group, int(sym), _ptr(codes), _ptr(scales),
                              _ptr(zeros), int(nthreads))
    return int(st), codes, scales, zeros


def unpack_codes(codes, K, sym):
    c = _c(codes, np.int32)
    N = c.shape[1]
    q = np.empty((K, N), dtype=np.int32)
    _load().w4o_unpack_codes(_ptr(c), K, N, int(sym), _ptr(q))
    return q


def unpack_zeros(zeros, G, N):
    z0 = _c(zeros, np.int32)
    z = np.empty((G, N), dtype=np.int32)
    _load().w4o_unpack_zeros(_ptr(z0), G, N, _ptr(z))
    return z


def dequant(codes, scales, zeros, K, N, group, sym):
    c = _c(codes, np.int32)
    s = _c(scales, np.uint16)
    z = None if sym else _c(zeros, np.int32)
    out = np.empty((K, N), dtype=np.float64)
    _load().w4o_dequant(_ptr(c), _ptr(s), _ptr(z), K, N, group, int(sym), _ptr(out))
    return out


# ----------------------------------------------------------------------------- linear layer
def linear(A_bits, a_dtype, codes, scales, zeros, N, group, sym, cols=None, nthreads=0):
    """y = A . dequant(W) in FP64 for the listed output columns (all when cols is None).

    Returns (Y [M, ncols], Yabs [M, ncols]) with Yabs = sum_k |a * w|.
    """
    A = _c(A_bits, np.uint16)
    M, K = A.shape
    c = _c(codes, np.int32)
    s = _c(scales, np.uint16)
    z = None if sym else _c(zeros, np.int32)
    if cols is None:
        ncols = N
        cols_arr = None
    else:
        cols_arr = _c(cols, np.int64)
        ncols = cols_arr.size
    Y = np.empty((M, ncols), dtype=np.float64)
    Yabs = np.empty((M, ncols), dtype=np.float64)
    st = _load().w4o_linear(_ptr(A), a_dtype, M, K, _ptr(c), _ptr(s), _ptr(z), N, group, int(sym),
                            _ptr(cols_arr), ncols, _ptr(Y), _ptr(Yabs), int(nthreads))
    if st != OK:
        raise ValueError(f"oracle linear rejected its arguments (status {st})")
    return Y, Yabs


def matmul(A_bits, a_dtype, What):
    A = _c(A_bits, np.uint16)
    M, K = A.shape
    W = _c(What, np.float64)
    N = W.shape[1]
    Y = np.empty((M, N), dtype=np.float64)
    _load().w4o_matmul(_ptr(A), a_dtype, M, K, _ptr(W), N, _ptr(Y))
    return Y


def within_bound(y, y_ref, y_abs, rel=2e-3, abs_=1e-5):
    """The acceptance bound |y - y_ref| <= rel * sum_k |a_k w_k| + abs_, elementwise."""
    y = np.asarray(y, dtype=np.float64)
    return np.abs(y - y_ref) <= rel * y_abs + abs_


# ----------------------------------------------------------------------------- tiled layout
def tiled_offsets(K, N, group, sym):
    """Sizes of the tiled buffer: bytes per unit record, the codes / scales / zeros offsets and
    sizes inside a record, and the whole buffer's size."""
    out = np.zeros(7, dtype=np.int64)
    _load().w4o_tiled_offsets(K, N, group, int(sym), _ptr(out))
    keys = ("record", "codes_bytes", "scales", "scales_bytes", "zeros", "zeros_bytes", "total")
    return {k: int(v) for k, v in zip(keys, out)}


def repack(codes, scales, zeros, K, N, group, sym):
    """The tiled buffer (uint8) holding the same bits as the plain packed weight."""
    off = tiled_offsets(K, N, group, sym)
    out = np.zeros(off["total"], dtype=np.uint8)
    c = _c(codes, np.int32)
    s = _c(scales, np.uint16)
    z = None if sym else _c(zeros, np.int32)
    st = _load().w4o_repack(_ptr(c), _ptr(s), _ptr(z), K, N, group, int(sym), _ptr(out))
    if st != OK:
        raise ValueError(f"oracle repack rejected its arguments (status {st})")
    return out
