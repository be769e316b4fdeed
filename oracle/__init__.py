"""CPU oracle for the FP8 delayed-scaling linear path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and the
two share no code: this package wraps ``fp8_oracle.c`` (plain single-threaded
C, fp64) through ctypes and composes its functions, in the order the pages
describe, into the linear-layer steps.

Arrays are numpy.  bf16 tensors travel as their raw ``uint16`` bit patterns.
Amax histories are ``[H, T]`` float32 (slot-major: row 0 is the amax recorded
in the current step).
"""
import ctypes
import numpy as np

from . import build as _build

E4M3 = 0
E5M2 = 1
F32 = 0
BF16 = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        f32 = ctypes.c_float
        L.orc_decode.restype = ctypes.c_double
        L.orc_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
        L.orc_encode.restype = ctypes.c_uint8
        L.orc_encode.argtypes = [f32, ctypes.c_int]
        L.orc_decode_table.argtypes = [ctypes.c_int, P]
        L.orc_encode_array.argtypes = [P, i64, ctypes.c_int, P]
        L.orc_scaled.restype = f32
        L.orc_scaled.argtypes = [f32, f32]
        L.orc_reciprocal.restype = f32
        L.orc_reciprocal.argtypes = [f32]
        L.orc_cast_transpose_amax.argtypes = [P, ctypes.c_int, i64, i64, ctypes.c_int, f32,
                                              P, P, P, P]
        L.orc_quantize.argtypes = [P, ctypes.c_int, i64, ctypes.c_int, f32, P, P, P]
        L.orc_amax.argtypes = [P, ctypes.c_int, i64, P]
        L.orc_update_scales.argtypes = [i64, ctypes.c_int, P, P, P, P]
        L.orc_update_scales_algo.argtypes = [i64, ctypes.c_int, P, P, P, P, ctypes.c_int]
        L.orc_gemm_rows.argtypes = [P, ctypes.c_int, P, ctypes.c_int, f32, f32, P,
                                    i64, i64, i64, P, i64, P]
        L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_round_bf16.argtypes = [ctypes.c_double]
        L.orc_round_bf16_array.argtypes = [P, i64, P]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fp8_max(fmt):
    return lib().orc_decode(0x7E if fmt == E4M3 else 0x7B, fmt)


def decode_table(fmt):
    """All 256 codes decoded exactly (float64; NaN for NaN codes)."""
    out = np.empty(256, np.float64)
    lib().orc_decode_table(fmt, _ptr(out))
    return out


def decode(codes, fmt):
    return decode_table(fmt)[np.asarray(codes, dtype=np.uint8)]


def encode(values, fmt):
    """Saturating round-to-nearest-even of float32 values to FP8 codes."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_encode_array(_ptr(v), v.size, fmt, _ptr(out))
    return out


def _as_input(x):
    """Return (contiguous array, dtype tag) for fp32 arrays or bf16 bit arrays."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError("oracle inputs are float32 or bf16 bit patterns (uint16), got %s" % x.dtype)


def scaled(x, scale):
    return np.float32(lib().orc_scaled(float(x), float(scale)))


def reciprocal(s):
    return np.float32(lib().orc_reciprocal(float(s)))


def cast_transpose_amax(x, fmt, scale, amax=0.0, transpose=True):
    """Cast a 2-D tensor with one scale.

    Returns (y [R,C] u8, yt [C,R] u8 or None, amax' float32, scale_inv float32),
    where amax' = max(amax, max|x|) over the unscaled input.
    """
    x, tag = _as_input(x)
    if x.ndim != 2:
        raise ValueError("2-D input expected")
    R, C = x.shape
    y = np.empty((R, C), np.uint8)
    yt = np.empty((C, R), np.uint8) if transpose else None
    am = np.array([amax], np.float32)
    si = np.zeros(1, np.float32)
    lib().orc_cast_transpose_amax(_ptr(x), tag, R, C, fmt, float(scale), _ptr(y), _ptr(yt),
                                  _ptr(am), _ptr(si))
    return y, yt, am[0], si[0]


def quantize(x, fmt, scale, amax=0.0):
    """Flat cast: returns (y u8 same shape, amax', scale_inv)."""
    x, tag = _as_input(x)
    y = np.empty(x.shape, np.uint8)
    am = np.array([amax], np.float32)
    si = np.zeros(1, np.float32)
    lib().orc_quantize(_ptr(x), tag, x.size, fmt, float(scale), _ptr(y), _ptr(am), _ptr(si))
    return y, am[0], si[0]


def amax(x, amax=0.0):
    """max(amax, max|x|) over the unscaled input, NaN ignored (float32)."""
    x, tag = _as_input(x)
    am = np.array([amax], np.float32)
    lib().orc_amax(_ptr(x), tag, x.size, _ptr(am))
    return am[0]


AMAX_MAX = 0
AMAX_MOST_RECENT = 1


def update_scales(hist, scale, scale_inv, fmts, algo=AMAX_MAX):
    """One delayed-scaling update over T metas; returns new (hist, scale, scale_inv).
    algo: AMAX_MAX (max over the history window) or AMAX_MOST_RECENT (the
    current step's amax)."""
    hist = np.array(hist, np.float32, copy=True, order="C")
    scale = np.array(scale, np.float32, copy=True)
    scale_inv = np.array(scale_inv, np.float32, copy=True)
    fmts = np.ascontiguousarray(fmts, dtype=np.uint8)
    H, T = hist.shape
    lib().orc_update_scales_algo(T, H, _ptr(hist), _ptr(scale), _ptr(scale_inv), _ptr(fmts), int(algo))
    return hist, scale, scale_inv


def round_bf16(d):
    """Round-to-nearest-even of fp64 values to bf16; returns uint16 bit patterns."""
    d = np.ascontiguousarray(d, dtype=np.float64)
    out = np.empty(d.shape, np.uint16)
    lib().orc_round_bf16_array(_ptr(d), d.size, _ptr(out))
    return out


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def gemm(A, fa, B, fb, a_scale_inv, b_scale_inv, bias=None, rows=None):
    """fp64 D[rows, N] = (A[rows] . B^T) * a_scale_inv * b_scale_inv + bias."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    if K != K2:
        raise ValueError("contraction sizes differ")
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    if rows is None:
        idx = None
        n_rows = M
    else:
        idx = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = idx.size
    D = np.zeros((n_rows, N), np.float64)
    lib().orc_gemm_rows(_ptr(A), fa, _ptr(B), fb, float(a_scale_inv), float(b_scale_inv),
                        _ptr(b), M, N, K, _ptr(idx), n_rows, _ptr(D))
    return D


from .linear import OracleMeta, OracleLinear  # noqa: E402,F401
