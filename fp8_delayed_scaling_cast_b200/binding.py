"""Thin Python binding of libfp8ds.so (ctypes; argument marshalling only).

Every function has the name of the C entry point it calls and the same
argument order; tensors are torch CUDA tensors whose device pointers are
passed through, the stream defaults to torch's current stream.  Nothing here
computes: if the shared library is missing, importing this module raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8ds.so")

E4M3 = 0
E5M2 = 1
F32 = 0
BF16 = 1
AMAX_MAX = 0
AMAX_MOST_RECENT = 1

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_TIMEOUT = 4

_FMT_NAMES = {"e4m3": E4M3, "e5m2": E5M2, E4M3: E4M3, E5M2: E5M2}

K_MAJOR = 0      # operand [m, k] / [n, k] row-major
MN_MAJOR = 1     # operand [k, m] / [k, n] row-major
_MAJOR = {"k": K_MAJOR, "mn": MN_MAJOR, K_MAJOR: K_MAJOR, MN_MAJOR: MN_MAJOR}


class Fp8dsError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("fp8ds status %d: %s" % (status, message))
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError("libfp8ds.so not found at %s; build it with "
                      "`python -m fp8_delayed_scaling_cast_b200.build`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int


class _Meta(ctypes.Structure):
    _fields_ = [("amax_history", _P), ("scale", _P), ("scale_inv", _P), ("formats", _P),
                ("num_tensors", _I64), ("hist_len", _I32)]


class _Linear(ctypes.Structure):
    _fields_ = [("w", _P), ("bias", _P), ("bias_dtype", _INT), ("in_features", _I64),
                ("out_features", _I64), ("w8", _P), ("w8t", _P), ("w_scale_inv", _P),
                ("meta_in", _I32), ("meta_w", _I32), ("meta_grad", _I32), ("cache_valid", _I32),
                ("workspace", _P), ("workspace_bytes", ctypes.c_size_t), ("w_noop_flag", _P)]


class _CastJob(ctypes.Structure):
    _fields_ = [("x", _P), ("x_dtype", _INT), ("rows", _I64), ("cols", _I64), ("fmt", _INT), ("scale", _P),
                ("y", _P), ("yt", _P), ("amax", _P), ("scale_inv", _P), ("noop_flag", _P)]


class _Fp8Io(ctypes.Structure):
    _fields_ = [("in_cast", _I32), ("out_meta", _I32), ("out8", _P), ("out8t", _P), ("out_scale_inv", _P)]


_SIGS = {
    "fp8_quantize": [_P, _INT, _I64, _INT, _P, _P, _P, _P, _P],
    "fp8_cast_transpose_amax": [_P, _INT, _I64, _I64, _INT, _P, _P, _P, _P, _P, _P],
    "fp8_cast_transpose_amax_noop": [_P, _INT, _I64, _I64, _INT, _P, _P, _P, _P, _P, _P, _P],
    "fp8_cast_transpose_amax_pair": [_P, _I64, _I64, _P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                     _INT, _INT, _P],
    "fp8_cast_transpose_amax_dynamic": [_P, _INT, _I64, _I64, _INT, _P, _P, _P, _P, _P, _P],
    "fp8_transpose": [_P, _I64, _I64, _P, _P],
    "fp8_update_scales": [_I64, _I32, _P, _P, _P, _P, _INT, _P],
    "fp8_gemm": [_P, _INT, _P, _P, _INT, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P],
    "fp8_gemm_ex": [_P, _INT, _P, _P, _INT, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P,
                    ctypes.c_size_t, _P],
    "fp8_gemm_workspace_size": [ctypes.POINTER(ctypes.c_size_t)],
    "fp8_gemm_plan": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)],
    "fp8_gemm_noalloc": [_P, _INT, _P, _P, _INT, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P],
    "fp8_gemm_cast": [_P, _INT, _INT, _P, _P, _INT, _INT, _P, _P, _INT, _I64, _I64, _I64, _INT, _P, _P, _P, _P, _P,
                      _P],
    "fp8_linear_fwd": [ctypes.POINTER(_Linear), ctypes.POINTER(_Meta), _P, _INT, _I64, _P, _INT,
                       _I32, _P, _P, _P, _P],
    "fp8_linear_fwd_ex": [ctypes.POINTER(_Linear), ctypes.POINTER(_Meta), _P, _INT, _I64, _P, _INT,
                          _I32, _P, _P, _P, ctypes.POINTER(_Fp8Io), _P],
    "fp8_linear_bwd_ex": [ctypes.POINTER(_Linear), ctypes.POINTER(_Meta), _P, _INT, _I64, _P, _P, _P, _P,
                          _INT, _P, _P, _P, _P, ctypes.POINTER(_Fp8Io), _P],
    "fp8_gemm_major": [_P, _INT, _INT, _P, _P, _INT, _INT, _P, _P, _INT, _P, _INT, _I64, _I64, _I64, _P],
    "fp8_linear_bwd": [ctypes.POINTER(_Linear), ctypes.POINTER(_Meta), _P, _INT, _I64, _P, _P, _P,
                       _INT, _P, _P, _P, _P, _P],
    "fp8ds_device_status": [ctypes.POINTER(_I32), _I32],
    "fp8_cast_transpose_amax_multi": [ctypes.POINTER(_CastJob), _I32, _P],
    "fp8ds_test_stream_k_withhold": [_I32, ctypes.c_uint64],
    "fp8_linear_refresh_weights": [ctypes.POINTER(ctypes.POINTER(_Linear)), _I32, ctypes.POINTER(_Meta),
                                   ctypes.POINTER(_CastJob), _I32, _P],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _INT
_lib.fp8ds_last_error.restype = ctypes.c_char_p
_lib.fp8ds_last_error.argtypes = []
_lib.fp8ds_version.restype = ctypes.c_char_p
_lib.fp8ds_version.argtypes = []


def fp8ds_last_error():
    return _lib.fp8ds_last_error().decode()


def fp8ds_version():
    return _lib.fp8ds_version().decode()


def _check(status):
    if status != OK:
        raise Fp8dsError(status, fp8ds_last_error())


def _ptr(t):
    """Device pointer of a CUDA tensor (None -> NULL).  Host tensors are
    refused here: every pointer the library takes is a device pointer."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfp8ds takes CUDA tensors; got a %s tensor on %s" % (t.dtype, t.device))
    return t.data_ptr()


# The current stream's handle without building a torch.cuda.Stream object
# (which costs about 3 us per call, a third of a cast call's host time).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_get_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream):
    if stream is None:
        if _raw_stream is not None and _get_device is not None:
            return _raw_stream(_get_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("expected float32 or bfloat16 tensor, got %s" % t.dtype)


def _fmt(f):
    return _FMT_NAMES[f]


def fp8_quantize(x, fmt, scale, y, amax=None, scale_inv=None, stream=None):
    _check(_lib.fp8_quantize(_ptr(x), _dtype(x), x.numel(), _fmt(fmt), _ptr(scale), _ptr(y),
                             _ptr(amax), _ptr(scale_inv), _stream(stream)))


def fp8_cast_transpose_amax(x, fmt, scale, y, yt=None, amax=None, scale_inv=None, stream=None):
    rows, cols = x.shape
    _check(_lib.fp8_cast_transpose_amax(_ptr(x), _dtype(x), rows, cols, _fmt(fmt), _ptr(scale),
                                        _ptr(y), _ptr(yt), _ptr(amax), _ptr(scale_inv),
                                        _stream(stream)))


def fp8_cast_transpose_amax_noop(x, fmt, scale, y, yt, amax, scale_inv, noop_flag, stream=None):
    rows, cols = x.shape
    _check(_lib.fp8_cast_transpose_amax_noop(_ptr(x), _dtype(x), rows, cols, _fmt(fmt), _ptr(scale), _ptr(y),
                                             _ptr(yt), _ptr(amax), _ptr(scale_inv), _ptr(noop_flag),
                                             _stream(stream)))


def fp8_cast_transpose_amax_pair(xa, xb, fmt, scale_a, ya, scale_b, yb, yt_a=None, amax_a=None, scale_inv_a=None,
                                 yt_b=None, amax_b=None, scale_inv_b=None, noop_b=None, stream=None):
    """Two casts of one dtype and format (b optionally skipped by a device
    flag), one launch where both suit it."""
    if xa.dtype != xb.dtype:
        raise TypeError("fp8_cast_transpose_amax_pair: both inputs must have one dtype")
    ra, ca = xa.shape
    rb, cb = xb.shape
    _check(_lib.fp8_cast_transpose_amax_pair(_ptr(xa), ra, ca, _ptr(scale_a), _ptr(ya), _ptr(yt_a), _ptr(amax_a),
                                             _ptr(scale_inv_a), _ptr(xb), rb, cb, _ptr(scale_b), _ptr(yb),
                                             _ptr(yt_b), _ptr(amax_b), _ptr(scale_inv_b), _ptr(noop_b),
                                             _dtype(xa), _fmt(fmt), _stream(stream)))


def cast_job(x, fmt, scale, y, yt=None, amax=None, scale_inv=None, noop_flag=None):
    """One job record of fp8_cast_transpose_amax_multi / the extra casts of
    fp8_linear_refresh_weights: the arguments of fp8_cast_transpose_amax_noop
    (x 2-D; a 1-D x is cast as one row)."""
    rows, cols = (x.shape[0], x.shape[1]) if x.dim() == 2 else (1, x.numel())
    return _CastJob(_ptr(x), _dtype(x), rows, cols, _fmt(fmt), _ptr(scale), _ptr(y), _ptr(yt), _ptr(amax),
                    _ptr(scale_inv), _ptr(noop_flag))


def _job_array(jobs):
    if isinstance(jobs, ctypes.Array):
        return jobs
    return (_CastJob * len(jobs))(*jobs) if len(jobs) else None


def cast_jobs(jobs):
    """A reusable job array (list of cast_job records -> ctypes array), so that
    repeated calls skip the marshalling."""
    return (_CastJob * len(jobs))(*jobs)


def fp8_cast_transpose_amax_multi(jobs, stream=None):
    """Many casts in one launch; jobs: cast_job records or a cast_jobs array."""
    arr = _job_array(jobs)
    _check(_lib.fp8_cast_transpose_amax_multi(arr, 0 if arr is None else len(arr), _stream(stream)))


def fp8_cast_transpose_amax_dynamic(x, fmt, scale, y, yt=None, amax=None, scale_inv=None, stream=None):
    """Dynamic scaling: amax of x, scale = fp8_max / amax (scale is in/out), cast."""
    rows, cols = x.shape
    _check(_lib.fp8_cast_transpose_amax_dynamic(_ptr(x), _dtype(x), rows, cols, _fmt(fmt), _ptr(scale), _ptr(y),
                                                _ptr(yt), _ptr(amax), _ptr(scale_inv), _stream(stream)))


def fp8_transpose(y, yt, stream=None):
    rows, cols = y.shape
    _check(_lib.fp8_transpose(_ptr(y), rows, cols, _ptr(yt), _stream(stream)))


def fp8_update_scales(amax_history, scale, scale_inv, formats, algo=AMAX_MAX, stream=None):
    hist_len, num_tensors = amax_history.shape
    _check(_lib.fp8_update_scales(num_tensors, hist_len, _ptr(amax_history), _ptr(scale),
                                  _ptr(scale_inv), _ptr(formats), algo, _stream(stream)))


def fp8_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, d, bias=None, stream=None):
    m, k = a.shape
    n = b.shape[0]
    _check(_lib.fp8_gemm(_ptr(a), _fmt(a_fmt), _ptr(a_scale_inv), _ptr(b), _fmt(b_fmt),
                         _ptr(b_scale_inv), _ptr(bias), F32 if bias is None else _dtype(bias),
                         _ptr(d), _dtype(d), m, n, k, _stream(stream)))


def fp8_gemm_ex(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, d, bias=None, workspace=None,
                stream=None):
    m, k = a.shape
    n = b.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.fp8_gemm_ex(_ptr(a), _fmt(a_fmt), _ptr(a_scale_inv), _ptr(b), _fmt(b_fmt),
                            _ptr(b_scale_inv), _ptr(bias), F32 if bias is None else _dtype(bias),
                            _ptr(d), _dtype(d), m, n, k, _ptr(workspace), ws_bytes, _stream(stream)))


def fp8_gemm_noalloc(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, d, bias=None, stream=None):
    m, k = a.shape
    n = b.shape[0]
    _check(_lib.fp8_gemm_noalloc(_ptr(a), _fmt(a_fmt), _ptr(a_scale_inv), _ptr(b), _fmt(b_fmt),
                                 _ptr(b_scale_inv), _ptr(bias), F32 if bias is None else _dtype(bias),
                                 _ptr(d), _dtype(d), m, n, k, _stream(stream)))


def fp8_gemm_cast(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, out_fmt, out_scale, d8, d8t=None,
                  out_amax=None, out_scale_inv=None, bias=None, a_major="k", b_major="k", stream=None):
    """GEMM with an FP8 output; a is [m, k] ("k") or [k, m] ("mn"), b is
    [n, k] ("k") or [k, n] ("mn")."""
    am, bm = _MAJOR[a_major], _MAJOR[b_major]
    m = a.shape[1] if am == MN_MAJOR else a.shape[0]
    k = a.shape[0] if am == MN_MAJOR else a.shape[1]
    n = b.shape[1] if bm == MN_MAJOR else b.shape[0]
    _check(_lib.fp8_gemm_cast(_ptr(a), _fmt(a_fmt), am, _ptr(a_scale_inv), _ptr(b), _fmt(b_fmt), bm,
                              _ptr(b_scale_inv), _ptr(bias), F32 if bias is None else _dtype(bias), m, n, k,
                              _fmt(out_fmt), _ptr(out_scale), _ptr(d8), _ptr(d8t), _ptr(out_amax),
                              _ptr(out_scale_inv), _stream(stream)))


def fp8_gemm_workspace_size():
    n = ctypes.c_size_t(0)
    _check(_lib.fp8_gemm_workspace_size(ctypes.byref(n)))
    return n.value


def fp8_gemm_plan(m, n, k):
    """The GEMM's tile schedule on the current device: dict with pair,
    m_sub, tiles, stream_k (taken with a workspace) and resident pairs."""
    info = (ctypes.c_int64 * 5)()
    _check(_lib.fp8_gemm_plan(m, n, k, info))
    return {"pair": bool(info[0]), "m_sub": int(info[1]), "tiles": int(info[2]), "stream_k": bool(info[3]),
            "resident": int(info[4])}


def gemm_workspace(device="cuda"):
    """A zero-filled workspace of fp8_gemm_workspace_size() bytes (uint8 tensor)."""
    return torch.zeros(fp8_gemm_workspace_size(), dtype=torch.uint8, device=device)


class Fp8Meta:
    """Packed DelayedScaling state of T FP8 tensors (caller-owned CUDA tensors)."""

    def __init__(self, formats, hist_len=16, device="cuda"):
        self.formats = torch.tensor([_fmt(f) for f in formats], dtype=torch.uint8, device=device)
        T = self.formats.numel()
        self.amax_history = torch.zeros(hist_len, T, dtype=torch.float32, device=device)
        self.scale = torch.ones(T, dtype=torch.float32, device=device)
        self.scale_inv = torch.ones(T, dtype=torch.float32, device=device)
        self._c = _Meta(_ptr(self.amax_history), _ptr(self.scale), _ptr(self.scale_inv),
                        _ptr(self.formats), T, hist_len)

    @property
    def num_tensors(self):
        return self.formats.numel()

    def update(self, algo=AMAX_MAX, stream=None):
        fp8_update_scales(self.amax_history, self.scale, self.scale_inv, self.formats, algo=algo,
                          stream=stream)


class Fp8Linear:
    """A linear layer's fp32 master weight, optional bias and FP8 weight cache."""

    def __init__(self, w, bias, meta_in, meta_w, meta_grad, workspace=None, w_noop_flag=None, transpose=True):
        """w_noop_flag: optional device int32 tensor; when given, the forward
        always enqueues the weight cast and the GPU skips it while the flag is
        non-zero (graph-capturable weight caching)."""
        out_f, in_f = w.shape
        self.w = w
        self.bias = bias
        self.workspace = workspace
        self.w_noop_flag = w_noop_flag
        self.w8 = torch.empty(out_f, in_f, dtype=torch.uint8, device=w.device)
        # transpose=False: no cached weight transpose (the backward reads w8 MN-major)
        self.w8t = torch.empty(in_f, out_f, dtype=torch.uint8, device=w.device) if transpose else None
        self.w_scale_inv = torch.ones(1, dtype=torch.float32, device=w.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        self._c = _Linear(_ptr(w), _ptr(bias), F32 if bias is None else _dtype(bias), in_f, out_f,
                          _ptr(self.w8), _ptr(self.w8t), _ptr(self.w_scale_inv),
                          meta_in, meta_w, meta_grad, 0, _ptr(workspace), ws_bytes, _ptr(w_noop_flag))

    @property
    def in_features(self):
        return self._c.in_features

    @property
    def out_features(self):
        return self._c.out_features

    @property
    def cache_valid(self):
        return bool(self._c.cache_valid)

    def invalidate_cache(self):
        self._c.cache_valid = 0


class LinearGroup:
    """Handles of several Fp8Linear layers as the C array that
    fp8_linear_refresh_weights takes (built once, reused every step)."""

    def __init__(self, lins):
        self.lins = list(lins)
        self._arr = (ctypes.POINTER(_Linear) * len(self.lins))(*[ctypes.pointer(l._c) for l in self.lins])

    def __len__(self):
        return len(self.lins)


def fp8_linear_refresh_weights(lins, meta, extra=(), stream=None):
    """Recast the FP8 weight caches of all `lins` (an LinearGroup or a list of
    Fp8Linear) and the `extra` casts (cast_job records or a cast_jobs array)
    in one launch; the forwards that follow pass is_first_microbatch=False."""
    group = lins if isinstance(lins, LinearGroup) else LinearGroup(lins)
    ex = _job_array(extra)
    _check(_lib.fp8_linear_refresh_weights(group._arr, len(group), ctypes.byref(meta._c), ex,
                                           0 if ex is None else len(ex), _stream(stream)))


def fp8_linear_fwd(lin, meta, x, y, is_first_microbatch, x8, x8t=None, x_scale_inv=None,
                   stream=None):
    flag = -1 if is_first_microbatch is None else (1 if is_first_microbatch else 0)
    _check(_lib.fp8_linear_fwd(ctypes.byref(lin._c), ctypes.byref(meta._c), _ptr(x), _dtype(x),
                               x.shape[0], _ptr(y), _dtype(y), flag, _ptr(x8), _ptr(x8t),
                               _ptr(x_scale_inv), _stream(stream)))


def fp8_linear_bwd(lin, meta, dy, x8t, x_scale_inv, dw, dy8, dy8t, dy_scale_inv, dx=None,
                   stream=None):
    _check(_lib.fp8_linear_bwd(ctypes.byref(lin._c), ctypes.byref(meta._c), _ptr(dy), _dtype(dy),
                               dy.shape[0], _ptr(x8t), _ptr(x_scale_inv), _ptr(dx),
                               BF16 if dx is None else _dtype(dx), _ptr(dw), _ptr(dy8),
                               _ptr(dy8t), _ptr(dy_scale_inv), _stream(stream)))


def _io(in_cast, out_meta, out8, out8t, out_scale_inv):
    return _Fp8Io(1 if in_cast else 0, -1 if out_meta is None else int(out_meta), _ptr(out8), _ptr(out8t),
                  _ptr(out_scale_inv))


def fp8_linear_fwd_ex(lin, meta, x, y, is_first_microbatch, x8, x8t=None, x_scale_inv=None, in_cast=False,
                      out_meta=None, out8=None, out8t=None, out_scale_inv=None, stream=None):
    """fp8_linear_fwd with FP8 hand-over: in_cast -> x8/x8t/x_scale_inv already
    hold the cast input (x may be None); out_meta -> the output is cast in the
    GEMM epilogue into out8/out8t/out_scale_inv (y may be None)."""
    flag = -1 if is_first_microbatch is None else (1 if is_first_microbatch else 0)
    io = _io(in_cast, out_meta, out8, out8t, out_scale_inv)
    _check(_lib.fp8_linear_fwd_ex(ctypes.byref(lin._c), ctypes.byref(meta._c), _ptr(x),
                                  F32 if x is None else _dtype(x), x8.shape[0], _ptr(y),
                                  BF16 if y is None else _dtype(y), flag, _ptr(x8), _ptr(x8t),
                                  _ptr(x_scale_inv), ctypes.byref(io), _stream(stream)))


def fp8_linear_bwd_ex(lin, meta, dy, x8t, x_scale_inv, dw, dy8, dy8t, dy_scale_inv, dx=None, in_cast=False,
                      out_meta=None, out8=None, out8t=None, out_scale_inv=None, x8=None, stream=None):
    """fp8_linear_bwd with FP8 hand-over: in_cast -> dy8/dy8t/dy_scale_inv
    already hold the cast gradient (dy may be None); out_meta -> the dgrad is
    cast in the GEMM epilogue into out8/out8t/out_scale_inv.  Transposes are
    optional: x8t None -> the wgrad reads x8; dy8t None -> it reads dy8; a
    linear without w8t -> the dgrad reads w8 (all MN-major)."""
    io = _io(in_cast, out_meta, out8, out8t, out_scale_inv)
    _check(_lib.fp8_linear_bwd_ex(ctypes.byref(lin._c), ctypes.byref(meta._c), _ptr(dy),
                                  BF16 if dy is None else _dtype(dy), dy8.shape[0], _ptr(x8), _ptr(x8t),
                                  _ptr(x_scale_inv), _ptr(dx), BF16 if dx is None else _dtype(dx), _ptr(dw),
                                  _ptr(dy8), _ptr(dy8t), _ptr(dy_scale_inv), ctypes.byref(io), _stream(stream)))



def fp8_gemm_major(a, a_fmt, a_major, a_scale_inv, b, b_fmt, b_major, b_scale_inv, d, bias=None, stream=None):
    """D[m, n] = A(m, k) B(n, k) scaled; a is [m, k] ("k") or [k, m] ("mn"),
    b is [n, k] ("k") or [k, n] ("mn")."""
    am, bm = _MAJOR[a_major], _MAJOR[b_major]
    m = a.shape[1] if am == MN_MAJOR else a.shape[0]
    k = a.shape[0] if am == MN_MAJOR else a.shape[1]
    n = b.shape[1] if bm == MN_MAJOR else b.shape[0]
    _check(_lib.fp8_gemm_major(_ptr(a), _fmt(a_fmt), am, _ptr(a_scale_inv), _ptr(b), _fmt(b_fmt), bm,
                               _ptr(b_scale_inv), _ptr(bias), F32 if bias is None else _dtype(bias), _ptr(d),
                               _dtype(d), m, n, k, _stream(stream)))


def fp8ds_device_status(clear=True):
    code = _I32(0)
    _check(_lib.fp8ds_device_status(ctypes.byref(code), 1 if clear else 0))
    return code.value
