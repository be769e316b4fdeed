"""The C ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before any launch (no GPU needed: the
argument checks run before the first CUDA call)."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "fp8ds.h")


@pytest.fixture(scope="module")
def lib():
    from fp8_delayed_scaling_cast_b200 import build
    build.build()
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(fp8\w*)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("fp8_quantize", "fp8_cast_transpose_amax", "fp8_update_scales", "fp8_gemm",
              "fp8_gemm_ex", "fp8_gemm_workspace_size", "fp8_gemm_noalloc", "fp8_gemm_cast",
              "fp8_linear_fwd_ex", "fp8_linear_bwd_ex", "fp8_cast_transpose_amax_noop",
              "fp8_cast_transpose_amax_pair",
              "fp8_cast_transpose_amax_dynamic", "fp8_transpose", "fp8_gemm_major",
              "fp8_linear_fwd", "fp8_linear_bwd", "fp8ds_last_error", "fp8ds_device_status",
              "fp8ds_version", "fp8_cast_transpose_amax_multi", "fp8_linear_refresh_weights",
              "fp8_gemm_plan"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(raw, n), n


def test_version(lib):
    assert "sm_100a" in lib.fp8ds_version()


P = ctypes.c_void_p
FAKE = P(0x10000)          # never dereferenced: every call below fails its checks first
FAKE_ODD = P(0x10001)


def test_gemm_argument_checks(lib):
    L = lib._lib
    s = P(0)
    ok_args = dict(a=FAKE, fa=0, sa=FAKE, b=FAKE, fb=0, sb=FAKE, bias=None, bt=0, d=FAKE, dt=1,
                   m=128, n=256, k=128)

    def call(**kw):
        a = dict(ok_args)
        a.update(kw)
        return L.fp8_gemm(a["a"], a["fa"], a["sa"], a["b"], a["fb"], a["sb"], a["bias"], a["bt"],
                          a["d"], a["dt"], a["m"], a["n"], a["k"], s)

    assert call(k=120) == lib.ERR_INVALID_ARG and "multiple of 16" in lib.fp8ds_last_error()
    assert call(a=None) == lib.ERR_INVALID_ARG
    assert call(m=0) == lib.ERR_INVALID_ARG
    assert call(n=12) == lib.ERR_INVALID_ARG           # bf16 output needs n % 8 == 0
    assert call(a=FAKE_ODD) == lib.ERR_INVALID_ARG and "aligned" in lib.fp8ds_last_error()
    assert call(fa=7) == lib.ERR_INVALID_ARG
    assert call(m=1 << 31) == lib.ERR_INVALID_ARG
    # the allocation-free variant checks the same arguments before anything else
    assert L.fp8_gemm_noalloc(FAKE, 0, FAKE, FAKE, 0, FAKE, None, 0, FAKE, 1, 128, 256, 120, s) == \
        lib.ERR_INVALID_ARG and "multiple of 16" in lib.fp8ds_last_error()
    # the workspace variant checks the same arguments plus the workspace alignment
    assert L.fp8_gemm_ex(FAKE, 0, FAKE, FAKE, 0, FAKE, None, 0, FAKE, 1, 128, 256, 120, FAKE, 64, s) == \
        lib.ERR_INVALID_ARG
    assert L.fp8_gemm_ex(FAKE, 0, FAKE, FAKE, 0, FAKE, None, 0, FAKE, 1, 128, 256, 128, FAKE_ODD, 64, s) == \
        lib.ERR_INVALID_ARG and "workspace" in lib.fp8ds_last_error()
    # the schedule query checks its arguments before it asks the device
    info = (ctypes.c_int64 * 5)()
    assert L.fp8_gemm_plan(128, 256, 128, None) == lib.ERR_INVALID_ARG
    assert L.fp8_gemm_plan(0, 256, 128, info) == lib.ERR_INVALID_ARG and "positive" in lib.fp8ds_last_error()


def test_cast_and_update_argument_checks(lib):
    L = lib._lib
    s = P(0)
    assert L.fp8_quantize(None, 0, 16, 0, FAKE, FAKE, None, None, s) == lib.ERR_INVALID_ARG
    assert L.fp8_quantize(FAKE, 0, -1, 0, FAKE, FAKE, None, None, s) == lib.ERR_INVALID_ARG
    assert L.fp8_quantize(FAKE, 0, 16, 3, FAKE, FAKE, None, None, s) == lib.ERR_INVALID_ARG
    assert L.fp8_quantize(FAKE, 5, 16, 0, FAKE, FAKE, None, None, s) == lib.ERR_INVALID_ARG
    assert L.fp8_cast_transpose_amax(FAKE, 0, 4, -4, 0, FAKE, FAKE, None, None, None, s) == lib.ERR_INVALID_ARG
    assert L.fp8_cast_transpose_amax(FAKE, 0, 4, 4, 0, None, FAKE, None, None, None, s) == lib.ERR_INVALID_ARG
    # the pair call checks both tensors before anything is launched
    pair_ok = [FAKE, 16, 16, FAKE, FAKE, None, None, None, FAKE, 16, 16, FAKE, FAKE, None, None, None, None, 0, 0, s]

    def pair(**kw):
        a = list(pair_ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return L.fp8_cast_transpose_amax_pair(*a)
    assert pair(a10=-16) == lib.ERR_INVALID_ARG and "(b)" in lib.fp8ds_last_error()
    assert pair(a3=None) == lib.ERR_INVALID_ARG and "(a)" in lib.fp8ds_last_error()
    assert pair(a12=None) == lib.ERR_INVALID_ARG and "(b)" in lib.fp8ds_last_error()
    assert pair(a17=5) == lib.ERR_INVALID_ARG
    assert pair(a18=4) == lib.ERR_INVALID_ARG
    assert L.fp8_update_scales(-1, 16, FAKE, FAKE, FAKE, FAKE, 0, s) == lib.ERR_INVALID_ARG
    assert L.fp8_update_scales(4, 0, FAKE, FAKE, FAKE, FAKE, 0, s) == lib.ERR_INVALID_ARG
    assert L.fp8_update_scales(4, 16, None, FAKE, FAKE, FAKE, 0, s) == lib.ERR_INVALID_ARG
    assert L.fp8_update_scales(4, 16, FAKE, FAKE, FAKE, FAKE, 2, s) == lib.ERR_UNSUPPORTED
    # zero tensors: nothing to do, nothing launched
    assert L.fp8_update_scales(0, 16, None, None, None, None, 0, s) == lib.OK


def test_linear_argument_checks(lib):
    L = lib._lib
    s = P(0)
    meta = lib._Meta(FAKE, FAKE, FAKE, FAKE, 3, 16)
    lin = lib._Linear(FAKE, None, 0, 256, 512, FAKE, FAKE, FAKE, 0, 1, 2, 0, None, 0)
    r = L.fp8_linear_fwd(ctypes.byref(lin), ctypes.byref(meta), FAKE, 0, 128, FAKE, 0, 2, FAKE,
                         FAKE, FAKE, s)
    assert r == lib.ERR_INVALID_ARG and "is_first_microbatch" in lib.fp8ds_last_error()
    bad = lib._Linear(FAKE, None, 0, 256, 512, FAKE, FAKE, FAKE, 0, 7, 2, 0, None, 0)
    r = L.fp8_linear_fwd(ctypes.byref(bad), ctypes.byref(meta), FAKE, 0, 128, FAKE, 0, 1, FAKE,
                         FAKE, FAKE, s)
    assert r == lib.ERR_INVALID_ARG and "out of range" in lib.fp8ds_last_error()
    r = L.fp8_linear_fwd(ctypes.byref(lin), ctypes.byref(meta), FAKE, 0, 128, FAKE, 0, 1, FAKE,
                         FAKE, None, s)
    assert r == lib.ERR_INVALID_ARG
    # backward before any forward: the cache is empty
    r = L.fp8_linear_bwd(ctypes.byref(lin), ctypes.byref(meta), FAKE, 1, 128, FAKE, FAKE, FAKE, 1,
                         FAKE, FAKE, FAKE, FAKE, s)
    assert r == lib.ERR_INVALID_ARG and "cache" in lib.fp8ds_last_error()


def test_gemm_cast_argument_checks(lib):
    """The FP8-output GEMM: codes need n % 16 (row pitch) and, with the
    transpose, m % 16; the output format must be known; the scale and the
    output must not be NULL.  Every call below fails a check (no launch)."""
    L = lib._lib
    s = P(0)

    def call(m=128, n=256, k=128, fmt=0, scale=FAKE, d8=FAKE, d8t=None, am=0):
        return L.fp8_gemm_cast(FAKE, 0, am, FAKE, FAKE, 0, 0, FAKE, None, 0, m, n, k, fmt, scale, d8, d8t, None, None,
                               s)

    assert call(n=264) == lib.ERR_INVALID_ARG and "multiple of 16" in lib.fp8ds_last_error()
    assert call(m=120, d8t=FAKE) == lib.ERR_INVALID_ARG and "transposed" in lib.fp8ds_last_error()
    assert call(fmt=5) == lib.ERR_INVALID_ARG and "format" in lib.fp8ds_last_error()
    assert call(scale=None) == lib.ERR_INVALID_ARG
    assert call(d8=None) == lib.ERR_INVALID_ARG
    assert call(d8t=FAKE_ODD) == lib.ERR_INVALID_ARG and "aligned" in lib.fp8ds_last_error()
    assert call(k=120) == lib.ERR_INVALID_ARG
    assert call(am=3) == lib.ERR_INVALID_ARG and "layout" in lib.fp8ds_last_error()


def test_linear_ex_argument_checks(lib):
    """FP8 hand-over options of the _ex linear calls (every call fails a check)."""
    L = lib._lib
    s = P(0)
    meta = lib._Meta(FAKE, FAKE, FAKE, FAKE, 4, 16)
    lin = lib._Linear(FAKE, None, 0, 256, 520, FAKE, FAKE, FAKE, 0, 1, 2, 0, None, 0)

    def fwd(io, x=FAKE, y=FAKE, lin_=lin):
        return L.fp8_linear_fwd_ex(ctypes.byref(lin_), ctypes.byref(meta), x, 0, 128, y, 1, 1, FAKE, FAKE, FAKE,
                                   ctypes.byref(io), s)

    # output meta out of range
    assert fwd(lib._Fp8Io(0, 9, FAKE, FAKE, FAKE)) == lib.ERR_INVALID_ARG and "out of range" in lib.fp8ds_last_error()
    # without in_cast the input must be given
    assert fwd(lib._Fp8Io(0, -1, None, None, None), x=None) == lib.ERR_INVALID_ARG
    # FP8 output requested but no buffer for it
    assert fwd(lib._Fp8Io(0, 3, None, None, None)) == lib.ERR_INVALID_ARG
    # 520 output features: bf16 is fine (n % 8) but FP8 codes need n % 16
    assert fwd(lib._Fp8Io(1, 3, FAKE, None, FAKE), x=None, y=None) == lib.ERR_INVALID_ARG and \
        "multiple of 16" in lib.fp8ds_last_error()

    def bwd(io, lin_, dy=FAKE, m=128):
        return L.fp8_linear_bwd_ex(ctypes.byref(lin_), ctypes.byref(meta), dy, 1, m, None, FAKE, FAKE, FAKE, 1,
                                   FAKE, FAKE, FAKE, FAKE, ctypes.byref(io), s)

    assert bwd(lib._Fp8Io(0, -1, None, None, None), lin) == lib.ERR_INVALID_ARG and \
        "cache" in lib.fp8ds_last_error()
    cached = lib._Linear(FAKE, None, 0, 256, 512, FAKE, FAKE, FAKE, 0, 1, 2, 1, None, 0)
    # without in_cast the gradient must be given
    assert bwd(lib._Fp8Io(0, -1, None, None, None), cached, dy=None) == lib.ERR_INVALID_ARG
    # transposed FP8 dgrad needs m % 16
    assert bwd(lib._Fp8Io(1, 3, FAKE, FAKE, FAKE), cached, dy=None, m=120) == lib.ERR_INVALID_ARG and \
        "transposed" in lib.fp8ds_last_error()
    assert bwd(lib._Fp8Io(1, 11, FAKE, FAKE, FAKE), cached, dy=None) == lib.ERR_INVALID_ARG and \
        "out of range" in lib.fp8ds_last_error()


def test_gemm_major_argument_checks(lib):
    """Operand layouts: an MN-major a needs m % 16, an MN-major b needs n % 16,
    k % 16 only with a K-major operand; unknown layouts are refused.  Every
    call below fails a check (no launch)."""
    L = lib._lib
    s = P(0)

    def call(am=0, bm=0, m=128, n=256, k=128):
        return L.fp8_gemm_major(FAKE, 0, am, FAKE, FAKE, 0, bm, FAKE, None, 0, FAKE, 1, m, n, k, s)

    assert call(am=2) == lib.ERR_INVALID_ARG and "layout" in lib.fp8ds_last_error()
    assert call(am=1, m=120) == lib.ERR_INVALID_ARG and "MN-major a" in lib.fp8ds_last_error()
    assert call(bm=1, n=264) == lib.ERR_INVALID_ARG and "MN-major b" in lib.fp8ds_last_error()
    assert call(am=0, bm=1, k=120) == lib.ERR_INVALID_ARG and "K-major" in lib.fp8ds_last_error()
    assert call(am=1, bm=1, k=120, n=12) == lib.ERR_INVALID_ARG   # k is free, but n % 16 is not met


def test_header_is_plain_c(tmp_path):
    """include/fp8ds.h compiles as strict C99 and as C++ on its own (no CUDA
    or torch headers), so any C caller can use the boundary."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    src = tmp_path / "use_header.c"
    src.write_text('#include "fp8ds.h"\nint main(void) { return fp8_gemm_workspace_size(0) == FP8DS_OK; }\n')
    for lang, std in (("c", "-std=c99"), ("c++", "-std=c++17")):
        r = subprocess.run([cc, "-x", lang, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I" + inc, "-c",
                            str(src), "-o", str(tmp_path / ("o_" + lang.replace("+", "p")))],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls_the_library(tmp_path, lib):
    """A plain C program links libfp8ds.so and gets its version string and
    an argument-check error (host-only paths: no device is touched)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(lib.LIB_PATH)
    src = tmp_path / "client.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "fp8ds.h"
int main(void) {
    float scale = 1.0f;
    unsigned char y[16];
    float x[16] = {0};
    fp8ds_status st = fp8_cast_transpose_amax(x, FP8DS_F32, 4, -4, FP8DS_E4M3, &scale, y, NULL, NULL, NULL, NULL);
    printf("%s|%d|%s\n", fp8ds_version(), (int)st, fp8ds_last_error());
    return st == FP8DS_ERR_INVALID_ARG && strlen(fp8ds_last_error()) > 0 ? 0 : 1;
}
''')
    exe = tmp_path / "client"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I" + inc, str(src), "-o", str(exe), "-L" + libdir,
                        "-l:libfp8ds.so", "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    version, status, msg = r.stdout.strip().split("|")
    assert "sm_100a" in version and int(status) == lib.ERR_INVALID_ARG and "negative" in msg


def test_multi_cast_and_refresh_argument_checks(lib):
    """The multi-tensor cast and the weight-cache refresh check every job (and
    every handle) before anything is launched, and name the bad job."""
    L = lib._lib
    s = P(0)
    good = lib._CastJob(FAKE, 0, 64, 32, 0, FAKE, FAKE, None, None, None, None)
    jobs = (lib._CastJob * 3)(good, good, good)
    jobs[2].scale = None
    assert L.fp8_cast_transpose_amax_multi(jobs, 3, s) == lib.ERR_INVALID_ARG
    assert "job 2" in lib.fp8ds_last_error()
    jobs[2].scale = FAKE
    jobs[1].rows = -1
    assert L.fp8_cast_transpose_amax_multi(jobs, 3, s) == lib.ERR_INVALID_ARG
    assert "job 1" in lib.fp8ds_last_error()
    jobs[1].rows = 64
    jobs[0].fmt = 7
    assert L.fp8_cast_transpose_amax_multi(jobs, 3, s) == lib.ERR_INVALID_ARG
    jobs[0].fmt = 0
    jobs[0].yt = FAKE
    jobs[0].rows = 1 << 31
    assert L.fp8_cast_transpose_amax_multi(jobs, 3, s) == lib.ERR_INVALID_ARG and "2^31" in lib.fp8ds_last_error()
    assert L.fp8_cast_transpose_amax_multi(None, 2, s) == lib.ERR_INVALID_ARG
    assert L.fp8_cast_transpose_amax_multi(jobs, -1, s) == lib.ERR_INVALID_ARG
    assert L.fp8_cast_transpose_amax_multi(None, 0, s) == lib.OK          # nothing to do
    # refresh: an incomplete handle or a bad meta index rejects the whole call
    # and leaves every cache flag as it was
    meta = lib._Meta(FAKE, FAKE, FAKE, FAKE, 6, 16)
    la = lib._Linear(FAKE, None, 0, 256, 512, FAKE, None, FAKE, 0, 1, 2, 0, None, 0)
    lb = lib._Linear(FAKE, None, 0, 512, 256, None, None, FAKE, 3, 4, 5, 0, None, 0)
    arr = (ctypes.POINTER(lib._Linear) * 2)(ctypes.pointer(la), ctypes.pointer(lb))
    assert L.fp8_linear_refresh_weights(arr, 2, ctypes.byref(meta), None, 0, s) == lib.ERR_INVALID_ARG
    assert "handle 1" in lib.fp8ds_last_error() and la.cache_valid == 0
    lb.w8 = FAKE
    lb.meta_w = 6
    assert L.fp8_linear_refresh_weights(arr, 2, ctypes.byref(meta), None, 0, s) == lib.ERR_INVALID_ARG
    assert "out of range" in lib.fp8ds_last_error() and la.cache_valid == 0
    lb.meta_w = 4
    bad_extra = (lib._CastJob * 1)(lib._CastJob(None, 0, 64, 32, 0, FAKE, FAKE, None, None, None, None))
    assert L.fp8_linear_refresh_weights(arr, 2, ctypes.byref(meta), bad_extra, 1, s) == lib.ERR_INVALID_ARG
    assert "job 2" in lib.fp8ds_last_error() and la.cache_valid == 0 and lb.cache_valid == 0
    assert L.fp8_linear_refresh_weights(None, 1, ctypes.byref(meta), None, 0, s) == lib.ERR_INVALID_ARG
