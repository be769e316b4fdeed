"""Build libfp8ds.so in-tree with nvcc for sm_100a.

Usage: python -m fp8_delayed_scaling_cast_b200.build [--force]

The library is compiled without fast-math (IEEE division/reciprocal and no
flush-to-zero, which the bit-exact cast and scale update rely on) and links
the CUDA runtime statically, so it loads beside any PyTorch build.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfp8ds.so")
SOURCES = ["api.cu", "cast.cu", "update.cu", "gemm_sm100.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, "fp8ds_internal.h"), os.path.join(CSRC, "ptx_sm100.cuh"),
              os.path.join(INCLUDE, "fp8ds.h")]
    return files


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force=False, verbose=False, extra=()):
    if not force and up_to_date():
        return LIB
    build_dir = os.path.join(PKG, "_build")
    os.makedirs(build_dir, exist_ok=True)
    objs = []
    common = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-I" + INCLUDE, "-I" + CSRC, "--expt-relaxed-constexpr", *extra]
    for s in SOURCES:
        obj = os.path.join(build_dir, s.replace(".cu", ".o"))
        cmd = common + ["-c", os.path.join(CSRC, s), "-o", obj]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [_nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force or bool(extra), verbose=True, extra=extra))
