"""fp8_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Such callers (a program whose device memory all belongs to a framework's
caching allocator or was reserved by a serving engine at start-up, or C code
that only receives tensor pointers) get the same GEMM with its split-tile
scratch taken from an array inside the library.  This file is collected last
so that a run stopping at the first failure has run every other test; it
passes alone in a fresh process as well.

The shapes below leave a ragged last wave of CTA pairs on a B200, so the
scratch is really used (256-row and 512-row pair tiles); the test asks the
library's own schedule (fp8_gemm_plan) whether the shape takes the split
tiles on this device before it runs.  The
output of two consecutive calls is compared with fp8_gemm (the existing entry
point) within the tolerances of the other GEMM tests; the two calls also show
that a call starts from whatever the previous one left in the shared scratch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import (abs_dot, accumulation_allowance, bf16_ulp, check_gemm_bf16, check_gemm_fp32, dev,
                            host_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _operands(M, N, K, seed):
    g = inputs.gen(seed)
    x = inputs.uniform((M, K), g)
    w = inputs.normal((N, K), g, 0.02)
    sx = np.float32(448.0) / np.float32(np.abs(x.numpy()).max())
    sw = np.float32(448.0) / np.float32(np.abs(w.numpy()).max())
    a, _, _, sa = o.cast_transpose_amax(x.numpy(), o.E4M3, sx, transpose=False)
    b, _, _, sb = o.cast_transpose_amax(w.numpy(), o.E4M3, sw, transpose=False)
    return a, b, np.float32(sa), np.float32(sb)


def _call_noalloc(fp8, a, sa, b, sb, d):
    """Straight through the C ABI (argument marshalling only)."""
    M, K = a.shape
    N = b.shape[0]
    P = ctypes.c_void_p
    st = fp8._lib.fp8_gemm_noalloc(P(a.data_ptr()), fp8.E4M3, P(sa.data_ptr()), P(b.data_ptr()), fp8.E4M3,
                                   P(sb.data_ptr()), None, fp8.F32, P(d.data_ptr()), fp8._dtype(d), M, N, K,
                                   P(torch.cuda.current_stream().cuda_stream))
    assert st == fp8.OK, fp8.fp8ds_last_error()


@pytest.mark.parametrize("shape", [(4096, 2048, 1024), (7168, 2048, 2048)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_fp8_gemm_twice(fp8, shape, out_dtype):
    M, N, K = shape
    # The split-tile schedule (and with it the static scratch) is taken only
    # when whole tiles leave a ragged last wave worth balancing; the library's
    # own plan says whether this shape does on this device (on the 74 CTA
    # pairs of a B200 both shapes do: 128 and 112 tiles).
    plan = fp8.fp8_gemm_plan(M, N, K)
    if not plan["stream_k"]:
        assert plan["resident"] != 74, plan
        pytest.skip("%d tiles on %d CTA pairs: no split tiles, the scratch would not be used"
                    % (plan["tiles"], plan["resident"]))
    a, b, sa, sb = _operands(M, N, K, seed=31)
    ad, bd = dev(a), dev(b)
    sad = torch.tensor([sa], device="cuda")
    sbd = torch.tensor([sb], device="cuda")
    ref = torch.empty(M, N, dtype=out_dtype, device="cuda")
    fp8.fp8_gemm(ad, "e4m3", sad, bd, "e4m3", sbd, ref)
    torch.cuda.synchronize()
    rows = np.array(sorted({0, 1, 255, 256, 511, 512, M // 2, M - 1} |
                           set(np.random.default_rng(M).integers(0, M, 24).tolist())), np.int64)
    exact = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    absdot = abs_dot(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    for call in range(2):
        d = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        _call_noalloc(fp8, ad, sad, bd, sbd, d)
        torch.cuda.synchronize()
        assert fp8.fp8ds_device_status() == 0
        if out_dtype == torch.float32:
            # against the existing entry point: the fp32 normwise bound
            check_gemm_fp32(d.cpu().numpy(), ref.cpu().double().numpy(), "noalloc vs fp8_gemm, call %d" % call)
            check_gemm_fp32(d.cpu()[torch.from_numpy(rows)].numpy(), exact, "noalloc vs exact, call %d" % call)
        else:
            # within the bf16 bound of the exact result on sampled rows ...
            got_bits = host_bits(d.cpu()[torch.from_numpy(rows)])
            ref_bits = host_bits(ref.cpu()[torch.from_numpy(rows)])
            check_gemm_bf16(got_bits, exact, "noalloc call %d" % call, absdot=absdot, K=K)
            # ... and against the existing entry point: each may sit up to its
            # bound (1 bf16 ulp + the fp32 accumulation allowance) from the
            # exact value, so they agree within twice that
            tol = bf16_ulp(o.round_bf16(exact)) + accumulation_allowance(absdot, K)
            gap = np.abs(o.bf16_bits_to_f32(got_bits).astype(np.float64) -
                         o.bf16_bits_to_f32(ref_bits).astype(np.float64))
            assert np.all(gap <= 2 * tol), "noalloc vs fp8_gemm: %d elements apart" % int((gap > 2 * tol).sum())
