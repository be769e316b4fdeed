"""Full-output integer-exact GEMM checks at the step's full sizes.

Every GEMM launch of the MLP-pair step runs one of the layouts and epilogues
below at 8192 x 8192 x 2048 or 8192 x 2048 x 8192 (the 512-row CTA-pair tile,
many tiles per pair, every tile boundary).  With small integer operands every
partial sum is an integer below 2^24, so the fp32 accumulation is exact in any
order and each output element has exactly one correct value:

* fp32 output: the exact product itself;
* bf16 output: its round-to-nearest-even to bf16 (oracle.round_bf16);
* FP8 output ("Accelerating PyTorch Training Workloads with FP8 -- Part 2",
  torch._scaled_mm with an FP8 out_dtype and output_amax, read as the next
  layer's cast of the bf16 result): oracle.quantize of those bf16 values with
  the delayed scale, and the amax of the bf16 values.

The exact product is the float64 matmul of the decoded integer operands (a
library product, exact here since all values are integers far below 2^53);
on sampled rows it is first checked against the oracle's own fp64 GEMM.  Then
every element of the GPU output is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, assert_f32_bits_equal, dev, host_bits

pytestmark = pytest.mark.gpu

FMT = {"e4m3": o.E4M3, "e5m2": o.E5M2}
SA, SB = 0.5, 4.0            # scale_invs: their product 2 keeps every value an integer


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _int_operand(rows, k, fmt, seed, lim=4):
    """Codes of integers in [-lim, lim] (exact in both formats) and their values."""
    vals = torch.randint(-lim, lim + 1, (rows, k), generator=inputs.gen(seed)).float().numpy()
    return o.encode(vals, FMT[fmt]), vals


def _exact(av, bv, bias=None):
    """(A . B^T) * SA * SB (+ bias) in float64 for integer-valued operands."""
    d = torch.from_numpy(av).double() @ torch.from_numpy(bv).double().T
    d = d.numpy() * (SA * SB)
    if bias is not None:
        d = d + bias.astype(np.float64)[None, :]
    return d


def _pin_rows(a, fa, b, fb, d_exact, bias, seed):
    """The float64 product equals the oracle's GEMM on sampled rows."""
    rows = np.array(sorted({0, 255, 256, 511, 512, d_exact.shape[0] - 1} |
                           set(np.random.default_rng(seed).integers(0, d_exact.shape[0], 6).tolist())), np.int64)
    ref = o.gemm(a, FMT[fa], b, FMT[fb], SA, SB, bias=bias, rows=rows)
    assert np.array_equal(ref, d_exact[rows])


def _stored(codes, major):
    """Operand as the GEMM reads it: [rows, k] (K-major) or [k, rows] (MN-major)."""
    return codes if major == "k" else np.ascontiguousarray(codes.T)


# (M, N, K, a layout, b layout, output, bias): the step's launches --
# fc1 forward / fc2 dgrad shape (K = 2048) and fc2 forward / fc1 dgrad /
# wgrad shapes (K = 8192) in the layouts the step reads.
CASES = [
    (8192, 8192, 2048, "k", "k", "bf16", True),      # fc1 forward shape, bf16 out
    (8192, 2048, 8192, "k", "k", "bf16", True),      # fc2 forward
    (8192, 2048, 8192, "k", "mn", "bf16", False),    # fc1 dgrad (W1 read MN-major)
    (2048, 8192, 8192, "mn", "mn", "f32", False),    # fc2 wgrad
    (8192, 2048, 8192, "mn", "mn", "f32", False),    # fc1 wgrad
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%dx%d-%s%s-%s" % c[:6])
def test_gemm_full_output_integer_exact(fp8, case):
    M, N, K, am, bm, out, with_bias = case
    fa, fb = ("e5m2", "e4m3") if (am, bm) != ("k", "k") else ("e4m3", "e4m3")
    a, av = _int_operand(M, K, fa, seed=M + 3 * K)
    b, bv = _int_operand(N, K, fb, seed=N + 5 * K)
    bias = None
    if with_bias:
        bias = torch.randint(-8, 9, (N,), generator=inputs.gen(11)).float().numpy()
    assert 16 * K < (1 << 24)         # |partial sums| <= 4 * 4 * K: exact in fp32
    d_exact = _exact(av, bv, bias)
    _pin_rows(a, fa, b, fb, d_exact, bias, seed=M + N)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    d = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    sa = torch.tensor([SA], device="cuda")
    sb = torch.tensor([SB], device="cuda")
    fp8.fp8_gemm_major(dev(_stored(a, am)), fa, am, sa, dev(_stored(b, bm)), fb, bm, sb, d,
                       bias=None if bias is None else dev(bias))
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    got = host_bits(d)
    if out == "f32":
        assert_f32_bits_equal(got, d_exact.astype(np.float32), "fp32 out %s" % (case,))
    else:
        assert_bytes_equal(got, o.round_bf16(d_exact), "bf16 out %s" % (case,))


# FP8 output with the 512-row tile (the half-by-half accumulator release):
# fc1 forward (e4m3 x e4m3 + bias -> e4m3) and fc2 dgrad (e5m2 x e4m3 with B
# MN-major -> e5m2).  The results spread about N(0, 600); the delayed scale
# puts about a third of them past fp8_max (saturation), and exact zeros
# occur.
FP8_CASES = [
    (8192, 8192, 2048, "e4m3", "e4m3", "k", "e4m3", 0.75, True),
    (8192, 8192, 2048, "e5m2", "e4m3", "mn", "e5m2", 96.0, False),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: "%s%s-b%s-out%s" % (c[3], c[4], c[5], c[6]))
def test_gemm_fp8_output_full_integer_exact(fp8, case):
    M, N, K, fa, fb, bm, fo, s_out, with_bias = case
    a, av = _int_operand(M, K, fa, seed=71)
    b, bv = _int_operand(N, K, fb, seed=72)
    bias = torch.randint(-8, 9, (N,), generator=inputs.gen(12)).float().numpy() if with_bias else None
    d_exact = _exact(av, bv, bias)
    _pin_rows(a, fa, b, fb, d_exact, bias, seed=73)
    h_bits = o.round_bf16(d_exact)                               # the bf16 result
    want, want_amax, want_si = o.quantize(h_bits, FMT[fo], np.float32(s_out))
    d8 = torch.full((M, N), 0xAA, dtype=torch.uint8, device="cuda")
    amax = torch.zeros(1, device="cuda")
    si = torch.zeros(1, device="cuda")
    fp8.fp8_gemm_cast(dev(a), fa, torch.tensor([SA], device="cuda"), dev(_stored(b, bm)), fb,
                      torch.tensor([SB], device="cuda"), fo, torch.tensor([s_out], device="cuda"), d8, None,
                      amax, si, bias=None if bias is None else dev(bias), b_major=bm)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    got = d8.cpu().numpy()
    # the workload reaches both ends of the format
    fmax_code = 0x7E if fo == "e4m3" else 0x7B
    assert (want & 0x7F == fmax_code).any() and (want & 0x7F == 0).any()
    assert_bytes_equal(got, want, "FP8 out %s" % (case,))
    assert_f32_bits_equal(amax.cpu().numpy(), [want_amax], "FP8 out amax")
    assert_f32_bits_equal(si.cpu().numpy(), [want_si], "FP8 out scale_inv")
