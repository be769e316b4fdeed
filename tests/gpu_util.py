"""Helpers shared by the GPU parity tests: moving seeded inputs to the device
and comparing results with the oracle (no arithmetic of the method here)."""
import numpy as np
import torch

import oracle as o


def dev(a):
    """numpy or torch CPU array -> CUDA tensor (same bytes)."""
    if isinstance(a, np.ndarray):
        a = torch.from_numpy(np.ascontiguousarray(a))
    return a.contiguous().cuda()


def host_bits(t):
    """Tensor -> numpy array for the oracle: fp32 as float32, bf16 as uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def f32(t):
    return t.detach().float().cpu().numpy()


def assert_bytes_equal(got, want, what):
    got = np.atleast_1d(np.asarray(got))
    want = np.atleast_1d(np.asarray(want))
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got != want)
    if bad[0].size:
        idx = tuple(b[:5] for b in bad)
        raise AssertionError("%s: %d mismatches, first at %s: got %s want %s" % (
            what, bad[0].size, [tuple(int(i) for i in p) for p in zip(*idx)], got[idx], want[idx]))


def assert_f32_bits_equal(got, want, what):
    g = np.asarray(got, np.float32).view(np.uint32)
    w = np.asarray(want, np.float32).view(np.uint32)
    assert_bytes_equal(g, w, what)


NORMWISE_TOL_F32 = 1e-5


def check_gemm_fp32(got, ref, what):
    """fp32 output: normwise relative error ||D - D_ref||_F / ||D_ref||_F <= 1e-5."""
    got = np.asarray(got, np.float64)
    num = np.linalg.norm(got - ref)
    den = np.linalg.norm(ref)
    err = num / den if den > 0 else num
    assert err <= NORMWISE_TOL_F32, "%s: normwise relative error %.3e > %.0e" % (what, err, NORMWISE_TOL_F32)
    return err


def bf16_ulp(bits):
    """Spacing of bf16 values at the magnitude of the given bf16 bit patterns."""
    b = np.asarray(bits, np.uint16).astype(np.uint32)
    exp = (b >> 7) & 0xFF
    # ulp = 2^(max(exp,1) - 127 - 7)
    e = np.maximum(exp.astype(np.int64), 1) - 127 - 7
    return np.ldexp(1.0, e)


def abs_dot(a, fa, b, fb, sa, sb, rows=None):
    """(|A| . |B|^T) * sa * sb from the oracle: the magnitude sum each output
    element accumulates (FP8 codes with the sign bit cleared)."""
    return o.gemm(np.asarray(a, np.uint8) & 0x7F, fa, np.asarray(b, np.uint8) & 0x7F, fb, sa, sb,
                  rows=rows)


def accumulation_allowance(absdot, K):
    """fp32 accumulation bound: the tensor core adds exact 32-term partial
    products into an fp32 accumulator, ceil(K/32) additions, plus the
    epilogue's fused multiply-add; each rounding is at most 2^-24 of the
    running magnitude, which is at most sum_k |a_k b_k| * sa * sb."""
    return (np.ceil(K / 32.0) + 2) * 2.0 ** -24 * np.asarray(absdot, np.float64)


# Largest share of a bf16 output's elements that may lie beyond the plain
# 1-ulp bound (inside the accumulation allowance): the allowance exists for
# the rare elements whose |D_ref| cancels far below sum_k |a_k b_k|; a
# regression that pushes many elements into it fails here.
BF16_BEYOND_ULP_MAX_SHARE = 1e-3
BF16_BEYOND_ULP_MIN_COUNT = 2

# (what, max ulp, share within 1 ulp, elements) of every bf16 check of the
# session; tests/conftest.py prints the summary at the end of the run.
BF16_CHECKS = []


def check_gemm_bf16(got_bits, ref, what, absdot=None, K=None):
    """bf16 output: every element within 1 bf16 ulp (at |bf16_rne(D_ref)|) of
    the fp64 reference, widened by the fp32 accumulation bound where
    cancellation makes |D_ref| small against sum_k |a_k b_k|.  At most
    BF16_BEYOND_ULP_MAX_SHARE of the elements (and never more than
    BF16_BEYOND_ULP_MIN_COUNT on small outputs) may need the widening.
    Returns (max ulp, share of elements within 1 ulp)."""
    got = o.bf16_bits_to_f32(got_bits).astype(np.float64)
    ulp = bf16_ulp(o.round_bf16(ref))
    tol = ulp if absdot is None else ulp + accumulation_allowance(absdot, K)
    diff = np.abs(got - ref)
    bad = diff > tol
    if bad.any():
        i = np.argmax(diff / tol)
        raise AssertionError("%s: %d elements beyond tolerance; worst %s got %r ref %r (%.2f ulp, "
                             "%.2f x tol)" % (what, int(bad.sum()), np.unravel_index(i, ref.shape),
                                              got.flat[i], ref.flat[i], (diff / ulp).flat[i],
                                              (diff / tol).flat[i]))
    beyond = int((diff > ulp).sum())
    max_ulp = float((diff / ulp).max()) if diff.size else 0.0
    within = 1.0 - beyond / diff.size if diff.size else 1.0
    BF16_CHECKS.append((what, max_ulp, within, int(diff.size)))
    limit = max(BF16_BEYOND_ULP_MIN_COUNT, int(BF16_BEYOND_ULP_MAX_SHARE * diff.size))
    assert beyond <= limit, "%s: %d of %d elements beyond 1 bf16 ulp (inside the accumulation allowance), " \
        "more than %d; max %.2f ulp" % (what, beyond, diff.size, limit, max_ulp)
    return max_ulp, within
