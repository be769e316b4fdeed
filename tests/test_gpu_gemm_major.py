"""GPU parity of fp8_gemm_major: GEMM operands stored MN-major ([k, m] /
[k, n] row-major, the tensors as their producers wrote them) read transposed
by the tensor core, against the oracle GEMM of the same logical operands.

The MN-major storage is the host transpose of the K-major operand, so the
oracle reference is the ordinary fp64 GEMM.  Checked: every layout pair, both
kernels (one CTA for M <= 128; CTA pairs with 256- and 512-row tiles), ragged
M, N and K (K free when both operands are MN-major), the mixed e5m2 x e4m3
wgrad/dgrad formats, bf16 and fp32 outputs; integer-valued operands whose
partial sums are exact in fp32 must give bit-identical output (a layout or
addressing error cannot hide there); and, on realistic operands, the MN-major
result equals the K-major one bit for bit.
"""
import functools

import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, dev, host_bits
from tests.test_gpu_gemm import TOP, _compare, _rows_for
from tests.test_gpu_gemm import _realistic_operands as _realistic_uncached

_realistic_operands = functools.lru_cache(maxsize=4)(_realistic_uncached)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _store(a, major):
    """K-major [rows, k] -> the stored array for that layout."""
    return np.ascontiguousarray(a.T) if major == "mn" else a


def _run(fp8, a, fa, am, sa, b, fb, bm, sb, out_dtype):
    M, K = a.shape
    N = b.shape[0]
    d = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    fp8.fp8_gemm_major(dev(_store(a, am)), fa, am, torch.tensor([sa], device="cuda"), dev(_store(b, bm)), fb, bm,
                       torch.tensor([sb], device="cuda"), d)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    return d


LAYOUTS = [("k", "mn"), ("mn", "k"), ("mn", "mn")]
# (M, N, K): one-CTA kernel, pair 256-row tiles, 512-row tiles (K >= 2048
# with enough tiles), ragged edges (a partial last k-block, M and N off the
# tile grid), more tiles than SM pairs.
SHAPES = [(128, 256, 128), (64, 512, 256), (384, 512, 512), (400, 528, 272), (1024, 512, 4096),
          (2048, 8192, 1024), (1040, 4880, 2064), (8192, 2048, 8192)]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_major_realistic(fp8, layout, shape, out_dtype):
    M, N, K = shape
    am, bm = layout
    a, b, sa, sb = _realistic_operands(M, N, K, "e4m3", "e4m3", seed=M + N + K)
    rows = _rows_for(M, N, K)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    d = _run(fp8, a, "e4m3", am, sa, b, "e4m3", bm, sb, out_dtype)
    _compare(d, ref, rows, out_dtype, "%s x %s %s" % (am, bm, shape), (a, "e4m3", b, "e4m3", sa, sb))
    # same accumulation as the K-major kernel path
    dk = torch.full_like(d, float("nan"))
    fp8.fp8_gemm(dev(a), "e4m3", torch.tensor([sa], device="cuda"), dev(b), "e4m3", torch.tensor([sb], device="cuda"),
                 dk)
    torch.cuda.synchronize()
    assert_bytes_equal(host_bits(d).view(np.uint8), host_bits(dk).view(np.uint8), "MN-major vs K-major")


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("shape", [(208, 528, 160), (1024, 1024, 512), (128, 256, 1040)])
def test_gemm_major_integer_exact(fp8, layout, shape):
    """e5m2 x e4m3 (the wgrad/dgrad formats) on small integers: exact in fp32."""
    M, N, K = shape
    am, bm = layout
    rng = np.random.default_rng(M + N + K)
    av = rng.integers(-3, 4, (M, K)).astype(np.float32)
    bv = rng.integers(-3, 4, (N, K)).astype(np.float32)
    a = o.encode(av, o.E5M2)
    b = o.encode(bv, o.E4M3)
    d = _run(fp8, a, "e5m2", am, np.float32(1.0), b, "e4m3", bm, np.float32(1.0), torch.float32)
    ref = av.astype(np.float64) @ bv.astype(np.float64).T
    got = d.cpu().numpy()
    assert np.array_equal(got, ref.astype(np.float32)), "%s x %s %s: %d mismatches" % (
        am, bm, shape, int((got != ref).sum()))


@pytest.mark.parametrize("K", [24, 200, 4100])
def test_gemm_major_k_free_when_both_mn(fp8, K):
    """Both operands MN-major: K needs no alignment (the tensor maps' inner
    dimensions are M and N); the partial last k-block reads zeros."""
    M, N = 256, 512
    a = inputs.fp8_codes((M, K), seed=K, fmt_max_code=TOP["e4m3"]).numpy()
    b = inputs.fp8_codes((N, K), seed=K + 1, fmt_max_code=TOP["e4m3"]).numpy()
    sa, sb = np.float32(2.0 ** -6), np.float32(2.0 ** -6)
    d = _run(fp8, a, "e4m3", "mn", sa, b, "e4m3", "mn", sb, torch.float32)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb)
    _compare(d, ref, None, torch.float32, "mn x mn K=%d" % K, None)
