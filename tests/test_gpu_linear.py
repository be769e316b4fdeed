"""GPU parity of fp8_linear_fwd / fp8_linear_bwd and the delayed-scaling loop
against the oracle composition (oracle.linear)."""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import (abs_dot, assert_bytes_equal, assert_f32_bits_equal, check_gemm_bf16,
                            check_gemm_fp32, host_bits, u8)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _meta_state(meta):
    return (meta.amax_history.cpu().numpy(), meta.scale.cpu().numpy(), meta.scale_inv.cpu().numpy())


def _check_meta(meta, ometa, what):
    h, s, si = _meta_state(meta)
    assert_f32_bits_equal(h, ometa.hist, what + " history")
    assert_f32_bits_equal(s, ometa.scale, what + " scale")
    assert_f32_bits_equal(si, ometa.scale_inv, what + " scale_inv")


def test_single_linear_two_steps(fp8):
    """X fp32 [128,256] ~ U[0,1), W fp32 [512,256] ~ N(0,0.02), no bias, e4m3,
    scale 1, history 16 of zeros.  Step 1: cast with scale 1, record amax,
    update.  Step 2: cast with the new scale, Y = X.W^T in fp32."""
    x, w = inputs.single_linear(seed=0)
    M, K = x.shape
    N = w.shape[0]
    meta = fp8.Fp8Meta(["e4m3", "e4m3"], hist_len=16)
    ometa = o.OracleMeta([o.E4M3, o.E4M3], 16)
    lin = fp8.Fp8Linear(w.cuda(), None, 0, 1, 1)
    olin = o.OracleLinear(w.numpy(), None, 0, 1, 1)
    xd = x.cuda()
    for step in range(2):
        y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        x8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        x8t = torch.empty(K, M, dtype=torch.uint8, device="cuda")
        xsi = torch.empty(1, dtype=torch.float32, device="cuda")
        fp8.fp8_linear_fwd(lin, meta, xd, y, None, x8, x8t, xsi)
        ry, (rx8, rx8t, rxsi) = olin.fwd(x.numpy(), ometa, None)
        torch.cuda.synchronize()
        assert_bytes_equal(u8(x8), rx8, "x8 step %d" % step)
        assert_bytes_equal(u8(x8t), rx8t, "x8t step %d" % step)
        assert_bytes_equal(u8(lin.w8), olin.w8, "w8 step %d" % step)
        assert_bytes_equal(u8(lin.w8t), olin.w8t, "w8t step %d" % step)
        assert_f32_bits_equal(xsi.cpu().numpy(), [rxsi], "x scale_inv")
        assert_f32_bits_equal(lin.w_scale_inv.cpu().numpy(), [olin.w_scale_inv], "w scale_inv")
        _check_meta(meta, ometa, "after fwd %d" % step)
        check_gemm_fp32(y.cpu().numpy(), ry, "Y step %d" % step)
        meta.update()
        ometa.update()
        torch.cuda.synchronize()
        _check_meta(meta, ometa, "after update %d" % step)
    # the second step really used the delayed scale 448 / amax(X)
    assert ometa.scale[0] == np.float32(448.0) / np.float32(x.numpy().max())


@pytest.mark.parametrize("first_flags", [[True, False, False, False], [None, None, None, None]])
def test_weight_cache_private_scale_inv(fp8, first_flags):
    """Four microbatches with an update after each.  With is_first_microbatch
    True then False the cached weight (cast at microbatch 0 with scale 1) is
    reused with its frozen private scale_inv while the meta's weight scale
    moves on; with None the weight is recast every time."""
    M, K, N = 256, 512, 384
    g = inputs.gen(4)
    w = inputs.normal((N, K), g, 0.02)
    bias = inputs.normal((N,), inputs.gen(1), 0.02)
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"], hist_len=16)
    ometa = o.OracleMeta([o.E4M3, o.E4M3, o.E5M2], 16)
    lin = fp8.Fp8Linear(w.cuda(), bias.cuda(), 0, 1, 2)
    olin = o.OracleLinear(w.numpy(), bias.numpy(), 0, 1, 2)
    for mb, flag in enumerate(first_flags):
        x = inputs.uniform((M, K), g)
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        x8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        xsi = torch.empty(1, device="cuda")
        fp8.fp8_linear_fwd(lin, meta, x.cuda(), y, flag, x8, None, xsi)
        ry, (rx8, _, rxsi) = olin.fwd(x.numpy(), ometa, flag)
        torch.cuda.synchronize()
        assert lin.cache_valid
        assert_f32_bits_equal(lin.w_scale_inv.cpu().numpy(), [olin.w_scale_inv], "w scale_inv mb %d" % mb)
        absdot = abs_dot(rx8, o.E4M3, olin.w8, o.E4M3, rxsi, olin.w_scale_inv)
        check_gemm_bf16(host_bits(y.cpu()), ry, "Y mb %d" % mb, absdot=absdot, K=K)
        meta.update()
        ometa.update()
        _check_meta(meta, ometa, "mb %d" % mb)
    if first_flags[0] is True:
        # frozen at the scale 1.0 of microbatch 0, while the meta moved on
        assert lin.w_scale_inv.item() == 1.0
        assert meta.scale_inv[1].item() != 1.0


def test_linear_backward_small(fp8):
    """fwd + bwd of one linear (HYBRID: e4m3 forward, e5m2 gradient) at a size
    the oracle computes in full: dgrad bf16, wgrad fp32."""
    M, K, N = 384, 256, 528
    g = inputs.gen(8)
    w = inputs.normal((N, K), g, 0.02)
    x = inputs.uniform((M, K), g)
    dy = (inputs.normal((M, N), g, 1e-3)).to(torch.bfloat16)
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"], hist_len=16)
    ometa = o.OracleMeta([o.E4M3, o.E4M3, o.E5M2], 16)
    lin = fp8.Fp8Linear(w.cuda(), None, 0, 1, 2)
    olin = o.OracleLinear(w.numpy(), None, 0, 1, 2)
    for step in range(3):
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        x8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        x8t = torch.empty(K, M, dtype=torch.uint8, device="cuda")
        xsi = torch.empty(1, device="cuda")
        fp8.fp8_linear_fwd(lin, meta, x.cuda(), y, True, x8, x8t, xsi)
        _, saved = olin.fwd(x.numpy(), ometa, True)
        dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
        dy8 = torch.empty(M, N, dtype=torch.uint8, device="cuda")
        dy8t = torch.empty(N, M, dtype=torch.uint8, device="cuda")
        dysi = torch.empty(1, device="cuda")
        fp8.fp8_linear_bwd(lin, meta, dy.cuda(), x8t, xsi, dw, dy8, dy8t, dysi, dx=dx)
        rdx, rdw, (rdy8, rdy8t, rdysi) = olin.bwd(host_bits(dy), ometa, saved)
        torch.cuda.synchronize()
        assert_bytes_equal(u8(dy8), rdy8, "dy8")
        assert_bytes_equal(u8(dy8t), rdy8t, "dy8t")
        assert_f32_bits_equal(dysi.cpu().numpy(), [rdysi], "dy scale_inv")
        absdot = abs_dot(rdy8, o.E5M2, olin.w8t, o.E4M3, rdysi, olin.w_scale_inv)
        check_gemm_bf16(host_bits(dx.cpu()), rdx, "dgrad step %d" % step, absdot=absdot, K=N)
        check_gemm_fp32(dw.cpu().numpy(), rdw, "wgrad step %d" % step)
        meta.update()
        ometa.update()
        _check_meta(meta, ometa, "step %d" % step)
