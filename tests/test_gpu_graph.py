"""CUDA-graph replay of the FP8 linear path with a device-side weight-cache
flag ("[PyTorch] Refactor FP8 workspaces in linear modules": a graph
captured around the forward must not bake in whether the cached FP8 weight is
refreshed; "CPU Overhead of te.Linear FP8 Layers": capturing the training
step in a CUDA graph removes the CPU overhead).

* fp8_cast_transpose_amax_noop: with the flag set nothing is written; with
  it clear the result is the oracle's cast.
* A linear forward + update captured once and replayed over four
  microbatches, the flag 0 on the first and 1 on the others, equals the eager
  calls with is_first_microbatch True, False, False, False, bit for bit
  (those are checked against the oracle in the linear tests).
* The fused MLP training step (FP8 hand-over, weights recast every step)
  replayed from a graph equals the eager step, bit for bit, over three steps.
"""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, assert_f32_bits_equal, host_bits, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


@pytest.mark.parametrize("rows,cols", [(256, 192), (100, 36)])     # TMA path, element path
def test_cast_noop_flag(fp8, rows, cols):
    x = inputs.normal((rows, cols), inputs.gen(21), 3.0).to(torch.bfloat16)
    xd = x.cuda()
    s = torch.tensor([7.5], device="cuda")
    y = torch.full((rows, cols), 0x5A, dtype=torch.uint8, device="cuda")
    yt = torch.full((cols, rows), 0x5A, dtype=torch.uint8, device="cuda")
    am = torch.tensor([0.125], device="cuda")
    si = torch.tensor([-1.0], device="cuda")
    flag = torch.ones(1, dtype=torch.int32, device="cuda")
    fp8.fp8_cast_transpose_amax_noop(xd, "e4m3", s, y, yt, am, si, flag)
    torch.cuda.synchronize()
    assert bool((y == 0x5A).all()) and bool((yt == 0x5A).all())
    assert am.item() == 0.125 and si.item() == -1.0
    flag.zero_()
    fp8.fp8_cast_transpose_amax_noop(xd, "e4m3", s, y, yt, am, si, flag)
    ry, ryt, ram, rsi = o.cast_transpose_amax(host_bits(x), o.E4M3, np.float32(7.5), amax=np.float32(0.125))
    torch.cuda.synchronize()
    assert_bytes_equal(u8(y), ry, "y")
    assert_bytes_equal(u8(yt), ryt, "yt")
    assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")
    assert_f32_bits_equal(si.cpu().numpy(), [rsi], "scale_inv")


def _linear_pair(fp8, N, K, flag):
    w = inputs.normal((N, K), inputs.gen(40), 0.02)
    b = inputs.normal((N,), inputs.gen(41), 0.02)
    out = []
    for noop in (None, flag):
        meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"], hist_len=16)
        lin = fp8.Fp8Linear(w.cuda(), b.cuda(), 0, 1, 2, w_noop_flag=noop)
        out.append((meta, lin))
    return out


def test_graph_linear_forward_microbatches(fp8):
    M, K, N = 512, 256, 384
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    (meta_e, lin_e), (meta_g, lin_g) = _linear_pair(fp8, N, K, flag)
    xs = [inputs.uniform((M, K), inputs.gen(50 + mb)).cuda() for mb in range(4)]
    e8, e8t, esi = (torch.empty(M, K, dtype=torch.uint8, device="cuda"),
                    torch.empty(K, M, dtype=torch.uint8, device="cuda"), torch.empty(1, device="cuda"))
    g8, g8t, gsi = torch.empty_like(e8), torch.empty_like(e8t), torch.empty_like(esi)
    ye = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    yg = torch.empty_like(ye)
    x_static = torch.empty(M, K, device="cuda")

    # warm the library's per-kernel launch set-up outside the capture on a
    # throw-away copy of the state
    meta_w, lin_w = _linear_pair(fp8, N, K, flag)[1]
    fp8.fp8_linear_fwd(lin_w, meta_w, xs[0], yg, None, g8, g8t, gsi)
    meta_w.update()
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fp8.fp8_linear_fwd(lin_g, meta_g, x_static, yg, None, g8, g8t, gsi)
        meta_g.update()
    for mb in range(4):
        fp8.fp8_linear_fwd(lin_e, meta_e, xs[mb], ye, mb == 0, e8, e8t, esi)
        meta_e.update()
        x_static.copy_(xs[mb])
        flag.fill_(0 if mb == 0 else 1)
        graph.replay()
        torch.cuda.synchronize()
        what = "microbatch %d" % mb
        assert_bytes_equal(host_bits(yg), host_bits(ye), what + ": y")
        assert_bytes_equal(u8(g8), u8(e8), what + ": x8")
        assert_bytes_equal(u8(g8t), u8(e8t), what + ": x8t")
        assert_bytes_equal(u8(lin_g.w8), u8(lin_e.w8), what + ": w8")
        assert_bytes_equal(u8(lin_g.w8t), u8(lin_e.w8t), what + ": w8t")
        assert_f32_bits_equal(lin_g.w_scale_inv.cpu().numpy(), lin_e.w_scale_inv.cpu().numpy(), what + ": w si")
        for name in ("amax_history", "scale", "scale_inv"):
            assert_f32_bits_equal(getattr(meta_g, name).cpu().numpy(), getattr(meta_e, name).cpu().numpy(),
                                  what + ": " + name)
    # the weight was cast once, with the initial scale, and then reused
    assert lin_g.w_scale_inv.item() == 1.0 and meta_g.scale[1].item() != 1.0
    assert fp8.fp8ds_device_status() == 0


def test_graph_fused_mlp_step(fp8):
    from tests.test_gpu_fused import _Mlp
    tokens, hidden, ffn = 1024, 512, 2048
    eager = _Mlp(fp8, tokens, hidden, ffn)
    graphed = _Mlp(fp8, tokens, hidden, ffn)
    steps = [inputs.mlp_step_inputs(s, tokens=tokens, hidden=hidden) for s in range(3)]
    x_static = torch.empty(tokens, hidden, device="cuda")
    dy_static = torch.empty(tokens, hidden, dtype=torch.bfloat16, device="cuda")
    warm = _Mlp(fp8, tokens, hidden, ffn)
    warm.step_fused(steps[0][0].cuda(), steps[0][1].cuda())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        graphed.step_fused(x_static, dy_static)
    for s, (x, dy) in enumerate(steps):
        eager.step_fused(x.cuda(), dy.cuda())
        x_static.copy_(x)
        dy_static.copy_(dy)
        graph.replay()
        torch.cuda.synchronize()
        what = "step %d" % s
        for name in ("x8", "x8t", "h8", "h8t", "dy8", "dy8t", "dh8", "dh8t"):
            assert_bytes_equal(u8(getattr(graphed, name)), u8(getattr(eager, name)), what + ": " + name)
        for name in ("y", "dx"):
            assert_bytes_equal(host_bits(getattr(graphed, name)), host_bits(getattr(eager, name)), what + ": " + name)
        for name in ("si", "dw1", "dw2"):
            assert_f32_bits_equal(getattr(graphed, name).cpu().numpy(), getattr(eager, name).cpu().numpy(),
                                  what + ": " + name)
        for name in ("amax_history", "scale", "scale_inv"):
            assert_f32_bits_equal(getattr(graphed.meta, name).cpu().numpy(), getattr(eager.meta, name).cpu().numpy(),
                                  what + ": meta " + name)
    assert fp8.fp8ds_device_status() == 0
