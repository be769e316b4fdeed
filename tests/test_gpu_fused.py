"""GPU parity of the FP8-output GEMM epilogue and of the FP8 hand-over between
linears.

fp8_gemm_cast restates torch._scaled_mm with an FP8 out_dtype and its
output_amax ("Accelerating PyTorch Training Workloads with FP8 -- Part 2"):
the GEMM's bf16 result h, cast with a delayed scale, transposed, its amax
recorded.  The oracle takes h from fp8_gemm (the same accumulation: the same
kernel schedule and MMA order), after h itself is checked against the exact
fp64 GEMM on sampled rows, and casts it with oracle.cast_transpose_amax; the
codes, the transpose, the amax and the private scale_inv must match bit for
bit.

fp8_linear_fwd_ex / fp8_linear_bwd_ex pass H and dH of an MLP from GEMM to
GEMM in FP8.  By their definition the results equal those of the unfused
calls, which the oracle checks elsewhere (the linear and full-size workload
tests), so every output, FP8 tensor and meta of the fused step is compared
with the unfused step bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import (abs_dot, assert_bytes_equal, assert_f32_bits_equal, check_gemm_bf16, dev, host_bits,
                            u8)

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
    bias = inputs.normal((N,), inputs.gen(seed + 1), 0.02)
    return a, b, np.float32(sa), np.float32(sb), bias


def _rows(M, seed):
    return np.array(sorted({0, M // 2, M - 1} | set(np.random.default_rng(seed).integers(0, M, 8).tolist())),
                    np.int64)


CASES = [
    # (M, N, K, out_fmt, bias, transpose, amax_init)
    (128, 256, 128, "e4m3", "f32", True, 0.0),       # one-CTA kernel (M <= 128)
    (400, 528, 256, "e4m3", "f32", True, 0.0),       # CTA pairs, 256-row tiles, ragged M and N
    (400, 528, 256, "e5m2", "bf16", True, 0.0),
    (1024, 512, 4096, "e4m3", None, True, 0.0),      # long K, few tiles (256-row pair tiles)
    (1024, 512, 4096, "e5m2", "f32", False, 1e9),    # no transpose; a larger running amax is kept
    # 512-row pair tiles (released to the next tile half by half), ragged in M, N and K
    (1040, 4880, 4112, "e4m3", "f32", False, 0.0),
    (1008, 4880, 2064, "e5m2", "bf16", True, 0.0),
    (2048, 8192, 2048, "e4m3", "f32", True, 0.0),    # the MLP's fc1 shape class
    # without the transpose the codes leave through the staged TMA store
    (128, 256, 128, "e4m3", "f32", False, 0.0),
    (400, 528, 256, "e5m2", "bf16", False, 0.0),
    (2048, 8192, 2048, "e4m3", "f32", False, 0.0),
]


@pytest.mark.parametrize("M,N,K,out_fmt,bias_kind,transpose,amax_init", CASES)
def test_gemm_cast_matches_cast_of_bf16_output(fp8, M, N, K, out_fmt, bias_kind, transpose, amax_init):
    a, b, sa, sb, bias = _operands(M, N, K, seed=M + N + K)
    ad, bd = dev(a), dev(b)
    sad = torch.tensor([sa], device="cuda")
    sbd = torch.tensor([sb], device="cuda")
    biasd = None
    bias_np = None
    if bias_kind == "f32":
        biasd = bias.cuda()
        bias_np = bias.numpy()
    elif bias_kind == "bf16":
        biasd = bias.to(torch.bfloat16).cuda()
        bias_np = o.bf16_bits_to_f32(host_bits(bias.to(torch.bfloat16)))
    fmt = o.E4M3 if out_fmt == "e4m3" else o.E5M2
    # h = the bf16 GEMM output, pinned to the exact GEMM on sampled rows
    h = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    fp8.fp8_gemm(ad, "e4m3", sad, bd, "e4m3", sbd, h, bias=biasd)
    torch.cuda.synchronize()
    rows = _rows(M, seed=K)
    exact = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, bias_np, rows=rows)
    absdot = abs_dot(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    h_bits = host_bits(h)
    check_gemm_bf16(h_bits[rows], exact, "bf16 GEMM rows", absdot=absdot, K=K)
    # a delayed scale that saturates the largest ~10 % of |h| (scale from the
    # exact rows, so that saturation, rounding and subnormals all occur)
    s = np.float32(o.fp8_max(fmt)) / np.float32(0.9 * np.abs(exact).max())
    sd = torch.tensor([s], device="cuda")
    d8 = torch.full((M, N), 0xAA, dtype=torch.uint8, device="cuda")
    d8t = torch.full((N, M), 0xAA, dtype=torch.uint8, device="cuda") if transpose else None
    am = torch.tensor([amax_init], dtype=torch.float32, device="cuda")
    si = torch.zeros(1, dtype=torch.float32, device="cuda")
    fp8.fp8_gemm_cast(ad, "e4m3", sad, bd, "e4m3", sbd, out_fmt, sd, d8, d8t, am, si, bias=biasd)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    y, yt, oam, osi = o.cast_transpose_amax(h_bits, fmt, s, amax=np.float32(amax_init))
    assert_bytes_equal(u8(d8), y, "codes")
    if transpose:
        assert_bytes_equal(u8(d8t), yt, "transposed codes")
    assert_f32_bits_equal(am.cpu().numpy(), [oam], "amax")
    assert_f32_bits_equal(si.cpu().numpy(), [osi], "scale_inv")
    # saturation really occurred
    assert np.any((y & 0x7F) == (0x7E if fmt == o.E4M3 else 0x7B))


@pytest.mark.parametrize("M,N,K,transpose", [
    (100, 256, 32, False),     # one-CTA tile of 128 rows: rows 100-127 are padding
    (300, 528, 32, False),     # 256-row pair tiles: rows 300-511 of the last tile
    (304, 528, 32, True),      # the same through the transpose epilogue (M % 16 == 0)
    (1040, 512, 2048, False),  # 512-row pair tiles: rows 1040-1535 of the last tile
])
def test_gemm_cast_amax_covers_output_rows_only(fp8, M, N, K, transpose):
    """The amax is that of D's M rows.  The last tile's rows past M hold
    acc = 0 (their A rows read as zeros), so there D would be the bias alone;
    here the bias is -(K - 0.5) and every real row has acc = K, so the real
    outputs are all 0.5 while the padding rows would give |D| = K - 0.5."""
    one = 0x38                                    # e4m3 code of 1.0
    a = np.full((M, K), one, dtype=np.uint8)
    b = np.full((N, K), one, dtype=np.uint8)
    assert o.decode(a[:1, :1], o.E4M3)[0, 0] == 1.0
    bias = torch.full((N,), -(K - 0.5), dtype=torch.float32, device="cuda")
    s1 = torch.ones(1, device="cuda")
    d8 = torch.full((M, N), 0xAA, dtype=torch.uint8, device="cuda")
    d8t = torch.full((N, M), 0xAA, dtype=torch.uint8, device="cuda") if transpose else None
    am = torch.zeros(1, device="cuda")
    si = torch.zeros(1, device="cuda")
    fp8.fp8_gemm_cast(dev(a), "e4m3", s1, dev(b), "e4m3", s1, "e4m3", s1, d8, d8t, am, si, bias=bias)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    y, yt, oam, _ = o.cast_transpose_amax(np.full((M, N), 0.5, dtype=np.float32), o.E4M3, np.float32(1.0))
    assert oam == 0.5
    assert_bytes_equal(u8(d8), y, "codes")
    if transpose:
        assert_bytes_equal(u8(d8t), yt, "transposed codes")
    assert_f32_bits_equal(am.cpu().numpy(), [oam], "amax")


class _Mlp:
    """fc1 (hidden -> ffn) and fc2 (ffn -> hidden) with metas [X, W1, dH, H, W2, dY]
    and all device buffers of one training step."""

    def __init__(self, fp8, tokens, hidden, ffn, workspace=None, transposes=True):
        w1, b1, w2, b2 = inputs.mlp_pair(seed=0, tokens=tokens, hidden=hidden, ratio=ffn // hidden)
        self.fp8 = fp8
        self.meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2", "e4m3", "e4m3", "e5m2"], hist_len=16)
        self.fc1 = fp8.Fp8Linear(w1.cuda(), b1.cuda(), 0, 1, 2, workspace=workspace, transpose=transposes)
        self.fc2 = fp8.Fp8Linear(w2.cuda(), b2.cuda(), 3, 4, 5, workspace=workspace, transpose=transposes)
        self.transposes = transposes
        M, Hd, F = tokens, hidden, ffn
        u = lambda *s: torch.zeros(*s, dtype=torch.uint8, device="cuda")   # noqa: E731
        f = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")  # noqa: E731
        b16 = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
        self.x8, self.x8t, self.h8, self.h8t = u(M, Hd), u(Hd, M), u(M, F), u(F, M)
        self.dy8, self.dy8t, self.dh8, self.dh8t = u(M, Hd), u(Hd, M), u(M, F), u(F, M)
        self.si = f(4)
        self.h, self.y, self.dh, self.dx = b16(M, F), b16(M, Hd), b16(M, F), b16(M, Hd)
        self.dw1, self.dw2 = f(F, Hd), f(Hd, F)

    def step_unfused(self, x, dy):
        fp8, m = self.fp8, self.meta
        fp8.fp8_linear_fwd(self.fc1, m, x, self.h, True, self.x8, self.x8t, self.si[0:1])
        fp8.fp8_linear_fwd(self.fc2, m, self.h, self.y, True, self.h8, self.h8t, self.si[1:2])
        fp8.fp8_linear_bwd(self.fc2, m, dy, self.h8t, self.si[1:2], self.dw2, self.dy8, self.dy8t, self.si[2:3],
                           dx=self.dh)
        fp8.fp8_linear_bwd(self.fc1, m, self.dh, self.x8t, self.si[0:1], self.dw1, self.dh8, self.dh8t,
                           self.si[3:4], dx=self.dx)
        m.update()

    def step_fused(self, x, dy):
        fp8, m = self.fp8, self.meta
        # fc1 writes H in FP8 straight into fc2's input buffers (meta 3 = fc2's input)
        fp8.fp8_linear_fwd_ex(self.fc1, m, x, None, True, self.x8, self.x8t, self.si[0:1], out_meta=3,
                              out8=self.h8, out8t=self.h8t, out_scale_inv=self.si[1:2])
        fp8.fp8_linear_fwd_ex(self.fc2, m, None, self.y, True, self.h8, self.h8t, self.si[1:2], in_cast=True)
        # fc2's dgrad writes dH in FP8 straight into fc1's gradient buffers (meta 2 = fc1's grad)
        fp8.fp8_linear_bwd_ex(self.fc2, m, dy, self.h8t, self.si[1:2], self.dw2, self.dy8, self.dy8t,
                              self.si[2:3], out_meta=2, out8=self.dh8, out8t=self.dh8t,
                              out_scale_inv=self.si[3:4])
        fp8.fp8_linear_bwd_ex(self.fc1, m, None, self.x8t, self.si[0:1], self.dw1, self.dh8, self.dh8t,
                              self.si[3:4], dx=self.dx, in_cast=True)
        m.update()

    def step_no_transposes(self, x, dy):
        """The fused step with no transposed copy anywhere: the GEMMs read
        X8, H8, dY8, dH8 and the weights MN-major where the transpose was used."""
        fp8, m = self.fp8, self.meta
        fp8.fp8_linear_fwd_ex(self.fc1, m, x, None, True, self.x8, None, self.si[0:1], out_meta=3,
                              out8=self.h8, out8t=None, out_scale_inv=self.si[1:2])
        fp8.fp8_linear_fwd_ex(self.fc2, m, None, self.y, True, self.h8, None, self.si[1:2], in_cast=True)
        fp8.fp8_linear_bwd_ex(self.fc2, m, dy, None, self.si[1:2], self.dw2, self.dy8, None, self.si[2:3],
                              out_meta=2, out8=self.dh8, out8t=None, out_scale_inv=self.si[3:4], x8=self.h8)
        fp8.fp8_linear_bwd_ex(self.fc1, m, None, None, self.si[0:1], self.dw1, self.dh8, None, self.si[3:4],
                              dx=self.dx, in_cast=True, x8=self.x8)
        m.update()


    def step_one_cast_launch(self, x, dy):
        """The step without transposes whose X, W1 and W2 casts are one launch
        (fp8_linear_refresh_weights with X as an extra job); the forwards then
        reuse the refreshed caches and take X8 as already cast."""
        fp8, m = self.fp8, self.meta
        if not hasattr(self, "group"):
            self.group = fp8.LinearGroup([self.fc1, self.fc2])
        xjob = fp8.cast_job(x, "e4m3", m.scale[0:1], self.x8, None, m.amax_history[0, 0:1], self.si[0:1])
        fp8.fp8_linear_refresh_weights(self.group, m, [xjob])
        fp8.fp8_linear_fwd_ex(self.fc1, m, None, None, False, self.x8, None, self.si[0:1], in_cast=True,
                              out_meta=3, out8=self.h8, out8t=None, out_scale_inv=self.si[1:2])
        fp8.fp8_linear_fwd_ex(self.fc2, m, None, self.y, False, self.h8, None, self.si[1:2], in_cast=True)
        fp8.fp8_linear_bwd_ex(self.fc2, m, dy, None, self.si[1:2], self.dw2, self.dy8, None, self.si[2:3],
                              out_meta=2, out8=self.dh8, out8t=None, out_scale_inv=self.si[3:4], x8=self.h8)
        fp8.fp8_linear_bwd_ex(self.fc1, m, None, None, self.si[0:1], self.dw1, self.dh8, None, self.si[3:4],
                              dx=self.dx, in_cast=True, x8=self.x8)
        m.update()


def _compare(u, f, what, names=("x8", "x8t", "h8", "h8t", "dy8", "dy8t", "dh8", "dh8t")):
    for name in names:
        assert_bytes_equal(u8(getattr(f, name)), u8(getattr(u, name)), "%s: %s" % (what, name))
    for name in ("y", "dx"):
        assert_bytes_equal(host_bits(getattr(f, name)), host_bits(getattr(u, name)), "%s: %s" % (what, name))
    for name in ("si", "dw1", "dw2"):
        assert_f32_bits_equal(getattr(f, name).cpu().numpy(), getattr(u, name).cpu().numpy(), what + ": " + name)
    for name in ("amax_history", "scale", "scale_inv"):
        assert_f32_bits_equal(getattr(f.meta, name).cpu().numpy(), getattr(u.meta, name).cpu().numpy(),
                              what + ": meta " + name)


@pytest.mark.parametrize("tokens,hidden,ffn,use_ws", [(384, 256, 1024, False), (1024, 512, 2048, True),
                                                      (7168, 2048, 2048, True), (8192, 2048, 8192, False)])
def test_mlp_fp8_handover_equals_unfused(fp8, tokens, hidden, ffn, use_ws):
    """Three delayed-scaling steps of the MLP pair, fused and unfused side by
    side from the same inputs; with a workspace the stream-K schedule may run
    (the same in both).  At 7168 tokens every GEMM takes 112 tiles of 512 x
    256 and runs stream-K; the FP8-output ones also release their
    accumulator half by half."""
    ws_u = fp8.gemm_workspace() if use_ws else None
    ws_f = fp8.gemm_workspace() if use_ws else None
    un = _Mlp(fp8, tokens, hidden, ffn, ws_u)
    fu = _Mlp(fp8, tokens, hidden, ffn, ws_f)
    for step in range(3):
        x, dy = inputs.mlp_step_inputs(step, tokens=tokens, hidden=hidden)
        xd, dyd = x.cuda(), dy.cuda()
        un.step_unfused(xd, dyd)
        fu.step_fused(xd, dyd)
        torch.cuda.synchronize()
        assert fp8.fp8ds_device_status() == 0
        _compare(un, fu, "step %d" % step)


@pytest.mark.parametrize("tokens,hidden,ffn", [(384, 256, 1024), (8192, 2048, 8192)])
def test_mlp_without_transposes_equals_unfused(fp8, tokens, hidden, ffn):
    """The B200 layout of the step: no FP8 transpose is ever written (casts
    without yt, weight caches without w8t, FP8 epilogues without the
    transposed output); the wgrads read X8/H8 and dY8/dH8 and the dgrads the
    weights MN-major.  Every output, FP8 tensor and meta equals the unfused
    step that casts and reads transposes, over three steps."""
    un = _Mlp(fp8, tokens, hidden, ffn)
    nt = _Mlp(fp8, tokens, hidden, ffn, transposes=False)
    for step in range(3):
        x, dy = inputs.mlp_step_inputs(step, tokens=tokens, hidden=hidden)
        xd, dyd = x.cuda(), dy.cuda()
        un.step_unfused(xd, dyd)
        nt.step_no_transposes(xd, dyd)
        torch.cuda.synchronize()
        assert fp8.fp8ds_device_status() == 0
        _compare(un, nt, "step %d" % step, names=("x8", "h8", "dy8", "dh8"))
        assert_bytes_equal(u8(nt.fc1.w8), u8(un.fc1.w8), "step %d: w1 cache" % step)
        assert_bytes_equal(u8(nt.fc2.w8), u8(un.fc2.w8), "step %d: w2 cache" % step)


@pytest.mark.parametrize("tokens,hidden,ffn", [(384, 256, 1024), (8192, 2048, 8192)])
def test_mlp_one_cast_launch_equals_unfused(fp8, tokens, hidden, ffn):
    """The benchmarked step: X, W1 and W2 cast in one launch (the weight-cache
    refresh of both linears with X as an extra job), no transposes.  Same
    bytes, outputs and metas as the unfused step over three steps."""
    un = _Mlp(fp8, tokens, hidden, ffn)
    one = _Mlp(fp8, tokens, hidden, ffn, transposes=False)
    for step in range(3):
        x, dy = inputs.mlp_step_inputs(step, tokens=tokens, hidden=hidden)
        xd, dyd = x.cuda(), dy.cuda()
        un.step_unfused(xd, dyd)
        one.step_one_cast_launch(xd, dyd)
        torch.cuda.synchronize()
        assert fp8.fp8ds_device_status() == 0
        _compare(un, one, "step %d" % step, names=("x8", "h8", "dy8", "dh8"))
        assert_bytes_equal(u8(one.fc1.w8), u8(un.fc1.w8), "step %d: w1 cache" % step)
        assert_bytes_equal(u8(one.fc2.w8), u8(un.fc2.w8), "step %d: w2 cache" % step)
