"""GPU parity of the multi-tensor cast (fp8_cast_transpose_amax_multi) and of
the one-launch weight-cache refresh (fp8_linear_refresh_weights) against the
oracle.

"[PyTorch] Refactor FP8 workspaces in linear modules" refreshes the FP8 weight
workspaces of the linears together; "CPU Overhead of te.Linear FP8 Layers"
names the per-tensor launches as the cost.  Every job of one launch must give
the bytes of its own fp8_cast_transpose_amax call: y, yt, the amax max-ed into
its slot (which starts non-zero here) and its private scale_inv -- compared
with oracle.cast_transpose_amax bit for bit.  The job list mixes input dtypes,
formats, transposes, tile-aligned and ragged shapes, unaligned pointers (the
element path), an empty tensor, a single row, tensors spanning many tiles,
and jobs whose device noop flag is set (nothing of them may be written).
"""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, assert_f32_bits_equal, host_bits, u8

pytestmark = pytest.mark.gpu

FMT = {"e4m3": o.E4M3, "e5m2": o.E5M2}
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


class _Job:
    """Device buffers of one job and its oracle expectation."""

    def __init__(self, fp8, rows, cols, dtype, fmt, transpose, seed, scale, amax0=0.25, noop=None, offset=0):
        g = inputs.gen(seed)
        x = inputs.normal((rows * cols + offset,), g) * 3.0
        if rows * cols > 64:
            x[7 + offset] = 900.0                          # saturates e4m3 at scale >= 0.5
        x = x.to(torch.bfloat16) if dtype == "bf16" else x
        self.base = x.cuda()
        self.x = self.base[offset:].view(rows, cols)        # offset > 0: not 16-byte aligned
        self.host = (host_bits(x[offset:]) if dtype == "bf16" else x[offset:].numpy()).reshape(rows, cols)
        self.fmt, self.transpose, self.noop = fmt, transpose, noop
        self.scale = torch.tensor([scale], device="cuda")
        self.y = torch.full((rows, cols), SENTINEL, dtype=torch.uint8, device="cuda")
        self.yt = torch.full((cols, rows), SENTINEL, dtype=torch.uint8, device="cuda") if transpose else None
        self.amax = torch.tensor([amax0], device="cuda")
        self.si = torch.full((1,), -1.0, device="cuda")
        self.amax0 = amax0
        self.flag = None if noop is None else torch.tensor([noop], dtype=torch.int32, device="cuda")
        self.rec = fp8.cast_job(self.x, fmt, self.scale, self.y, self.yt, self.amax, self.si, self.flag)

    def check(self, what):
        if self.noop:
            assert (u8(self.y) == SENTINEL).all(), what + ": noop job wrote y"
            if self.yt is not None:
                assert (u8(self.yt) == SENTINEL).all(), what + ": noop job wrote yt"
            assert self.amax.item() == self.amax0 and self.si.item() == -1.0, what + ": noop job wrote amax/scale_inv"
            return
        y, yt, am, si = o.cast_transpose_amax(self.host, FMT[self.fmt], np.float32(self.scale.item()),
                                              np.float32(self.amax0), transpose=self.transpose)
        assert_bytes_equal(u8(self.y), y, what + ": y")
        if self.transpose:
            assert_bytes_equal(u8(self.yt), yt, what + ": yt")
        assert_f32_bits_equal(self.amax.cpu().numpy(), [am], what + ": amax")
        assert_f32_bits_equal(self.si.cpu().numpy(), [si], what + ": scale_inv")


def _mixed_jobs(fp8):
    specs = [
        # rows, cols, dtype, fmt, transpose, scale, noop, offset
        (1024, 2048, "f32", "e4m3", False, 1.0, None, 0),      # many flat tiles
        (512, 512, "bf16", "e5m2", True, 64.0, None, 0),       # transpose, vector tiles
        (300, 136, "f32", "e5m2", True, 0.5, 0, 0),            # ragged rows: edge tiles; flag 0 runs
        (200, 100, "bf16", "e4m3", False, 2.0, None, 0),       # flat, partial last tile
        (64, 64, "f32", "e4m3", True, 1.0, 1, 0),              # flag set: skipped
        (0, 128, "f32", "e4m3", False, 4.0, None, 0),          # empty: only scale_inv
        (1, 4100, "bf16", "e4m3", False, 0.75, None, 0),       # one row
        (96, 48, "f32", "e4m3", False, 1.5, None, 1),          # unaligned x: element path
        (128, 64, "bf16", "e5m2", True, 8.0, None, 1),         # unaligned with transpose
        (2048, 1024, "bf16", "e4m3", True, 448.0 / 900.0, None, 0),
        (4096, 256, "f32", "e5m2", False, 1.0, 1, 0),          # large and skipped
    ]
    return [_Job(fp8, r, c, dt, f, t, seed=40 + i, scale=s, noop=n, offset=off)
            for i, (r, c, dt, f, t, s, n, off) in enumerate(specs)]


def test_multi_cast_mixed_jobs(fp8):
    jobs = _mixed_jobs(fp8)
    fp8.fp8_cast_transpose_amax_multi([j.rec for j in jobs])
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    for i, j in enumerate(jobs):
        j.check("job %d" % i)


def test_multi_cast_equals_single_calls(fp8):
    """The same tensors cast one call each give the same bytes and amaxes."""
    a = _mixed_jobs(fp8)
    b = _mixed_jobs(fp8)
    fp8.fp8_cast_transpose_amax_multi([j.rec for j in a])
    for j in b:
        if j.flag is None:
            fp8.fp8_cast_transpose_amax(j.x, j.fmt, j.scale, j.y, j.yt, j.amax, j.si)
        else:
            fp8.fp8_cast_transpose_amax_noop(j.x, j.fmt, j.scale, j.y, j.yt, j.amax, j.si, j.flag)
    torch.cuda.synchronize()
    for i, (ja, jb) in enumerate(zip(a, b)):
        assert torch.equal(ja.y, jb.y), i
        if ja.yt is not None:
            assert torch.equal(ja.yt, jb.yt), i
        assert torch.equal(ja.amax.view(torch.int32), jb.amax.view(torch.int32)), i
        assert torch.equal(ja.si.view(torch.int32), jb.si.view(torch.int32)), i


@pytest.mark.parametrize("dtype,fmt,transpose", [("f32", "e4m3", False), ("bf16", "e5m2", True)])
def test_multi_cast_same_kind_jobs(fp8, dtype, fmt, transpose):
    """Up to eight tensors of one input dtype and format, all with or all
    without transpose, that suit the TMA path go through the TMA kernel in one
    launch (the MLP step's X, W1, W2; a TEBlock's five inputs): every job
    exact, a flagged job skipped, ragged edge tiles included."""
    specs = [(512, 2048, 1.0, None), (1024, 512, 64.0, 0), (256, 1024, 0.5, 1), (208, 136, 2.0, None),
             (2048, 256, 448.0 / 900.0, None), (16, 8, 4.0, None), (640, 64, 1.0, None), (128, 4096, 0.25, None)]
    jobs = [_Job(fp8, r, c, dtype, fmt, transpose, seed=300 + i, scale=sc, noop=n)
            for i, (r, c, sc, n) in enumerate(specs)]
    fp8.fp8_cast_transpose_amax_multi([j.rec for j in jobs])
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    for i, j in enumerate(jobs):
        j.check("job %d" % i)


def test_multi_cast_more_jobs_than_one_launch(fp8):
    """300 small tensors, more than the 256 of one launch (so two launches),
    mixed dtypes, formats and transposes: every cast exact."""
    jobs = []
    for i in range(300):
        rows, cols = 16 + (i % 7) * 16, 8 + (i % 5) * 24
        jobs.append(_Job(fp8, rows, cols, "bf16" if i % 3 else "f32", "e5m2" if i % 2 else "e4m3", i % 4 == 0,
                         seed=1000 + i, scale=1.0 + (i % 9), amax0=0.0))
    fp8.fp8_cast_transpose_amax_multi(fp8.cast_jobs([j.rec for j in jobs]))
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    for i, j in enumerate(jobs):
        j.check("job %d" % i)


def test_multi_cast_graph_replay(fp8):
    """Captured once, replayed: the flags decide on the GPU at replay time."""
    jobs = _mixed_jobs(fp8)
    flagged = [j for j in jobs if j.flag is not None]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fp8.fp8_cast_transpose_amax_multi([j.rec for j in jobs])
    for j in flagged:                  # every flagged job runs at replay
        j.flag.fill_(0)
        j.noop = 0
    g.replay()
    torch.cuda.synchronize()
    for i, j in enumerate(jobs):
        j.check("replayed job %d" % i)
    del g


# ---------------------------------------------------- weight-cache refresh --

def test_refresh_weights_one_launch(fp8):
    """Six TEBlock-shaped linears (scaled down 4x), half with a cached
    transpose, refreshed in one launch together with an extra cast (a layer
    input): caches, private scale_invs and amaxes exactly the oracle's; the
    forward that follows with is_first_microbatch=False reuses them and gives
    the bytes of a forward that refreshes its own cache."""
    ws, bs = inputs.teblock_weights(seed=3, scale=4)
    L = len(ws)
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"] * L, hist_len=16)
    meta.scale[1::3] = torch.tensor([0.5 + i for i in range(L)], device="cuda")
    lins = [fp8.Fp8Linear(w.cuda(), None if b is None else b.cuda(), 3 * i, 3 * i + 1, 3 * i + 2,
                          transpose=(i % 2 == 0)) for i, (w, b) in enumerate(zip(ws, bs))]
    twins = [fp8.Fp8Linear(w.cuda(), None if b is None else b.cuda(), 3 * i, 3 * i + 1, 3 * i + 2,
                           transpose=(i % 2 == 0)) for i, (w, b) in enumerate(zip(ws, bs))]
    M, K = 256, ws[0].shape[1]
    x = inputs.uniform((M, K), inputs.gen(8)).cuda()
    x8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    x_si = torch.zeros(1, device="cuda")
    extra = fp8.cast_job(x, "e4m3", meta.scale[0:1], x8, None, meta.amax_history[0, 0:1], x_si)
    group = fp8.LinearGroup(lins)
    fp8.fp8_linear_refresh_weights(group, meta, [extra])
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    assert all(lin.cache_valid for lin in lins)
    hist = meta.amax_history[0].cpu().numpy()
    for i, (lin, w) in enumerate(zip(lins, ws)):
        y, yt, am, si = o.cast_transpose_amax(w.numpy(), o.E4M3, np.float32(0.5 + i), transpose=lin.w8t is not None)
        assert_bytes_equal(u8(lin.w8), y, "linear %d w8" % i)
        if lin.w8t is not None:
            assert_bytes_equal(u8(lin.w8t), yt, "linear %d w8t" % i)
        assert_f32_bits_equal(lin.w_scale_inv.cpu().numpy(), [si], "linear %d scale_inv" % i)
        assert_f32_bits_equal(hist[3 * i + 1], am, "linear %d weight amax" % i)
    xy, _, xam, xsi = o.cast_transpose_amax(x.cpu().numpy(), o.E4M3, np.float32(1.0), transpose=False)
    assert_bytes_equal(u8(x8), xy, "extra cast")
    assert_f32_bits_equal(hist[0], xam, "extra amax")
    # forwards on the refreshed caches vs forwards that refresh their own
    for i in range(L):
        k = lins[i].in_features
        xi = inputs.uniform((M, k), inputs.gen(20 + i)).cuda()
        outs = []
        for lin, first in ((lins[i], False), (twins[i], True)):
            y = torch.empty(M, lin.out_features, dtype=torch.bfloat16, device="cuda")
            xb8 = torch.empty(M, k, dtype=torch.uint8, device="cuda")
            si = torch.zeros(1, device="cuda")
            fp8.fp8_linear_fwd(lin, meta, xi, y, first, xb8, None, si)
            outs.append(y)
        torch.cuda.synchronize()
        assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), "linear %d forward" % i
        assert torch.equal(lins[i].w8, twins[i].w8)
