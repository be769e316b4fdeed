"""GPU parity of the tcgen05 FP8 GEMM against the oracle.

fp32 output: normwise relative error <= 1e-5 against the fp64 oracle;
bf16 output: every element within 1 bf16 ulp of the fp64 oracle, widened by
the fp32 accumulation bound (ceil(K/32)+2) * 2^-24 * sum_k |a_k b_k| * sa * sb
for elements where cancellation makes the result small.  Exactness
check: integer-valued operands whose every partial sum is exact in fp32 must
give bit-identical fp32 output (catches layout and transposition errors).
Shapes cover one tile, ragged M/N/K edges, the minimum sizes, more tiles than
SMs (persistent loop, both accumulators, barrier phase wrap) and the full
8192x2048x8192 / 8192x8192x2048 shapes on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import abs_dot, check_gemm_bf16, check_gemm_fp32, dev, f32, host_bits

pytestmark = pytest.mark.gpu

FMT = {"e4m3": o.E4M3, "e5m2": o.E5M2}
TOP = {"e4m3": 0x7E, "e5m2": 0x7B}


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _realistic_operands(M, N, K, fa, fb, seed):
    """A = cast of U[0,1) activations, B = cast of N(0,0.02) weights, each with
    its delayed scale fp8_max/amax (the forward's operands)."""
    g = inputs.gen(seed)
    x = inputs.uniform((M, K), g)
    w = inputs.normal((N, K), g, 0.02)
    fmax = {"e4m3": 448.0, "e5m2": 57344.0}
    sx = np.float32(fmax[fa]) / np.float32(np.abs(x.numpy()).max())
    sw = np.float32(fmax[fb]) / np.float32(np.abs(w.numpy()).max())
    a, _, _, sa_inv = o.cast_transpose_amax(x.numpy(), FMT[fa], sx, transpose=False)
    b, _, _, sb_inv = o.cast_transpose_amax(w.numpy(), FMT[fb], sw, transpose=False)
    return a, b, np.float32(sa_inv), np.float32(sb_inv)


def _random_codes(M, N, K, fa, fb, seed):
    a = inputs.fp8_codes((M, K), seed, TOP[fa]).numpy()
    b = inputs.fp8_codes((N, K), seed + 1, TOP[fb]).numpy()
    return a, b, np.float32(0.375), np.float32(1.25)


def _run(fp8, a, fa, sa, b, fb, sb, out_dtype, bias=None):
    M, K = a.shape
    N = b.shape[0]
    d = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    fp8.fp8_gemm(dev(a), fa, torch.tensor([sa], device="cuda"), dev(b), fb,
                 torch.tensor([sb], device="cuda"), d, bias=None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    return d


def _rows_for(M, N, K):
    if M * N * K <= (1 << 29):
        return None
    r = set(range(0, min(M, 3))) | {M - 1, M - 2} | {min(M - 1, 127), min(M - 1, 128)}
    rng = np.random.default_rng(M + N + K)
    r |= set(rng.integers(0, M, 56).tolist())
    return np.array(sorted(r), np.int64)


def _compare(d, ref, rows, out_dtype, what, ops):
    """ops = (a, fa, b, fb, sa, sb): the operands, for the accumulation bound."""
    got = d.cpu()
    if rows is not None:
        got = got[torch.from_numpy(rows)]
    if out_dtype == torch.float32:
        return check_gemm_fp32(got.numpy(), ref, what)
    a, fa, b, fb, sa, sb = ops
    absdot = abs_dot(a, FMT[fa], b, FMT[fb], sa, sb, rows=rows)
    return check_gemm_bf16(host_bits(got), ref, what, absdot=absdot, K=a.shape[1])


# M <= 128 runs the 1-SM kernel, larger M the CTA-pair kernel: pair tile
# 256 x 256, or 512 x 256 when M > 256, K >= 2048 and the 512-row tiles fill
# the last wave of pairs as well (at least ~75 tiles of 256 rows).  Covered:
# ragged M inside a pair and inside the 512-row tile (1040 = 2 x 512 + 16,
# 1000), a second CTA with one row, B rows of the second CTA entirely out of
# range (N <= 128), a partial last k-block, more tiles than SM pairs, long K
# with few tiles (which keeps the 256-row tile).
SHAPES = [(128, 256, 128), (128, 512, 256), (300, 520, 272), (1, 8, 16), (129, 264, 144),
          (256, 256, 1024), (4096, 8, 256), (1000, 136, 528), (4096, 2048, 256),
          (2048, 8192, 1024), (600, 264, 4096), (1024, 512, 4112), (257, 136, 4096),
          (1040, 4880, 4112), (1000, 4880, 2064)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_e4m3_realistic(fp8, shape, out_dtype):
    M, N, K = shape
    a, b, sa, sb = _realistic_operands(M, N, K, "e4m3", "e4m3", seed=sum(shape))
    rows = _rows_for(M, N, K)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    d = _run(fp8, a, "e4m3", sa, b, "e4m3", sb, out_dtype)
    _compare(d, ref, rows, out_dtype, "e4m3 %s %s" % (shape, out_dtype),
             (a, "e4m3", b, "e4m3", sa, sb))


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e5m2", "e4m3"), ("e4m3", "e5m2"),
                                   ("e5m2", "e5m2")])
@pytest.mark.parametrize("shape", [(200, 264, 160), (384, 512, 512), (640, 264, 4096)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_format_pairs_random_codes(fp8, fa, fb, shape, out_dtype):
    M, N, K = shape
    a, b, sa, sb = _random_codes(M, N, K, fa, fb, seed=M + K)
    ref = o.gemm(a, FMT[fa], b, FMT[fb], sa, sb)
    d = _run(fp8, a, fa, sa, b, fb, sb, out_dtype)
    _compare(d, ref, None, out_dtype, "%s x %s %s" % (fa, fb, shape), (a, fa, b, fb, sa, sb))


@pytest.mark.parametrize("bias_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_bias(fp8, bias_dtype, out_dtype):
    M, N, K = 260, 520, 384
    a, b, sa, sb = _realistic_operands(M, N, K, "e4m3", "e4m3", seed=77)
    bias = (inputs.normal((N,), inputs.gen(1), 0.02)).to(bias_dtype)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, bias=bias.float().numpy())
    d = _run(fp8, a, "e4m3", sa, b, "e4m3", sb, out_dtype, bias=bias)
    _compare(d, ref, None, out_dtype, "bias %s -> %s" % (bias_dtype, out_dtype),
             (a, "e4m3", b, "e4m3", sa, sb))


def _integer_codes(shape, fmt, seed):
    """FP8 codes of the integers -k..k exactly representable in the format."""
    lim = 16 if fmt == "e4m3" else 8
    g = inputs.gen(seed)
    vals = torch.randint(-lim, lim + 1, shape, generator=g).float().numpy()
    return o.encode(vals, FMT[fmt]), vals


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e5m2", "e4m3")])
@pytest.mark.parametrize("shape", [(128, 256, 128), (300, 520, 1040), (1024, 1024, 512),
                                   (1100, 520, 4096)])
def test_gemm_integer_exact(fp8, fa, fb, shape):
    M, N, K = shape
    a, av = _integer_codes((M, K), fa, 5)
    b, bv = _integer_codes((N, K), fb, 6)
    # every partial sum is an integer below 2^24: exact in fp32 in any order
    assert 16 * 16 * K < (1 << 24)
    d = _run(fp8, a, fa, np.float32(0.5), b, fb, np.float32(4.0), torch.float32)
    ref = (av.astype(np.float64) @ bv.astype(np.float64).T) * 2.0
    ora = o.gemm(a, FMT[fa], b, FMT[fb], 0.5, 4.0)
    assert np.array_equal(ora, ref)
    got = f32(d).astype(np.float64)
    bad = np.nonzero(got != ora)
    assert bad[0].size == 0, "first mismatches at %s" % (list(zip(*[x[:5] for x in bad])),)


@pytest.mark.parametrize("shape", [(8192, 2048, 8192), (8192, 8192, 2048)])
def test_gemm_full_size_sampled(fp8, shape):
    M, N, K = shape
    a, b, sa, sb = _realistic_operands(M, N, K, "e4m3", "e4m3", seed=1)
    rows = _rows_for(M, N, K)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    d = _run(fp8, a, "e4m3", sa, b, "e4m3", sb, torch.bfloat16)
    _compare(d, ref, rows, torch.bfloat16, "full %s" % (shape,), (a, "e4m3", b, "e4m3", sa, sb))


def test_gemm_repeatable(fp8):
    """Same inputs, same bits, run after run."""
    a, b, sa, sb = _realistic_operands(1024, 2048, 1024, "e4m3", "e4m3", seed=9)
    d1 = _run(fp8, a, "e4m3", sa, b, "e4m3", sb, torch.float32)
    d2 = _run(fp8, a, "e4m3", sa, b, "e4m3", sb, torch.float32)
    assert torch.equal(d1.view(torch.int32), d2.view(torch.int32))


def test_gemm_plan_reports_the_schedule(fp8):
    """fp8_gemm_plan on this device: one-CTA tiles up to M = 128, the 512-row
    pair tile for the MLP's K >= 2048 shapes, tile counts, and stream-K only
    where whole tiles leave a ragged last wave worth balancing."""
    small = fp8.fp8_gemm_plan(128, 256, 128)
    assert not small["pair"] and small["m_sub"] == 0 and small["tiles"] == 1 and not small["stream_k"]
    assert small["resident"] == torch.cuda.get_device_properties(0).multi_processor_count
    fwd = fp8.fp8_gemm_plan(8192, 8192, 2048)
    assert fwd["pair"] and fwd["m_sub"] == 2 and fwd["tiles"] == 16 * 32
    pairs = fwd["resident"]
    assert 0 < pairs <= torch.cuda.get_device_properties(0).multi_processor_count // 2
    # 512 tiles: whole waves but the last, which is nearly full -> no stream-K
    assert fwd["stream_k"] == (3 * (512 % pairs) >= pairs and 8 * (512 % pairs) <= 7 * pairs)
    k8 = fp8.fp8_gemm_plan(8192, 2048, 8192)
    assert k8["pair"] and k8["m_sub"] == 2 and k8["tiles"] == 16 * 8
    short = fp8.fp8_gemm_plan(4096, 2048, 256)   # 128 tiles of 256 rows, but only 2 k-blocks
    assert short["pair"] and short["m_sub"] == 1 and short["tiles"] == 16 * 8 and not short["stream_k"]
    if pairs == 74:                               # a B200
        assert not fwd["stream_k"] and k8["stream_k"]
    with pytest.raises(fp8.Fp8dsError):
        fp8.fp8_gemm_plan(0, 256, 128)


# ------------------------------------------------------------------ stream-K --
# With a workspace, shapes whose pair tiles leave a ragged last wave run the
# stream-K schedule: the whole waves of tiles as before, then every pair takes
# an equal share of the remaining tiles' (tile, k-block) units; a tile split
# between two to four consecutive pairs is combined through the workspace in
# a fixed order.  On the 74 pairs of a B200:
#   (4096, 2048, 1024)  128 tiles of 256x256: 74 whole, 54 shared (up to
#                       three pairs per tile)
#   (4000, 2000, 1024)  the same with ragged M and N edges
#   (7168, 2048, 2048)  112 tiles of 512x256: 74 whole, 38 shared
#   (2048, 2048, 4096)  64 tiles of 256x256, all shared by the 74 pairs
#   (8192, 2048, 8192), (2048, 8192, 8192)  the MLP's 128 tiles of 512x256
SK_SHAPES = [(4096, 2048, 1024), (4000, 2000, 1024), (7168, 2048, 2048), (2048, 2048, 4096)]

@pytest.fixture(scope="module")
def ws(fp8):
    return fp8.gemm_workspace()


def _flags_clear(ws):
    return int(ws[:4096].view(torch.int32).abs().sum().item()) == 0


def _require_stream_k(fp8, M, N, K):
    """The shape must take the stream-K schedule; on a device with another
    number of resident CTA pairs than a B200's 74 it may not (skip then)."""
    plan = fp8.fp8_gemm_plan(M, N, K)
    if not plan["stream_k"]:
        assert plan["resident"] != 74, plan
        pytest.skip("%d tiles on %d CTA pairs: no split tiles" % (plan["tiles"], plan["resident"]))


@pytest.mark.parametrize("shape", SK_SHAPES)
@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e5m2", "e4m3")])
def test_gemm_stream_k_integer_exact(fp8, ws, shape, fa, fb):
    """Integer operands: every partial sum, and every sum of partials, is
    exact in fp32, so the split tiles must reproduce the exact product."""
    M, N, K = shape
    _require_stream_k(fp8, M, N, K)
    a, av = _integer_codes((M, K), fa, 15)
    b, bv = _integer_codes((N, K), fb, 16)
    d = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    fp8.fp8_gemm_ex(dev(a), fa, torch.tensor([0.5], device="cuda"), dev(b), fb,
                    torch.tensor([4.0], device="cuda"), d, workspace=ws)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    ref = (torch.from_numpy(av).double() @ torch.from_numpy(bv).double().T) * 2.0
    got = d.cpu().double()
    bad = torch.nonzero(got != ref)
    assert bad.shape[0] == 0, "mismatches at %s" % bad[:5].tolist()
    assert _flags_clear(ws)


@pytest.mark.parametrize("shape", [(8192, 2048, 8192), (2048, 8192, 8192), (4000, 2000, 1024)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_stream_k_realistic(fp8, ws, shape, out_dtype):
    M, N, K = shape
    _require_stream_k(fp8, M, N, K)
    a, b, sa, sb = _realistic_operands(M, N, K, "e4m3", "e4m3", seed=21)
    rows = _rows_for(M, N, K)
    ref = o.gemm(a, o.E4M3, b, o.E4M3, sa, sb, rows=rows)
    d = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    fp8.fp8_gemm_ex(dev(a), "e4m3", torch.tensor([sa], device="cuda"), dev(b), "e4m3",
                    torch.tensor([sb], device="cuda"), d, workspace=ws)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    _compare(d, ref, rows, out_dtype, "stream-K %s" % (shape,), (a, "e4m3", b, "e4m3", sa, sb))
    assert _flags_clear(ws)


def test_gemm_stream_k_repeatable(fp8, ws):
    """The split tiles are combined in a fixed order: same bits every run."""
    _require_stream_k(fp8, 4096, 2048, 1024)
    a, b, sa, sb = _realistic_operands(4096, 2048, 1024, "e4m3", "e4m3", seed=22)
    outs = []
    for _ in range(3):
        d = torch.empty(4096, 2048, dtype=torch.float32, device="cuda")
        fp8.fp8_gemm_ex(dev(a), "e4m3", torch.tensor([sa], device="cuda"), dev(b), "e4m3",
                        torch.tensor([sb], device="cuda"), d, workspace=ws)
        outs.append(d)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))
    assert torch.equal(outs[0].view(torch.int32), outs[2].view(torch.int32))


# ------------------------------------------------------------ error path --

def test_stream_k_partial_wait_gives_up_and_reports(fp8, ws):
    """The bounded wait for another pair's partial sum, made to run out: with
    the test setting the pairs that compute the later k-blocks of every split
    tile withhold their publication, so the owners of those tiles wait 5 ms,
    give up, record a timeout at the partial-sum site in the device error word
    and exit (no fault, no hang).  The context stays usable: the workspace's
    publication words are clear and the next normal call is exact."""
    M, N, K = 4096, 2048, 1024                      # 128 tiles of 256 x 256
    _require_stream_k(fp8, M, N, K)
    a, av = _integer_codes((M, K), "e4m3", 25)
    b, bv = _integer_codes((N, K), "e4m3", 26)
    ad, bd = dev(a), dev(b)
    sa, sb = torch.tensor([0.5], device="cuda"), torch.tensor([4.0], device="cuda")
    assert fp8.fp8ds_device_status() == 0
    d = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    assert fp8._lib.fp8ds_test_stream_k_withhold(1, 5_000_000) == fp8.OK
    try:
        fp8.fp8_gemm_ex(ad, "e4m3", sa, bd, "e4m3", sb, d, workspace=ws)
        torch.cuda.synchronize()
    finally:
        assert fp8._lib.fp8ds_test_stream_k_withhold(0, 0) == fp8.OK
    code = fp8.fp8ds_device_status()                 # read and cleared
    assert code == (5 << 8) | fp8.ERR_TIMEOUT, hex(code)
    assert fp8.fp8ds_device_status() == 0
    assert _flags_clear(ws)
    ref = (torch.from_numpy(av).double() @ torch.from_numpy(bv).double().T) * 2.0
    # tiles computed whole (not split) are exact even in the aborted launch
    got = d.cpu().double()
    assert int((got == ref).sum()) > M * N // 4
    # the next launch, without the setting, is exact everywhere
    d.fill_(float("nan"))
    fp8.fp8_gemm_ex(ad, "e4m3", sa, bd, "e4m3", sb, d, workspace=ws)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    assert torch.equal(d.cpu().double(), ref)
    assert _flags_clear(ws)
