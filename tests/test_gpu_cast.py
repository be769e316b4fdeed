"""GPU parity of fp8_quantize and fp8_cast_transpose_amax against the oracle.

Bit-exact: FP8 bytes, transposed bytes, amax and the private scale_inv.
Covers tiles of the vector path, ragged edges, unaligned pointers, empty
inputs, the special values (NaN, +-inf, -0, fp32 subnormals), the full
cast-transpose-amax workload (bf16 [8192, 2048] with 0.1% spikes, both
formats, scale 1 and fp8_max/amax) and every fp32 bit pattern whose
exponent reaches either format.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, assert_f32_bits_equal, dev, host_bits, u8

pytestmark = pytest.mark.gpu

FMT = {"e4m3": o.E4M3, "e5m2": o.E5M2}
FMAX = {"e4m3": 448.0, "e5m2": 57344.0}


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _gpu_cast_transpose(fp8, x, fmt, scale, amax0=0.0, transpose=True):
    R, C = x.shape
    xd = x.cuda()
    y = torch.full((R, C), 0xAA, dtype=torch.uint8, device="cuda")
    yt = torch.full((C, R), 0xAA, dtype=torch.uint8, device="cuda") if transpose else None
    s = torch.tensor([scale], dtype=torch.float32, device="cuda")
    am = torch.tensor([amax0], dtype=torch.float32, device="cuda")
    si = torch.zeros(1, dtype=torch.float32, device="cuda")
    fp8.fp8_cast_transpose_amax(xd, fmt, s, y, yt, am, si)
    torch.cuda.synchronize()
    return u8(y), (u8(yt) if transpose else None), am.cpu().numpy(), si.cpu().numpy()


def _check_ct(fp8, x, fmt, scale, amax0=0.0, transpose=True):
    y, yt, am, si = _gpu_cast_transpose(fp8, x, fmt, scale, amax0, transpose)
    ry, ryt, ram, rsi = o.cast_transpose_amax(host_bits(x), FMT[fmt], scale, amax0, transpose)
    assert_bytes_equal(y, ry, "y")
    if transpose:
        assert_bytes_equal(yt, ryt, "yt")
    assert_f32_bits_equal(am, [ram], "amax")
    assert_f32_bits_equal(si, [rsi], "scale_inv")


# rows % 16 == 0 and cols % 8 == 0 (16-byte aligned) take the TMA-fed kernel,
# including tiles that reach past the tensor; the others the element kernel.
SHAPES = [(1, 1), (1, 64), (17, 33), (128, 64), (256, 128), (129, 257), (130, 72), (384, 200),
          (16, 8), (2048, 64), (48, 136), (256, 72), (144, 128), (4096, 4104)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_cast_transpose_shapes(fp8, shape, dtype, fmt):
    g = inputs.gen(sum(shape))
    x = (inputs.normal(shape, g) * 40).to(dtype)
    _check_ct(fp8, x, fmt, 1.0)
    _check_ct(fp8, x, fmt, 3.71875, amax0=0.25)


def _gpu_pair(fp8, xa, xb, fmt, sa, sb, transpose, amax0=(0.0, 0.0), noop_b=None):
    """fp8_cast_transpose_amax_pair on fresh outputs (y, yt filled 0xAA)."""
    outs = []
    for x, am0 in ((xa, amax0[0]), (xb, amax0[1])):
        R, C = x.shape
        outs.append([torch.full((R, C), 0xAA, dtype=torch.uint8, device="cuda"),
                     torch.full((C, R), 0xAA, dtype=torch.uint8, device="cuda") if transpose else None,
                     torch.tensor([am0], dtype=torch.float32, device="cuda"), torch.zeros(1, device="cuda")])
    (ya, yta, ama, sia), (yb, ytb, amb, sib) = outs
    fp8.fp8_cast_transpose_amax_pair(xa.cuda(), xb.cuda(), fmt, torch.tensor([sa], device="cuda"), ya,
                                     torch.tensor([sb], device="cuda"), yb, yt_a=yta, amax_a=ama, scale_inv_a=sia,
                                     yt_b=ytb, amax_b=amb, scale_inv_b=sib, noop_b=noop_b)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    return [[u8(t) if t is not None and t.dtype == torch.uint8 else (None if t is None else t.cpu().numpy())
             for t in o_] for o_ in outs]


def _check_against_oracle(got, x, fmt, scale, amax0, transpose, what):
    y, yt, am, si = got
    ry, ryt, ram, rsi = o.cast_transpose_amax(host_bits(x), FMT[fmt], scale, amax0, transpose)
    assert_bytes_equal(y, ry, what + " y")
    if transpose:
        assert_bytes_equal(yt, ryt, what + " yt")
    assert_f32_bits_equal(am, [ram], what + " amax")
    assert_f32_bits_equal(si, [rsi], what + " scale_inv")


# (shape a, shape b, dtype, format, transpose).  Both TMA-eligible: one launch
# whose tiles run over a, then b (a linear's input and weight); b with ragged
# tiles; b not TMA-eligible (cols % 8 != 0): two launches.
PAIRS = [((256, 512), (1024, 256), torch.float32, "e4m3", False),
         ((256, 512), (1024, 256), torch.float32, "e4m3", True),
         ((512, 2048), (144, 136), torch.bfloat16, "e5m2", True),
         ((128, 64), (128, 64), torch.float32, "e5m2", True),
         ((256, 512), (100, 36), torch.float32, "e4m3", False)]


@pytest.mark.parametrize("sa_shape,sb_shape,dtype,fmt,transpose", PAIRS)
def test_cast_pair_matches_oracle(fp8, sa_shape, sb_shape, dtype, fmt, transpose):
    xa = (inputs.normal(sa_shape, inputs.gen(11)) * 40).to(dtype)
    xb = (inputs.normal(sb_shape, inputs.gen(12)) * 300).to(dtype)
    ga, gb = _gpu_pair(fp8, xa, xb, fmt, 3.71875, 0.5, transpose, amax0=(0.25, 1e9))
    _check_against_oracle(ga, xa, fmt, 3.71875, 0.25, transpose, "a")
    _check_against_oracle(gb, xb, fmt, 0.5, 1e9, transpose, "b")


def test_cast_pair_noop_skips_b(fp8):
    """With b's device flag set nothing of b is written; a is cast as usual."""
    xa = inputs.normal((256, 512), inputs.gen(13)) * 40
    xb = inputs.normal((512, 256), inputs.gen(14)) * 40
    for flag in (1, 0):
        f = torch.tensor([flag], dtype=torch.int32, device="cuda")
        ga, gb = _gpu_pair(fp8, xa, xb, "e4m3", 2.0, 4.0, True, amax0=(0.0, 7.5), noop_b=f)
        _check_against_oracle(ga, xa, "e4m3", 2.0, 0.0, True, "a (flag %d)" % flag)
        if flag:
            assert (gb[0] == 0xAA).all() and (gb[1] == 0xAA).all()
            assert gb[2][0] == np.float32(7.5) and gb[3][0] == 0.0
        else:
            _check_against_oracle(gb, xb, "e4m3", 4.0, 7.5, True, "b (flag 0)")


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_cast_transpose_no_transpose_and_empty(fp8, fmt):
    x = inputs.normal((64, 96), inputs.gen(3))
    _check_ct(fp8, x, fmt, 2.0, transpose=False)
    # empty input: only scale_inv is written, amax untouched
    for shape in [(0, 16), (16, 0)]:
        y, yt, am, si = _gpu_cast_transpose(fp8, torch.zeros(shape), fmt, 4.0, amax0=1.5)
        assert am[0] == np.float32(1.5) and si[0] == np.float32(0.25)


def test_cast_transpose_special_values(fp8):
    x = torch.linspace(-3, 3, 128 * 64).reshape(128, 64)
    sv = torch.tensor([float("nan"), float("inf"), -float("inf"), -0.0, 0.0, 1e-40, -1e-40,
                       1e-45, 3.0e38, -3.0e38, 448.0, 464.0, -464.0, 57344.0, 61440.0, 1e-3])
    x.view(-1)[: sv.numel()] = sv
    x.view(-1)[5000: 5000 + sv.numel()] = sv
    for fmt in ("e4m3", "e5m2"):
        for scale in (1.0, 2.0 ** -10, 1024.0):
            _check_ct(fp8, x, fmt, scale)
        # vector path and element path see the same values
        _check_ct(fp8, x[:, :63].contiguous(), fmt, 1.0)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_cast_transpose_unaligned_pointers(fp8, fmt):
    base = inputs.normal((128 * 64 + 3,), inputs.gen(5)) * 10
    x = base[3:].reshape(128, 64)  # 12-byte offset: element path
    R, C = x.shape
    xd = base.cuda()[3:].reshape(R, C)
    ybuf = torch.zeros(R * C + 1, dtype=torch.uint8, device="cuda")
    ytbuf = torch.zeros(R * C + 1, dtype=torch.uint8, device="cuda")
    y, yt = ybuf[1:].view(R, C), ytbuf[1:].view(C, R)
    s = torch.tensor([1.5], device="cuda")
    am = torch.zeros(1, device="cuda")
    si = torch.zeros(1, device="cuda")
    fp8.fp8_cast_transpose_amax(xd, fmt, s, y, yt, am, si)
    torch.cuda.synchronize()
    ry, ryt, ram, rsi = o.cast_transpose_amax(x.numpy(), FMT[fmt], 1.5)
    assert_bytes_equal(u8(y), ry, "y")
    assert_bytes_equal(u8(yt), ryt, "yt")
    assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")
    # sentinel bytes before the outputs untouched
    assert ybuf[0].item() == 0 and ytbuf[0].item() == 0


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_cast_transpose_full_workload(fp8, fmt):
    """bf16 [8192, 2048] ~ N(0,1) with 0.1% of entries x1000 (saturation probes):
    scale 1.0, then the delayed scale fp8_max / amax of the first pass."""
    x = inputs.spiky_bf16()
    y, yt, am, si = _gpu_cast_transpose(fp8, x, fmt, 1.0)
    ry, ryt, ram, rsi = o.cast_transpose_amax(host_bits(x), FMT[fmt], 1.0)
    assert_bytes_equal(y, ry, "y")
    assert_bytes_equal(yt, ryt, "yt")
    assert_f32_bits_equal(am, [ram], "amax")
    s2 = float(np.float32(FMAX[fmt]) / np.float32(ram))
    _check_ct(fp8, x, fmt, s2)


SIZES = [0, 1, 15, 16, 17, 255, 4096 + 5, 1 << 20, 3 * (1 << 20) + 7]


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_quantize_sizes(fp8, n, dtype, fmt):
    x = (inputs.normal((n,), inputs.gen(n + 1)) * 100).to(dtype)
    for offset in (0, 1):
        if offset and n < 2:
            continue
        xs = x[offset:]
        xd = x.cuda()[offset:]
        y = torch.full((xs.numel(),), 0xAA, dtype=torch.uint8, device="cuda")
        s = torch.tensor([0.8125], device="cuda")
        am = torch.tensor([0.5], device="cuda")
        si = torch.zeros(1, device="cuda")
        fp8.fp8_quantize(xd, fmt, s, y, am, si)
        torch.cuda.synchronize()
        ry, ram, rsi = o.quantize(host_bits(xs), FMT[fmt], 0.8125, amax=0.5)
        assert_bytes_equal(u8(y), ry, "y")
        assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")
        assert_f32_bits_equal(si.cpu().numpy(), [rsi], "scale_inv")


def _exhaustive_slices(fmt):
    lo, hi = (-13, 9) if fmt == "e4m3" else (-20, 16)
    return [(s, e + 127) for s in (0, 1) for e in range(lo, hi + 1)]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_quantize_exhaustive_fp32(fp8, fmt):
    """Every fp32 bit pattern with an exponent from far below the smallest
    subnormal to above max, plus every exponent's extreme mantissas and all
    specials, through the GPU cast (scale 1) against the oracle."""
    m = np.arange(1 << 23, dtype=np.uint32)
    slices = _exhaustive_slices(fmt)
    y = torch.empty(1 << 23, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, device="cuda")

    def oracle_slice(args):
        sign, e = args
        bits = (np.uint32(sign) << np.uint32(31)) | (np.uint32(e) << np.uint32(23)) | m
        return o.encode(bits.view(np.float32), FMT[fmt])

    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        refs = ex.map(oracle_slice, slices)
        for (sign, e), ref in zip(slices, refs):
            bits = (np.uint32(sign) << np.uint32(31)) | (np.uint32(e) << np.uint32(23)) | m
            xd = dev(bits.view(np.float32))
            fp8.fp8_quantize(xd, fmt, s, y)
            assert_bytes_equal(u8(y), ref, "exp %d sign %d" % (e - 127, sign))
    # far exponents: the first and last 4096 mantissas of every remaining exponent
    far = [e for e in range(256) if e not in {b for _, b in slices}]
    edge = np.concatenate([np.arange(4096), np.arange((1 << 23) - 4096, 1 << 23)]).astype(np.uint32)
    bits = np.concatenate([(np.uint32(sg) << np.uint32(31)) | (np.uint32(e) << np.uint32(23)) | edge
                           for sg in (0, 1) for e in far])
    v = bits.view(np.float32)
    yd = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    fp8.fp8_quantize(dev(v), fmt, s, yd)
    assert_bytes_equal(u8(yd), o.encode(v, FMT[fmt]), "far exponents")


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_quantize_all_bf16_patterns(fp8, fmt):
    bits = np.arange(1 << 16, dtype=np.uint16)
    x = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    for scale in (1.0, 3.0, 2.0 ** 20):
        y = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
        am = torch.zeros(1, device="cuda")
        fp8.fp8_quantize(x.cuda(), fmt, torch.tensor([scale], device="cuda"), y, am)
        ry, ram, _ = o.quantize(bits, FMT[fmt], scale)
        assert_bytes_equal(u8(y), ry, "bf16 patterns, scale %g" % scale)
        assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")


def test_amax_accumulates_across_calls(fp8):
    """Several casts atomically max into one slot (the meta's slot 0)."""
    am = torch.zeros(1, device="cuda")
    s = torch.ones(1, device="cuda")
    ref = np.float32(0)
    for i in range(5):
        x = inputs.normal((256, 128), inputs.gen(100 + i)) * (i + 1)
        y = torch.empty(256, 128, dtype=torch.uint8, device="cuda")
        fp8.fp8_cast_transpose_amax(x.cuda(), "e4m3", s, y, None, am)
        _, _, ref, _ = o.cast_transpose_amax(x.numpy(), o.E4M3, 1.0, ref, transpose=False)
    torch.cuda.synchronize()
    assert_f32_bits_equal(am.cpu().numpy(), [ref], "amax")


def _oracle_dynamic(x_host, fmt, scale_in):
    """Dynamic scaling from oracle pieces: the tensor's amax, the update with a
    window of one on it (scale kept when the amax is not positive and finite),
    then the cast with that scale."""
    am = o.amax(x_host)
    _, s, si = o.update_scales(np.array([[am]], np.float32), [scale_in], [1.0], [FMT[fmt]], o.AMAX_MOST_RECENT)
    y, yt, _, si2 = o.cast_transpose_amax(x_host, FMT[fmt], s[0])
    assert si2 == si[0]
    return y, yt, am, s[0], si[0]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype,rows,cols", [("bf16", 8192, 2048), ("bf16", 100, 36), ("f32", 256, 192),
                                             ("f32", 37, 53)])
def test_dynamic_scaling_cast(fp8, fmt, dtype, rows, cols):
    x = inputs.normal((rows, cols), inputs.gen(rows + cols), 2.0)
    x[rows // 3, cols // 2] = -300.0
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    xh = host_bits(x)
    xd = x.cuda()
    y = torch.full((rows, cols), 0xAA, dtype=torch.uint8, device="cuda")
    yt = torch.full((cols, rows), 0xAA, dtype=torch.uint8, device="cuda")
    s = torch.tensor([3.0], device="cuda")
    am = torch.tensor([12345.0], device="cuda")       # overwritten, not accumulated
    si = torch.zeros(1, device="cuda")
    fp8.fp8_cast_transpose_amax_dynamic(xd, fmt, s, y, yt, am, si)
    ry, ryt, ram, rs, rsi = _oracle_dynamic(xh, fmt, np.float32(3.0))
    torch.cuda.synchronize()
    assert_bytes_equal(u8(y), ry, "y")
    assert_bytes_equal(u8(yt), ryt, "yt")
    assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")
    assert_f32_bits_equal(s.cpu().numpy(), [rs], "scale")
    assert_f32_bits_equal(si.cpu().numpy(), [rsi], "scale_inv")
    # the largest magnitude lands exactly on the format's max
    assert (ry.reshape(-1)[np.argmax(np.abs(o.bf16_bits_to_f32(xh) if dtype == "bf16" else xh))] & 0x7F) == \
        (0x7E if fmt == "e4m3" else 0x7B)


def test_dynamic_scaling_all_zero_keeps_scale(fp8):
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.full((64, 64), 0xAA, dtype=torch.uint8, device="cuda")
    s = torch.tensor([5.0], device="cuda")
    am = torch.tensor([7.0], device="cuda")
    si = torch.zeros(1, device="cuda")
    fp8.fp8_cast_transpose_amax_dynamic(x, "e4m3", s, y, None, am, si)
    torch.cuda.synchronize()
    assert am.item() == 0.0 and s.item() == 5.0 and si.item() == np.float32(0.2)
    assert bool((y == 0).all())


def test_cast_transpose_beyond_2g_elements(fp8):
    """A bf16 [65536, 32776] cast (2.15e9 elements: more than 2^31, so every
    byte offset past 2 GB must be formed in 64 bits; 32776 columns leave a
    ragged last column tile).  The input is drawn in seeded row chunks
    (generator 4000 + chunk, N(0,1)) straight to the device.  Checked: the
    amax over the whole tensor (oracle amax of every chunk), the scale_inv,
    and the FP8 bytes of sampled rows of y and of yt (oracle casts of those
    rows and columns)."""
    R, C, CH = 65536, 32776, 4096
    xd = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
    am_ref = np.float32(0.0)
    rows = np.array([0, 1, 4095, 4096, 32767, 32768, 65534, 65535], np.int64)
    cols = np.array([0, 1, 63, 64, 16383, 16384, 32767, 32768, 32775], np.int64)
    row_bits, col_bits = {}, np.empty((R, cols.size), np.uint16)
    for c in range(R // CH):
        xc = inputs.normal((CH, C), inputs.gen(4000 + c)).to(torch.bfloat16)
        if c == R // CH - 1:
            xc[CH - 1, C - 1] = 3072.0           # the largest entry (exact in bf16), last row and column
        bits = host_bits(xc)
        am_ref = o.amax(bits, am_ref)
        for r in rows[(rows >= c * CH) & (rows < (c + 1) * CH)]:
            row_bits[int(r)] = bits[r - c * CH].copy()
        col_bits[c * CH:(c + 1) * CH] = bits[:, cols]
        xd[c * CH:(c + 1) * CH].copy_(xc)
        del xc, bits
    s = np.float32(448.0) / np.float32(1000.0)
    y = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    yt = torch.empty(C, R, dtype=torch.uint8, device="cuda")
    sd = torch.tensor([s], device="cuda")
    am = torch.zeros(1, device="cuda")
    si = torch.zeros(1, device="cuda")
    fp8.fp8_cast_transpose_amax(xd, "e4m3", sd, y, yt, am, si)
    torch.cuda.synchronize()
    assert fp8.fp8ds_device_status() == 0
    assert_f32_bits_equal(am.cpu().numpy(), [am_ref], "amax")
    assert am.item() == 3072.0
    assert_f32_bits_equal(si.cpu().numpy(), [np.float32(1.0) / s], "scale_inv")
    ridx = torch.from_numpy(rows).cuda()
    got_rows = y.index_select(0, ridx).cpu().numpy()
    for k, r in enumerate(rows):
        ry, _, _, _ = o.cast_transpose_amax(row_bits[int(r)][None, :], o.E4M3, s, transpose=False)
        assert_bytes_equal(got_rows[k], ry[0], "y row %d" % r)
    got_cols = yt.index_select(0, torch.from_numpy(cols).cuda()).cpu().numpy()
    ry, _, _, _ = o.cast_transpose_amax(np.ascontiguousarray(col_bits.T), o.E4M3, s, transpose=False)
    assert_bytes_equal(got_cols, ry, "yt rows (x columns)")
    del xd, y, yt
    torch.cuda.empty_cache()
