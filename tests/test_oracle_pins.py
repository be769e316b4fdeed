"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test checks the oracle against something it does not compute itself:
values the pages print (tests/golden/), a library routine (torch's float8
dtypes and CPU cast, numpy IEEE float32 arithmetic, numpy float64 matmul),
closed forms, or brute force.  A plausible mistake in the oracle (a wrong bias,
a dropped subnormal branch, ties away from zero, a transposed operand, an
off-by-one history window) fails at least one of them.
"""
import json
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as o
from tests.conftest import GOLDEN

FMTS = {o.E4M3: torch.float8_e4m3fn, o.E5M2: torch.float8_e5m2}
NAMES = {o.E4M3: "float8_e4m3fn", o.E5M2: "float8_e5m2"}


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------ formats / finfo --

@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_finfo_table(fmt):
    """max, min, smallest normal and eps as printed in the finfo table."""
    g = _golden("finfo_table.json")[NAMES[fmt]]
    dec = o.decode_table(fmt)
    finite = dec[np.isfinite(dec)]
    assert finite.max() == g["max"]
    assert finite.min() == g["min"]
    # smallest normal: exponent field 1, mantissa 0
    code_sn = 0x08 if fmt == o.E4M3 else 0x04
    assert dec[code_sn] == pytest.approx(g["smallest_normal"], rel=1e-5)
    # it is the smallest positive value with an implicit leading one
    assert dec[code_sn - 1] < dec[code_sn] and dec[code_sn - 1] == (code_sn - 1) * dec[1]
    # eps: distance from 1.0 to the next representable value
    one = int(np.where(dec == 1.0)[0][0])
    assert dec[one + 1] - 1.0 == g["eps"]


def test_code_census():
    """e4m3fn: 254 finite codes + 2 NaN; e5m2: 248 finite + 2 inf + 6 NaN."""
    d4 = o.decode_table(o.E4M3)
    d5 = o.decode_table(o.E5M2)
    assert np.isfinite(d4).sum() == 254 and np.isnan(d4).sum() == 2
    assert np.isfinite(d5).sum() == 248 and np.isinf(d5).sum() == 2 and np.isnan(d5).sum() == 6
    # smallest subnormals 2^-9 and 2^-16
    assert d4[1] == 2.0 ** -9 and d5[1] == 2.0 ** -16


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_decode_matches_torch_dtype(fmt):
    """Library pin: torch's float8 dtype decodes every byte to the same value."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(FMTS[fmt]).to(torch.float64).numpy()
    dec = o.decode_table(fmt)
    assert np.array_equal(np.isnan(ref), np.isnan(dec))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], dec[ok])
    # sign of zero
    assert np.signbit(dec[0x80]) and not np.signbit(dec[0x00])


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_positive_codes_monotone(fmt):
    """The encoder's binary search relies on positive codes decoding in order."""
    dec = o.decode_table(fmt)
    top = 0x7E if fmt == o.E4M3 else 0x7B
    assert np.all(np.diff(dec[: top + 1]) > 0)


# ---------------------------------------------------------------- the cast --

def test_worked_cast_example():
    """The page's worked example: fp32 -> e4m3fn and e5m2 (and bf16) values."""
    g = _golden("worked_cast_example.json")
    x = np.array(g["float32"], np.float32)
    assert np.array_equal(o.decode(o.encode(x, o.E4M3), o.E4M3), np.array(g["float8_e4m3fn"]))
    assert np.array_equal(o.decode(o.encode(x, o.E5M2), o.E5M2), np.array(g["float8_e5m2"]))
    bf = o.bf16_bits_to_f32(o.round_bf16(x.astype(np.float64)))
    assert np.allclose(bf, np.array(g["bfloat16"]), rtol=0, atol=5e-8)


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_round_trip_all_codes(fmt):
    """encode(decode(c)) == c for every finite code; NaN -> 0x7F; inf saturates."""
    dec = o.decode_table(fmt)
    top = 0x7E if fmt == o.E4M3 else 0x7B
    enc = o.encode(dec.astype(np.float32), fmt)
    for c in range(256):
        if np.isnan(dec[c]):
            assert enc[c] == 0x7F
        elif np.isinf(dec[c]):
            assert enc[c] == (top | (c & 0x80))
        else:
            assert enc[c] == c, hex(c)


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_ties_and_saturation(fmt):
    """Hand-picked midpoints go to the even code; overflow saturates; signs kept."""
    dec = o.decode_table(fmt)
    top = 0x7E if fmt == o.E4M3 else 0x7B
    for c in range(0, top):
        mid = np.float32((dec[c] + dec[c + 1]) / 2)  # exact: few significant bits
        assert float(mid) == (dec[c] + dec[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert o.encode(np.array([mid]), fmt)[0] == want
        assert o.encode(np.array([-mid]), fmt)[0] == (want | 0x80)
        up = np.nextafter(mid, np.float32(np.inf))
        dn = np.nextafter(mid, np.float32(0))
        assert o.encode(np.array([up]), fmt)[0] == c + 1
        assert o.encode(np.array([dn]), fmt)[0] == c
    fmax = dec[top]
    big = np.array([fmax * 1.01, fmax * 4, 3e38, np.inf], np.float32)
    assert np.all(o.encode(big, fmt) == top)
    assert np.all(o.encode(-big, fmt) == (top | 0x80))
    assert o.encode(np.array([-1e-30], np.float32), fmt)[0] == 0x80
    assert o.encode(np.array([np.nan], np.float32), fmt)[0] == 0x7F


def _exhaustive_slice(args):
    fmt, sign, exp_biased = args
    m = np.arange(1 << 23, dtype=np.uint32)
    bits = (np.uint32(sign) << np.uint32(31)) | (np.uint32(exp_biased) << np.uint32(23)) | m
    v = bits.view(np.float32)
    mine = o.encode(v, fmt)
    fmax = 448.0 if fmt == o.E4M3 else 57344.0
    ref = torch.from_numpy(v).clamp(-fmax, fmax).to(FMTS[fmt]).view(torch.uint8).numpy()
    bad = np.nonzero(mine != ref)[0]
    return (fmt, sign, exp_biased, bad[:4].tolist(), v[bad[:4]].tolist())


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_encode_matches_torch_exhaustive(fmt):
    """Library pin, exhaustive over every fp32 bit pattern whose exponent can
    reach the format (from well below the smallest subnormal to above max):
    oracle == torch.clamp(v, -max, max).to(fp8) (torch's CPU cast is RNE and
    does not saturate, so the clamp is what saturates)."""
    lo, hi = (-13, 9) if fmt == o.E4M3 else (-20, 16)
    jobs = [(fmt, s, e + 127) for s in (0, 1) for e in range(lo, hi + 1)]
    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        res = list(ex.map(_exhaustive_slice, jobs))
    bad = [r for r in res if r[3]]
    assert not bad, bad[:3]


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
def test_encode_matches_torch_everywhere_sampled(fmt):
    """Same pin on a seeded sample of all finite fp32 patterns (the far ranges
    only underflow to signed zero or saturate)."""
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    fmax = 448.0 if fmt == o.E4M3 else 57344.0
    ref = torch.from_numpy(v.copy()).clamp(-fmax, fmax).to(FMTS[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(o.encode(v, fmt), ref)


def test_scaled_product_and_reciprocal_ieee():
    """fl32(x*s) and fl32(1/s) equal numpy's IEEE float32 multiply and divide."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    s = np.exp(rng.uniform(-30, 30, 20000)).astype(np.float32)
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 3.4e38, np.inf], np.float32)
    x = np.concatenate([x, specials])
    s = np.concatenate([s, np.array([2.0, 3.0, 0.5, 7.0, 2.0, 1.0], np.float32)])
    with np.errstate(over="ignore", under="ignore"):
        ref = x * s
    mine = np.array([o.scaled(a, b) for a, b in zip(x, s)], np.float32)
    assert np.array_equal(mine.view(np.uint32), ref.view(np.uint32))
    with np.errstate(divide="ignore"):
        rr = np.float32(1.0) / s
    mr = np.array([o.reciprocal(b) for b in s], np.float32)
    assert np.array_equal(mr.view(np.uint32), rr.view(np.uint32))


@pytest.mark.parametrize("fmt", [o.E4M3, o.E5M2])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_cast_transpose_amax_properties(fmt, dtype):
    """y = encode(x*s) elementwise (numpy float32 product), yt = y^T exactly,
    amax = max|x| (numpy), scale_inv = 1/s (numpy float32)."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(37, 53, generator=g) * 3
    x[3, 4] = 1e4
    x[5, 6] = -2e5
    s = np.float32(1.7)
    if dtype == "bf16":
        xb = x.to(torch.bfloat16)
        xin = xb.view(torch.int16).numpy().view(np.uint16)
        xf = xb.float().numpy()
    else:
        xin = x.numpy()
        xf = xin
    y, yt, am, si = o.cast_transpose_amax(xin, fmt, s, amax=0.5)
    assert np.array_equal(yt, y.T)
    assert am == np.float32(np.abs(xf).max())
    assert si == np.float32(1.0) / s
    assert np.array_equal(y, o.encode(xf * s, fmt))
    # amax keeps a larger running value
    _, _, am2, _ = o.cast_transpose_amax(xin, fmt, s, amax=1e9, transpose=False)
    assert am2 == np.float32(1e9)
    # NaN inputs do not enter the amax
    xn = np.array(xf, np.float32, copy=True)
    xn[0, 0] = np.nan
    _, _, am3, _ = o.cast_transpose_amax(xn, fmt, s)
    assert am3 == np.float32(np.nanmax(np.abs(xn)))


def test_amax_ignores_every_nan_pattern():
    """Every bf16 bit pattern (quiet and signalling NaNs included): the amax is
    numpy's nanmax of the absolute values."""
    bits = np.arange(1 << 16, dtype=np.uint16)
    v = o.bf16_bits_to_f32(bits)
    _, am, _ = o.quantize(bits, o.E4M3, 1.0)
    assert am == np.nanmax(np.abs(v)) and np.isinf(am)
    # the amax-only reduction over the same patterns, and over the finite ones
    assert o.amax(bits) == am
    finite = bits[np.isfinite(v)]
    assert o.amax(finite) == np.float32(np.abs(o.bf16_bits_to_f32(finite)).max()) == np.float32(3.3895314e38)
    # a history window containing NaN entries ignores them as well
    hist = np.zeros((4, 1), np.float32)
    hist[:, 0] = [np.float32(2.0), np.uint32(0x7F810000).view(np.float32), np.nan, 1.0]
    _, s2, _ = o.update_scales(hist, [1.0], [1.0], [0])
    assert s2[0] == np.float32(224.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_amax_alone(dtype):
    """max|x| of the unscaled input (numpy), a running value kept when larger,
    NaN skipped wherever it sits (first element included), empty input."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((301, 7)) * 4).astype(np.float32)
    x[100, 3] = -768.0
    xin = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else x
    xf = o.bf16_bits_to_f32(xin) if dtype == "bf16" else x
    assert o.amax(xin) == np.float32(np.abs(xf).max()) == np.float32(768.0)
    assert o.amax(xin, amax=1000.0) == np.float32(1000.0)
    xn = np.array(xin, copy=True)
    xn.flat[0] = np.uint16(0x7FC1) if dtype == "bf16" else np.float32(np.nan)
    xn.flat[-1] = np.uint16(0xFF81) if dtype == "bf16" else np.float32(-np.nan)
    assert o.amax(xn) == np.float32(768.0)
    assert o.amax(xin[:0]) == np.float32(0.0)


def test_quantize_is_flat_cast():
    x = np.random.default_rng(1).standard_normal(1001).astype(np.float32)
    y, am, si = o.quantize(x, o.E4M3, 2.0)
    assert np.array_equal(y, o.encode(x * np.float32(2.0), o.E4M3))
    assert am == np.abs(x).max() and si == np.float32(0.5)


# ------------------------------------------------------------------ update --

def _brute_force_trajectory(amaxes, fmt_max, H, s0=1.0):
    """Window of the last H recorded amaxes as a plain list; scale by numpy
    float32 division; previous scale kept when the window max is not > 0 and
    finite or the quotient overflows."""
    recorded, s, out = [], np.float32(s0), []
    for a in amaxes:
        recorded.append(np.float32(a))
        window = recorded[-H:]
        m = max(window)
        if m > 0 and np.isfinite(m):
            with np.errstate(over="ignore"):
                q = np.float32(fmt_max) / np.float32(m)
            if np.isfinite(q):
                s = q
        out.append(s)
    return out


def test_update_matches_brute_force_window():
    rng = np.random.default_rng(5)
    H, T, steps = 16, 5, 45
    fmts = np.array([0, 1, 0, 1, 0], np.uint8)
    amax_seq = rng.uniform(0.01, 5.0, size=(steps, T)).astype(np.float32)
    amax_seq[3, 0] = 1000.0     # spike that must leave the window 16 steps later
    amax_seq[:, 4] = 0.0        # never recorded: scale stays 1
    amax_seq[10, 4] = 2.0
    meta = o.OracleMeta(fmts, H)
    got = []
    for k in range(steps):
        for t in range(T):
            meta.record(t, amax_seq[k, t])
        meta.update()
        got.append(meta.scale.copy())
        assert np.array_equal(meta.scale_inv, np.float32(1.0) / meta.scale)
        assert np.all(meta.hist[0] == 0)
    got = np.array(got)
    for t in range(T):
        fmax = 448.0 if fmts[t] == 0 else 57344.0
        ref = _brute_force_trajectory(amax_seq[:, t], fmax, H)
        assert np.array_equal(got[:, t], np.array(ref, np.float32)), t
    # the spike dominates exactly while it is one of the last 16 amaxes
    assert got[3, 0] == np.float32(448.0) / np.float32(1000.0)
    assert got[3 + H - 1, 0] == np.float32(448.0) / np.float32(1000.0)
    assert got[3 + H, 0] != np.float32(448.0) / np.float32(1000.0)


def test_update_most_recent_is_a_window_of_one():
    """amax_compute_algo "most_recent": the scale follows the current step's
    amax alone (the brute-force window of length 1), zero amaxes keep the
    scale, a spike is forgotten the very next step; the history rolls exactly
    as with "max"."""
    rng = np.random.default_rng(9)
    H, T, steps = 16, 3, 30
    fmts = np.array([0, 1, 0], np.uint8)
    amax_seq = rng.uniform(0.01, 5.0, size=(steps, T)).astype(np.float32)
    amax_seq[4, 0] = 1000.0
    amax_seq[7:12, 2] = 0.0
    amax_seq[20, 1] = np.inf
    recent = o.OracleMeta(fmts, H)
    window = o.OracleMeta(fmts, H)
    got = []
    for k in range(steps):
        for t in range(T):
            recent.record(t, amax_seq[k, t])
            window.record(t, amax_seq[k, t])
        recent.update(algo=o.AMAX_MOST_RECENT)
        window.update()
        got.append(recent.scale.copy())
        assert np.array_equal(recent.hist.view(np.uint32), window.hist.view(np.uint32))
        assert np.array_equal(recent.scale_inv, np.float32(1.0) / recent.scale)
    got = np.array(got)
    for t in range(T):
        fmax = 448.0 if fmts[t] == 0 else 57344.0
        ref = _brute_force_trajectory(amax_seq[:, t], fmax, 1)
        assert np.array_equal(got[:, t], np.array(ref, np.float32)), t
    assert got[4, 0] == np.float32(448.0) / np.float32(1000.0)
    assert got[5, 0] == np.float32(448.0) / amax_seq[5, 0]
    assert np.all(got[7:12, 2] == got[6, 2])          # zero amax: scale kept
    assert got[20, 1] == got[19, 1]                   # infinite amax: scale kept


def test_update_history_layout_closed_form():
    """After k < H steps, slots H-k..H-1 hold the k recorded amaxes oldest first
    and slot 0 is zero."""
    H, k = 16, 6
    meta = o.OracleMeta([0], H)
    vals = [np.float32(v) for v in (1.5, 2.5, 0.25, 7.0, 3.0, 0.125)]
    for v in vals:
        meta.record(0, v)
        meta.update()
    col = meta.hist[:, 0]
    assert np.all(col[: H - k] == 0)
    assert np.array_equal(col[H - k:], np.array(vals, np.float32))


def test_update_special_amaxes_keep_scale():
    hist = np.zeros((16, 4), np.float32)
    hist[0] = [0.0, np.inf, 1e-44, 2.0]
    scale = np.array([3.0, 5.0, 7.0, 1.0], np.float32)
    h2, s2, si2 = o.update_scales(hist, scale, np.ones(4, np.float32), [0, 0, 0, 1])
    assert s2[0] == 3.0 and s2[1] == 5.0 and s2[2] == 7.0       # zero, inf, overflowing quotient
    assert s2[3] == np.float32(57344.0) / np.float32(2.0)
    assert np.array_equal(si2, np.float32(1.0) / s2)
    assert h2[15, 3] == 2.0 and h2[0, 3] == 0.0


# -------------------------------------------------------------------- GEMM --

def _decoded(codes, fmt):
    return o.decode_table(fmt)[codes]


@pytest.mark.parametrize("fa,fb", [(o.E4M3, o.E4M3), (o.E5M2, o.E4M3), (o.E5M2, o.E5M2)])
def test_gemm_matches_numpy_f64(fa, fb):
    """Library pin: numpy float64 matmul of the decoded operands (its own
    summation order) times the scale_invs plus bias."""
    rng = np.random.default_rng(9)
    M, N, K = 37, 29, 96
    top_a = 0x7E if fa == o.E4M3 else 0x7B
    top_b = 0x7E if fb == o.E4M3 else 0x7B
    A = (rng.integers(0, top_a + 1, (M, K)) | (rng.integers(0, 2, (M, K)) << 7)).astype(np.uint8)
    B = (rng.integers(0, top_b + 1, (N, K)) | (rng.integers(0, 2, (N, K)) << 7)).astype(np.uint8)
    bias = rng.standard_normal(N).astype(np.float32)
    sa, sb = np.float32(0.37), np.float32(2.5)
    ref = (_decoded(A, fa) @ _decoded(B, fb).T) * np.float64(sa) * np.float64(sb) + bias
    D = o.gemm(A, fa, B, fb, sa, sb, bias)
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-9 * np.abs(ref).max())
    rows = np.array([5, 0, 36, 17])
    assert np.array_equal(o.gemm(A, fa, B, fb, sa, sb, bias, rows=rows), D[rows])


def test_gemm_hand_example():
    """2x3 . (2x3)^T with small exact values, computed by hand:
    A = [[1, 2, 0.5], [-3, 0.25, 4]], B = [[2, -1, 8], [0.5, 0.5, -2]]
    A.B^T = [[2-2+4, 0.5+1-1], [-6-0.25+32, -1.5+0.125-8]] = [[4, 0.5], [25.75, -9.375]]
    then * 0.5 * 4 (scale_invs) + [1, -1] (bias)."""
    A = o.encode(np.array([[1, 2, 0.5], [-3, 0.25, 4]], np.float32), o.E4M3)
    B = o.encode(np.array([[2, -1, 8], [0.5, 0.5, -2]], np.float32), o.E4M3)
    D = o.gemm(A, o.E4M3, B, o.E4M3, 0.5, 4.0, np.array([1.0, -1.0], np.float32))
    assert np.array_equal(D, np.array([[9.0, 0.0], [52.5, -19.75]]))


def test_round_bf16_pins():
    """Library pin on fp32 inputs (torch's fp32->bf16 is one RNE), plus direct
    rounding of fp64 values that an fp32 detour would double-round."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-80, 80, 100000))).astype(np.float32)
    x = np.concatenate([x, np.array([0.0, -0.0, 1e-40, -1e-40, 3.39e38, 3.4e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.round_bf16(x.astype(np.float64)), ref)
    one = 0x3F80
    assert o.round_bf16(np.array([1 + 2.0 ** -8]))[0] == one                 # tie -> even
    assert o.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == one + 2        # tie -> even (up)
    assert o.round_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == one + 1  # no double rounding
