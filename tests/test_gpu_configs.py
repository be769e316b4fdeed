"""GPU parity of the full-size linear workloads against the oracle.

* TEBlock forward ("CPU Overhead of te.Linear FP8 Layers", repro script):
  six linears at 8192 tokens, hidden 2048, mlp_ratio 4, fp32 masters, bf16
  outputs, four microbatches with ``is_first_microbatch`` True then False and
  the delayed-scaling update after each microbatch.
* MLP pair 2048 -> 8192 -> 2048 forward + backward at 8192 tokens, 20 steps of
  the delayed-scaling loop (HYBRID: e4m3 forward, e5m2 gradients), dY of step 2
  multiplied by 8 so that an amax spike enters the 16-slot window and leaves it
  at step 18.
* 32 TEBlocks (192 linears, 576 metas) forward for 16 steps, one update
  launch over all metas per step.

What is checked where (the oracle is plain single-threaded C, about 60 ns per
cast element, so full-size checks are split):

* every recorded amax and every meta (history, scale, scale_inv) after every
  update, bit-exactly.  Amaxes of the seeded inputs and weights come from the
  oracle alone; the amaxes of H (fc1's output, cast by fc2) and dH (fc2's dgrad
  output, cast by fc1's backward) are the oracle's amax of the GPU's own H and
  dH (teacher forcing: those tensors are GEMM outputs, equal to the oracle's
  only within the GEMM tolerance);
* FP8 bytes, transposes and private scale_invs of every cast in full on the
  listed steps (the oracle composition ``oracle.linear``), again teacher-forced
  on the GPU's H and dH;
* GEMM outputs on seeded sampled rows (bf16: 1 ulp plus the fp32 accumulation
  allowance; fp32: normwise 1e-5 over the sampled rows).
"""
import numpy as np
import pytest
import torch

import oracle as o
from oracle.linear import OracleLinear, OracleMeta
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import (abs_dot, assert_bytes_equal, assert_f32_bits_equal, check_gemm_bf16,
                            check_gemm_fp32, host_bits, u8)

pytestmark = pytest.mark.gpu

E4, E5 = o.E4M3, o.E5M2


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


def _rows(M, seed, n=12):
    """Seeded sample of output rows: both ends, a tile boundary, the middle."""
    fixed = {0, 1, 127, 128, M // 2, M - 1}
    extra = np.random.default_rng(seed).integers(0, M, n).tolist()
    return np.array(sorted(fixed | set(extra)), np.int64)


def _meta_host(meta):
    return (meta.amax_history.cpu().numpy(), meta.scale.cpu().numpy(), meta.scale_inv.cpu().numpy())


def _check_meta(meta, ometa, what):
    h, s, si = _meta_host(meta)
    assert_f32_bits_equal(h, ometa.hist, what + ": amax history")
    assert_f32_bits_equal(s, ometa.scale, what + ": scale")
    assert_f32_bits_equal(si, ometa.scale_inv, what + ": scale_inv")


def _check_recorded(meta, ometa, what):
    """The amaxes recorded in this step (history slot 0) before the update."""
    assert_f32_bits_equal(meta.amax_history[0].cpu().numpy(), ometa.hist[0], what + ": recorded amaxes")


def _rows_of(t, rows):
    return host_bits(t[torch.from_numpy(rows).to(t.device)])


def _check_bf16_rows(got, rows, exact, a8, fa, b8, fb, sa, sb, K, what):
    """Sampled rows of a bf16 GEMM output against the exact rows."""
    absdot = abs_dot(a8, fa, b8, fb, sa, sb, rows=rows)
    check_gemm_bf16(_rows_of(got, rows), exact, what, absdot=absdot, K=K)


def _check_linear_cache(lin, olin, what):
    assert_bytes_equal(u8(lin.w8), olin.w8, what + ": w8")
    assert_bytes_equal(u8(lin.w8t), olin.w8t, what + ": w8t")
    assert_f32_bits_equal(lin.w_scale_inv.cpu().numpy(), [olin.w_scale_inv], what + ": w scale_inv")


class _Saved:
    """Device buffers a forward keeps for the backward (x8, x8t, private scale_inv)."""

    def __init__(self, M, K, dev="cuda"):
        self.x8 = torch.empty(M, K, dtype=torch.uint8, device=dev)
        self.x8t = torch.empty(K, M, dtype=torch.uint8, device=dev)
        self.si = torch.empty(1, dtype=torch.float32, device=dev)

    def check(self, saved_oracle, what):
        rx8, rx8t, rsi = saved_oracle
        assert_bytes_equal(u8(self.x8), rx8, what + ": x8")
        assert_bytes_equal(u8(self.x8t), rx8t, what + ": x8t")
        assert_f32_bits_equal(self.si.cpu().numpy(), [rsi], what + ": private scale_inv")


# --------------------------------------------------------------- TEBlock --

def test_teblock_forward_four_microbatches(fp8):
    """Six linears, 4 microbatches (is_first_microbatch True, False, False,
    False), update after each.  The weights are cast once, at microbatch 0 with
    the initial scale 1.0, and microbatches 1-3 must use that frozen private
    scale_inv although the meta's weight scales move on; the grad metas are
    never recorded and keep scale 1.0."""
    M = inputs.TOKENS
    ws, bs = inputs.teblock_weights(seed=0)
    L = len(ws)
    fmts = [E4, E4, E5] * L
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"] * L, hist_len=16)
    ometa = OracleMeta(fmts, 16)
    lins, olins = [], []
    for i, (w, b) in enumerate(zip(ws, bs)):
        lins.append(fp8.Fp8Linear(w.cuda(), None if b is None else b.cuda(), 3 * i, 3 * i + 1, 3 * i + 2))
        olins.append(OracleLinear(w.numpy(), None if b is None else b.numpy(), 3 * i, 3 * i + 1, 3 * i + 2))
    saved = [_Saved(M, w.shape[1]) for w in ws]
    outs = [torch.empty(M, w.shape[0], dtype=torch.bfloat16, device="cuda") for w in ws]
    rows = _rows(M, seed=3)
    for mb in range(4):
        flag = mb == 0
        x = inputs.teblock_microbatch(mb)
        xd = x.cuda()
        for i in range(L):
            src = outs[4] if i == 5 else xd            # fc2 consumes fc1's bf16 output
            fp8.fp8_linear_fwd(lins[i], meta, src, outs[i], flag, saved[i].x8, saved[i].x8t, saved[i].si)
        torch.cuda.synchronize()
        h_bits = host_bits(outs[4])
        for i in range(L):
            src = h_bits if i == 5 else x.numpy()
            ry, so = olins[i].fwd(src, ometa, flag, rows=rows)
            what = "microbatch %d linear %d" % (mb, i)
            saved[i].check(so, what)
            _check_linear_cache(lins[i], olins[i], what)
            _check_bf16_rows(outs[i], rows, ry, so[0], E4, olins[i].w8, E4, so[2], olins[i].w_scale_inv,
                             ws[i].shape[1], what + ": Y rows")
        _check_recorded(meta, ometa, "microbatch %d" % mb)
        meta.update()
        ometa.update()
        torch.cuda.synchronize()
        _check_meta(meta, ometa, "after microbatch %d" % mb)
    for i in range(L):
        assert lins[i].w_scale_inv.item() == 1.0               # cast once, with the initial scale
        assert meta.scale[3 * i + 1].item() != 1.0              # while the meta moved on
        assert meta.scale[3 * i + 2].item() == 1.0              # grad meta never recorded


# -------------------------------------------------------------- MLP pair --

MLP_STEPS = 20
MLP_SPIKE_STEP = 2
MLP_FULL_STEPS = (0, 1, 2, 19)    # initial scale, first delayed scale, the spike, after it left


def test_mlp_pair_twenty_steps(fp8):
    M, Hd = inputs.TOKENS, inputs.HIDDEN
    F = inputs.MLP_RATIO * Hd
    w1, b1, w2, b2 = inputs.mlp_pair(seed=0)
    # metas: fc1 (X, W1, dH) and fc2 (H, W2, dY)
    fmts = [E4, E4, E5, E4, E4, E5]
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2", "e4m3", "e4m3", "e5m2"], hist_len=16)
    ometa = OracleMeta(fmts, 16)
    fc1 = fp8.Fp8Linear(w1.cuda(), b1.cuda(), 0, 1, 2)
    fc2 = fp8.Fp8Linear(w2.cuda(), b2.cuda(), 3, 4, 5)
    ofc1 = OracleLinear(w1.numpy(), b1.numpy(), 0, 1, 2)
    ofc2 = OracleLinear(w2.numpy(), b2.numpy(), 3, 4, 5)
    s1, s2 = _Saved(M, Hd), _Saved(M, F)
    g1, g2 = _Saved(M, F), _Saved(M, Hd)          # dH8 / dY8 with transposes and scale_invs
    h = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(M, Hd, dtype=torch.bfloat16, device="cuda")
    dh = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    dx = torch.empty(M, Hd, dtype=torch.bfloat16, device="cuda")
    dw1 = torch.empty(F, Hd, dtype=torch.float32, device="cuda")
    dw2 = torch.empty(Hd, F, dtype=torch.float32, device="cuda")
    w1_am, w2_am = o.amax(w1.numpy()), o.amax(w2.numpy())
    rows_m, rows_f, rows_h = _rows(M, 5), _rows(F, 6), _rows(Hd, 7)
    dy_amaxes = []
    for step in range(MLP_STEPS):
        x, dy = inputs.mlp_step_inputs(step, spike_step=MLP_SPIKE_STEP)
        fp8.fp8_linear_fwd(fc1, meta, x.cuda(), h, True, s1.x8, s1.x8t, s1.si)
        fp8.fp8_linear_fwd(fc2, meta, h, y, True, s2.x8, s2.x8t, s2.si)
        fp8.fp8_linear_bwd(fc2, meta, dy.cuda(), s2.x8t, s2.si, dw2, g2.x8, g2.x8t, g2.si, dx=dh)
        fp8.fp8_linear_bwd(fc1, meta, dh, s1.x8t, s1.si, dw1, g1.x8, g1.x8t, g1.si, dx=dx)
        torch.cuda.synchronize()
        h_bits, dh_bits, dy_bits = host_bits(h), host_bits(dh), host_bits(dy)
        what = "step %d" % step
        if step in MLP_FULL_STEPS:
            ry, so1 = ofc1.fwd(x.numpy(), ometa, True, rows=rows_m)
            s1.check(so1, what + " fc1 input")
            _check_linear_cache(fc1, ofc1, what + " fc1")
            _check_bf16_rows(h, rows_m, ry, so1[0], E4, ofc1.w8, E4, so1[2], ofc1.w_scale_inv, Hd, what + " H rows")
            ry, so2 = ofc2.fwd(h_bits, ometa, True, rows=rows_m)
            s2.check(so2, what + " fc2 input")
            _check_linear_cache(fc2, ofc2, what + " fc2")
            _check_bf16_rows(y, rows_m, ry, so2[0], E4, ofc2.w8, E4, so2[2], ofc2.w_scale_inv, F, what + " Y rows")
            rdh, rdw2, sg2 = ofc2.bwd(dy_bits, ometa, so2, rows_dgrad=rows_m, rows_wgrad=rows_h)
            g2.check(sg2, what + " dY cast")
            _check_bf16_rows(dh, rows_m, rdh, sg2[0], E5, ofc2.w8t, E4, sg2[2], ofc2.w_scale_inv, Hd,
                             what + " dH rows")
            check_gemm_fp32(dw2.cpu().numpy()[rows_h], rdw2, what + " dW2 rows")
            rdx, rdw1, sg1 = ofc1.bwd(dh_bits, ometa, so1, rows_dgrad=rows_m, rows_wgrad=rows_f)
            g1.check(sg1, what + " dH cast")
            _check_bf16_rows(dx, rows_m, rdx, sg1[0], E5, ofc1.w8t, E4, sg1[2], ofc1.w_scale_inv, F,
                             what + " dX rows")
            check_gemm_fp32(dw1.cpu().numpy()[rows_f], rdw1, what + " dW1 rows")
        else:
            # the amaxes each cast records, in the path's order
            for t, src in ((0, x.numpy()), (1, None), (3, h_bits), (4, None), (5, dy_bits), (2, dh_bits)):
                am = {1: w1_am, 4: w2_am}.get(t) if src is None else o.amax(src)
                ometa.record(t, max(ometa.hist[0, t], am))
        dy_amaxes.append(o.amax(dy_bits))
        _check_recorded(meta, ometa, what)
        meta.update()
        ometa.update()
        torch.cuda.synchronize()
        _check_meta(meta, ometa, "after " + what)
        # the window is the last 16 recorded amaxes: the spike of step 2 sets
        # the dY scale exactly while it is inside the window
        window = dy_amaxes[max(0, step - 15):step + 1]
        assert ometa.scale[5] == np.float32(57344.0) / np.float32(max(window))
        if step >= MLP_SPIKE_STEP:
            assert (max(window) == dy_amaxes[MLP_SPIKE_STEP]) == (step < MLP_SPIKE_STEP + 16)


# ------------------------------------------------------- 32-block model --

TOY_BLOCKS = 32
TOY_STEPS = 16
TOY_CHECK_BLOCKS = (0, TOY_BLOCKS - 1)    # H amax checked against the oracle every step
TOY_ALL_BLOCK_STEPS = (0, 7, TOY_STEPS - 1)   # ... and of all 32 blocks on these steps
TOY_FULL_CHECKS = ((0, 0), (TOY_STEPS - 1, TOY_BLOCKS - 1))   # (step, block): casts in full, GEMM rows


def test_toy_model_576_metas(fp8):
    """32 TEBlocks (6 linears each, fc2 consuming fc1's output), 16 forward
    steps with a fresh input each step, weights recast every step
    (is_first_microbatch None), ONE fp8_update_scales launch over the 576
    metas per step.

    Bit-exact every step: all recorded amaxes of X and the weights (oracle), the
    H amaxes of blocks 0 and 31 (oracle amax of the GPU's H), and all 576 metas
    after the update -- the oracle update runs on the oracle's amaxes, taking
    the other 30 blocks' H amaxes as recorded by the GPU (those H are GEMM
    outputs) except on steps 0, 7 and 15, where the H amax of every block is
    the oracle's amax of that block's H.  The grad metas are never recorded: their scale stays 1.0.  Block
    0 at the first step and block 31 at the last: every cast in full and the
    GEMM outputs on sampled rows."""
    M = inputs.TOKENS
    per_block = len(inputs.TEBLOCK_LINEARS)
    T = 3 * per_block * TOY_BLOCKS
    assert T == 576
    fmts = [E4, E4, E5] * (per_block * TOY_BLOCKS)
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"] * (per_block * TOY_BLOCKS), hist_len=16)
    ometa = OracleMeta(fmts, 16)
    lins, w_amax, olins = [], [], {}
    for i, (w, bias) in enumerate(inputs.iter_teblock_weights(seed=0, blocks=TOY_BLOCKS)):
        lins.append(fp8.Fp8Linear(w.cuda(), None if bias is None else bias.cuda(), 3 * i, 3 * i + 1, 3 * i + 2))
        w_amax.append(o.amax(w.numpy()))
        if i // per_block in TOY_CHECK_BLOCKS:
            olins[i] = OracleLinear(w.numpy(), None if bias is None else bias.numpy(), 3 * i, 3 * i + 1, 3 * i + 2)
    assert len(lins) == per_block * TOY_BLOCKS
    K = [lin.in_features for lin in lins[:per_block]]
    N = [lin.out_features for lin in lins[:per_block]]
    saved = [_Saved(M, k) for k in K]                     # reused by every block
    outs = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in N]
    rows = _rows(M, seed=9, n=4)
    fc1, fc2 = per_block - 2, per_block - 1
    for step in range(TOY_STEPS):
        x = inputs.toy_step_input(step)
        xd = x.cuda()
        x_am = o.amax(x.numpy())
        h_am = {}
        for blk in range(TOY_BLOCKS):
            for j in range(per_block):
                i = blk * per_block + j
                src = outs[fc1] if j == fc2 else xd
                fp8.fp8_linear_fwd(lins[i], meta, src, outs[j], None, saved[j].x8, saved[j].x8t, saved[j].si)
            if blk not in TOY_CHECK_BLOCKS and step not in TOY_ALL_BLOCK_STEPS:
                continue
            torch.cuda.synchronize()
            h_bits = host_bits(outs[fc1])
            i_h = blk * per_block + fc2
            h_am[i_h] = o.amax(h_bits)
            assert_f32_bits_equal(meta.amax_history[0, 3 * i_h].cpu().numpy(), h_am[i_h],
                                  "step %d block %d: H amax" % (step, blk))
            if (step, blk) in TOY_FULL_CHECKS:
                ometa_probe = OracleMeta(fmts, 16)
                ometa_probe.scale[:], ometa_probe.scale_inv[:] = ometa.scale, ometa.scale_inv
                for j in range(per_block):
                    i = blk * per_block + j
                    src = h_bits if j == fc2 else x.numpy()
                    ry, so = olins[i].fwd(src, ometa_probe, None, rows=rows)
                    what = "step %d block %d linear %d" % (step, blk, j)
                    saved[j].check(so, what)
                    _check_linear_cache(lins[i], olins[i], what)
                    _check_bf16_rows(outs[j], rows, ry, so[0], E4, olins[i].w8, E4, so[2], olins[i].w_scale_inv,
                                     K[j], what + ": Y rows")
        torch.cuda.synchronize()
        recorded = meta.amax_history[0].cpu().numpy()
        for i in range(per_block * TOY_BLOCKS):
            j = i % per_block
            if j == fc2:
                ometa.record(3 * i, h_am.get(i, recorded[3 * i]))     # oracle amax where checked
            else:
                ometa.record(3 * i, x_am)
            ometa.record(3 * i + 1, w_amax[i])
        _check_recorded(meta, ometa, "step %d" % step)
        meta.update()                                     # one launch for all 576 metas
        ometa.update()
        torch.cuda.synchronize()
        _check_meta(meta, ometa, "after step %d" % step)
    assert np.all(ometa.scale[2::3] == 1.0)
