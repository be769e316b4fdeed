"""GPU parity of fp8_update_scales (one launch over all metas) against the
oracle: amax history, scale and scale_inv bit-exact, over many steps and the
special amaxes (zero, inf, subnormal, quotient overflow)."""
import numpy as np
import pytest
import torch

import oracle as o
from tests.gpu_util import assert_f32_bits_equal, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


@pytest.mark.parametrize("algo", [o.AMAX_MAX, o.AMAX_MOST_RECENT])
@pytest.mark.parametrize("T,H", [(1, 16), (2, 16), (18, 16), (576, 16), (1000, 16), (7, 1),
                                 (130, 3), (33, 1024)])
def test_update_trajectory(fp8, T, H, algo):
    rng = np.random.default_rng(T * 31 + H)
    fmts = rng.integers(0, 2, T).astype(np.uint8)
    hist = np.zeros((H, T), np.float32)
    scale = np.ones(T, np.float32)
    scale_inv = np.ones(T, np.float32)
    dh, ds, dsi, df = dev(hist), dev(scale), dev(scale_inv), dev(fmts)
    for step in range(40):
        am = rng.uniform(0.0, 10.0, T).astype(np.float32) * np.float32(10.0 ** rng.integers(-3, 4))
        am[rng.random(T) < 0.1] = 0.0
        if step == 5:
            am[0] = np.inf
            am[-1] = np.float32(1e-44)
        hist[0] = am
        dh[0].copy_(torch.from_numpy(am))
        hist, scale, scale_inv = o.update_scales(hist, scale, scale_inv, fmts, algo)
        fp8.fp8_update_scales(dh, ds, dsi, df, algo=algo)
        torch.cuda.synchronize()
        assert_f32_bits_equal(dh.cpu().numpy(), hist, "history step %d" % step)
        assert_f32_bits_equal(ds.cpu().numpy(), scale, "scale step %d" % step)
        assert_f32_bits_equal(dsi.cpu().numpy(), scale_inv, "scale_inv step %d" % step)


def test_update_meta_object(fp8):
    meta = fp8.Fp8Meta(["e4m3", "e5m2", "e4m3"], hist_len=16)
    meta.amax_history[0] = torch.tensor([2.0, 4.0, 0.0], device="cuda")
    meta.update()
    torch.cuda.synchronize()
    assert meta.scale.cpu().tolist() == [224.0, 14336.0, 1.0]
    assert meta.amax_history[15].cpu().tolist() == [2.0, 4.0, 0.0]
    assert meta.amax_history[0].abs().sum().item() == 0.0
