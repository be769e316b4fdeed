"""GPU parity of fp8_transpose and of the sharded FP8 weight cast that the
FSDP-style all-gather builds on ("support delayed scaling of weight in float8
all-gather"): row shards cast with the one delayed scale into their slices of
the weight, then the transpose cache from the gathered bytes, equal the
oracle's cast and transpose of the whole weight."""
import socket

import numpy as np
import pytest
import torch

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from tests.gpu_util import assert_bytes_equal, assert_f32_bits_equal, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from fp8_delayed_scaling_cast_b200 import binding
    return binding


@pytest.mark.parametrize("rows,cols", [(8192, 2048), (2048, 8192), (160, 48), (100, 36), (1, 17), (64, 0)])
def test_transpose(fp8, rows, cols):
    y = torch.from_numpy(inputs.fp8_codes((rows, cols), seed=rows + cols).numpy()) if rows * cols else \
        torch.zeros(rows, cols, dtype=torch.uint8)
    yd = y.cuda()
    yt = torch.full((cols, rows), 0xAA, dtype=torch.uint8, device="cuda")
    fp8.fp8_transpose(yd, yt)
    torch.cuda.synchronize()
    assert_bytes_equal(u8(yt), y.numpy().T, "transpose %dx%d" % (rows, cols))


@pytest.mark.parametrize("shards", [2, 4])
def test_sharded_weight_cast_equals_whole(fp8, shards):
    """What every rank does in the all-gather, emulated on one GPU: shard s is
    cast with the shared scale into rows s*N/shards.. of w8 (amaxes max-ed into
    one slot, as the amax sync would), then the transpose of the gathered w8."""
    N, K = 8192, 2048
    w = inputs.normal((N, K), inputs.gen(3), 0.02)
    w[N - 5, 7] = 0.75
    scale = np.float32(448.0) / np.float32(0.6)      # a delayed scale: the spike saturates
    wd = w.cuda()
    w8 = torch.full((N, K), 0xAA, dtype=torch.uint8, device="cuda")
    w8t = torch.full((K, N), 0xAA, dtype=torch.uint8, device="cuda")
    s = torch.tensor([scale], device="cuda")
    am = torch.zeros(1, device="cuda")
    si = torch.zeros(1, device="cuda")
    rows = N // shards
    for sh in range(shards):
        fp8.fp8_cast_transpose_amax(wd[sh * rows:(sh + 1) * rows], "e4m3", s, w8[sh * rows:(sh + 1) * rows], None,
                                    am, si)
    fp8.fp8_transpose(w8, w8t)
    y, yt, ram, rsi = o.cast_transpose_amax(w.numpy(), o.E4M3, scale)
    torch.cuda.synchronize()
    assert_bytes_equal(u8(w8), y, "gathered w8")
    assert_bytes_equal(u8(w8t), yt, "w8 transpose")
    assert_f32_bits_equal(am.cpu().numpy(), [ram], "amax")
    assert_f32_bits_equal(si.cpu().numpy(), [rsi], "scale_inv")


def test_weight_allgather_one_rank_nccl(fp8):
    """fp8_weight_allgather with its CUDA kernels in a one-rank NCCL group:
    the cast lands in place and the transpose follows."""
    import torch.distributed as dist
    from fp8_delayed_scaling_cast_b200.dist import fp8_weight_allgather, sync_amax
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    import datetime
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, K = 512, 256
        w = inputs.normal((N, K), inputs.gen(5), 0.02)
        meta = fp8.Fp8Meta(["e4m3"], hist_len=16)
        w8 = torch.empty(N, K, dtype=torch.uint8, device="cuda")
        w8t = torch.empty(K, N, dtype=torch.uint8, device="cuda")
        si = torch.empty(1, device="cuda")
        for step in range(2):
            fp8_weight_allgather(w.cuda(), meta, 0, w8, w8t, si)
            sync_amax(meta)
            y, yt, am, rsi = o.cast_transpose_amax(w.numpy(), o.E4M3, np.float32(meta.scale[0].item()))
            torch.cuda.synchronize()
            assert_bytes_equal(u8(w8), y, "w8 step %d" % step)
            assert_bytes_equal(u8(w8t), yt, "w8t step %d" % step)
            assert meta.amax_history[0, 0].item() == am
            meta.update()
        assert meta.scale[0].item() == np.float32(448.0) / am
    finally:
        dist.destroy_process_group()
