"""FSDP-style FP8 weight all-gather with delayed scaling on CPU ranks (gloo,
world 2) -- "support delayed scaling of weight in float8 all-gather".

Each rank holds a row shard of the fp32 master weight.  fp8_weight_allgather
casts the shard with the delayed scale (known before the cast), all-gathers
the FP8 bytes and builds the transpose; sync_amax max-reduces the recorded
amax before the update.  On these CPU-only ranks the two kernels are stood in
by host implementations (the oracle's cast and a plain byte transpose), so the
test checks the orchestration: shard slicing, the in-place gather, the amax
sync, and that every rank ends with exactly the single-process cast of the
whole weight and the same meta, over three delayed-scaling steps.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs

WORLD = 2
N, K = 64, 48
STEPS = 3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _weight(step):
    w = inputs.normal((N, K), inputs.gen(77), 0.02) * (1.0 + step)
    w[N - 3, 5] = 0.5 * (1.0 + step)       # the largest entry sits in rank 1's shard
    return w


class _HostMeta:
    """The fields of a packed meta as CPU tensors (the library's Fp8Meta holds
    CUDA tensors); update() is the oracle's delayed-scaling update."""

    def __init__(self, hist_len=16):
        self.amax_history = torch.zeros(hist_len, 1)
        self.scale = torch.ones(1)
        self.scale_inv = torch.ones(1)

    def update(self):
        h, s, si = o.update_scales(self.amax_history.numpy(), self.scale.numpy(), self.scale_inv.numpy(), [o.E4M3])
        self.amax_history.copy_(torch.from_numpy(h))
        self.scale.copy_(torch.from_numpy(s))
        self.scale_inv.copy_(torch.from_numpy(si))


class _HostOps:
    """Host stand-ins for the two kernels (the oracle's cast; a byte transpose)."""

    def cast(self, w_shard, meta, t, out8, scale_inv, stream=None):
        y, _, am, si = o.cast_transpose_amax(w_shard.numpy(), o.E4M3, np.float32(meta.scale[t].item()),
                                             np.float32(meta.amax_history[0, t].item()), transpose=False)
        out8.copy_(torch.from_numpy(y))
        meta.amax_history[0, t] = float(am)
        scale_inv.fill_(float(si))

    def transpose(self, w8, w8t, stream=None):
        w8t.copy_(w8.t())


def _rank_main(rank, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    from fp8_delayed_scaling_cast_b200.dist import fp8_weight_allgather, sync_amax
    meta = _HostMeta()
    rows = N // WORLD
    got = []
    for step in range(STEPS):
        shard = _weight(step)[rank * rows:(rank + 1) * rows].contiguous()
        w8 = torch.zeros(N, K, dtype=torch.uint8)
        w8t = torch.zeros(K, N, dtype=torch.uint8)
        si = torch.zeros(1)
        fp8_weight_allgather(shard, meta, 0, w8, w8t, si, ops=_HostOps())
        sync_amax(meta)
        amax_synced = meta.amax_history[0, 0].item()
        meta.update()
        got.append((w8.numpy().copy(), w8t.numpy().copy(), si.item(), amax_synced,
                    meta.amax_history.numpy().copy(), meta.scale.numpy().copy()))
    q.put((rank, got))
    dist.destroy_process_group()


def test_weight_allgather_matches_single_process_cast():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ometa = o.OracleMeta([o.E4M3], 16)
    for step in range(STEPS):
        w = _weight(step).numpy()
        y, yt, am, si = o.cast_transpose_amax(w, o.E4M3, ometa.scale[0], ometa.hist[0, 0])
        ometa.record(0, am)
        for r in range(WORLD):
            w8, w8t, gsi, gam, hist, scale = results[r][step]
            assert np.array_equal(w8, y), (step, r)
            assert np.array_equal(w8t, yt), (step, r)
            assert np.float32(gsi) == si and np.float32(gam) == am, (step, r)
        ometa.update()
        for r in range(WORLD):
            _, _, _, _, hist, scale = results[r][step]
            assert np.array_equal(hist.view(np.uint32), ometa.hist.view(np.uint32)), (step, r)
            assert np.array_equal(scale.view(np.uint32), ometa.scale.view(np.uint32)), (step, r)
    # the weight's scale after step 0 comes from the spike in rank 1's shard
    assert results[0][0][5][0] == np.float32(448.0) / np.float32(0.5)
