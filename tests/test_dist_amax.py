"""The data-parallel exchange of delayed scaling on CPU ranks (gloo, world 2).

Each rank casts its own shard of the batch and records its amaxes; before the
update the ranks max-reduce the contiguous row 0 of the [H, T] history (the
amax sync of "support delayed scaling of weight in float8 all-gather").  The
synced scales must equal, bit for bit, the scales of one process that saw the
whole batch, and every rank must end with identical metas.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as o
from fp8_delayed_scaling_cast_b200 import inputs
from fp8_delayed_scaling_cast_b200.dist import sync_amax

WORLD = 2
STEPS = 20
T = 3   # input (e4m3), weight (e4m3), grad (e5m2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _batch(step):
    g = inputs.gen(500 + step)
    x = inputs.uniform((64, 32), g) * (1 + step % 5)
    dy = inputs.normal((64, 16), g, 1e-3).to(torch.bfloat16)
    if step == 3:
        x[17, 3] = 300.0     # a spike on rank 0's half only
    return x, dy


W = inputs.normal((16, 32), inputs.gen(9), 0.02).numpy()


class _HistView:
    """What sync_amax reads from a meta: the [H, T] history as a torch tensor
    (here a view of the oracle's numpy history, sharing its memory)."""

    def __init__(self, hist):
        assert hist.flags["C_CONTIGUOUS"]
        self.amax_history = torch.from_numpy(hist)


def _rank_main(rank, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    meta = o.OracleMeta([o.E4M3, o.E4M3, o.E5M2], 16)
    for step in range(STEPS):
        x, dy = _batch(step)
        lo, hi = rank * 32, (rank + 1) * 32          # this rank's tokens
        xs = x[lo:hi].numpy()
        dys = inputs.bf16_bits(dy[lo:hi])
        _, _, am_x, _ = o.cast_transpose_amax(xs, o.E4M3, meta.scale[0], meta.hist[0, 0])
        _, _, am_w, _ = o.cast_transpose_amax(W, o.E4M3, meta.scale[1], meta.hist[0, 1])
        _, _, am_g, _ = o.cast_transpose_amax(dys, o.E5M2, meta.scale[2], meta.hist[0, 2])
        meta.record(0, am_x)
        meta.record(1, am_w)
        meta.record(2, am_g)
        # the product's exchange, on a torch view that shares the oracle's
        # history memory (row 0 is reduced in place)
        sync_amax(_HistView(meta.hist))
        meta.update()
    out[rank] = (meta.hist.copy(), meta.scale.copy(), meta.scale_inv.copy())
    dist.destroy_process_group()


def _single_process():
    meta = o.OracleMeta([o.E4M3, o.E4M3, o.E5M2], 16)
    traj = []
    for step in range(STEPS):
        x, dy = _batch(step)
        _, _, am_x, _ = o.cast_transpose_amax(x.numpy(), o.E4M3, meta.scale[0], meta.hist[0, 0])
        _, _, am_w, _ = o.cast_transpose_amax(W, o.E4M3, meta.scale[1], meta.hist[0, 1])
        _, _, am_g, _ = o.cast_transpose_amax(inputs.bf16_bits(dy), o.E5M2, meta.scale[2],
                                              meta.hist[0, 2])
        meta.record(0, am_x)
        meta.record(1, am_w)
        meta.record(2, am_g)
        meta.update()
        traj.append(meta.scale.copy())
    return meta, traj


def _spawn_target(rank, port, q):
    res = {}
    _rank_main(rank, port, res)
    q.put((rank, res[rank]))


def test_amax_sync_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_spawn_target, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(WORLD))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref, traj = _single_process()
    for r in range(WORLD):
        h, s, si = results[r]
        assert np.array_equal(h.view(np.uint32), ref.hist.view(np.uint32)), r
        assert np.array_equal(s.view(np.uint32), ref.scale.view(np.uint32)), r
        assert np.array_equal(si.view(np.uint32), ref.scale_inv.view(np.uint32)), r
    # the spike seen by rank 0 alone set the input scale of every rank while it
    # stayed in the window
    assert traj[3][0] == np.float32(448.0) / np.float32(300.0)


def test_unsynced_ranks_diverge():
    """Without the exchange the ranks' scales differ (the exchange is needed)."""
    metas = []
    for rank in range(WORLD):
        meta = o.OracleMeta([o.E4M3], 16)
        x, _ = _batch(3)
        xs = x[rank * 32:(rank + 1) * 32].numpy()
        _, _, am, _ = o.cast_transpose_amax(xs, o.E4M3, 1.0)
        meta.record(0, am)
        meta.update()
        metas.append(meta.scale[0])
    assert metas[0] != metas[1]
