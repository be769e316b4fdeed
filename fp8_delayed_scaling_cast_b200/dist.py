"""Data-parallel plumbing of the FP8 delayed-scaling path over torch.distributed.

Both functions follow "support delayed scaling of weight in float8
all-gather" (float8_experimental PR #312):

* sync_amax: the amax sync of delayed scaling.  Before the update, every
  rank max-reduces the amaxes recorded in this step, which sit in row 0 of the
  slot-major history as one contiguous buffer.  Every replica then computes
  the same scales, and those equal the single-process scales of the
  concatenated batch: the max of the per-rank maxima is the global max.
* fp8_weight_allgather: FSDP-style weight sharding with delayed scaling.
  Each rank holds a row shard of the fp32 master weight.  The delayed scale
  is known before the weight exists in FP8, so:
  1. every rank casts its own shard with that same scale and records the
     shard's amax (the next sync_amax makes it the global weight amax);
  2. the FP8 bytes are all-gathered, 1 byte per element on the wire instead
     of 4;
  3. the transpose cache is built from the gathered weight.
  The gathered weight equals the cast of the unsharded weight byte for byte,
  and so does its transpose.

The casts and the transpose run in libfp8ds.so; this module only issues the
collectives.  `ops` lets tests on CPU-only gloo ranks substitute host
implementations of the two kernels.
"""
import torch
import torch.distributed as dist


class _KernelOps:
    """The CUDA kernels of the library (the default)."""

    def __init__(self):
        from . import binding
        self.fp8 = binding

    def cast(self, w_shard, meta, t, out8, scale_inv, stream=None):
        self.fp8.fp8_cast_transpose_amax(w_shard, "e4m3", meta.scale[t:t + 1], out8, None,
                                         meta.amax_history[0, t:t + 1], scale_inv, stream=stream)

    def transpose(self, w8, w8t, stream=None):
        self.fp8.fp8_transpose(w8, w8t, stream=stream)


def sync_amax(meta, group=None):
    """All-reduce(MAX) of the amaxes recorded in this step (row 0 of
    meta.amax_history), in place.  Call it on every rank before
    meta.update()."""
    dist.all_reduce(meta.amax_history[0], op=dist.ReduceOp.MAX, group=group)


def fp8_weight_allgather(w_shard, meta, t, w8, w8t, w_scale_inv, group=None, ops=None, stream=None):
    """All-gather an FP8 weight that is sharded by rows across the group.

    w_shard      [N / world, K] fp32, this rank's rows (rank r holds rows
                 r * N / world ... (r + 1) * N / world - 1)
    meta, t      packed meta and the weight's index in it: the cast uses
                 meta.scale[t] and max-es the shard's amax into
                 meta.amax_history[0, t]
    w8           [N, K] uint8 output, the whole FP8 weight on every rank;
                 this rank's rows are cast in place, then gathered
    w8t          [K, N] uint8 output, its transpose (may be None)
    w_scale_inv  [1] fp32 output, the private scale_inv the weight was cast with
    """
    ops = ops if ops is not None else _KernelOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    rows = w_shard.shape[0]
    if w8.shape[0] != rows * world or w8.shape[1] != w_shard.shape[1]:
        raise ValueError("w8 must be [world * shard rows, K]: got %s for shard %s and world %d"
                         % (tuple(w8.shape), tuple(w_shard.shape), world))
    mine = w8[rank * rows:(rank + 1) * rows]
    ops.cast(w_shard, meta, t, mine, w_scale_inv, stream=stream)
    if world > 1:
        if stream is not None:
            torch.cuda.current_stream().wait_stream(stream)
        dist.all_gather_into_tensor(w8, mine, group=group)
    if w8t is not None:
        ops.transpose(w8, w8t, stream=stream)
