"""Row-sharded quantization of one tensor over several GPUs.

When one tensor (or one per-tensor-scale segment) is split by rows across
ranks, its NVFP4 tensor scale still depends on the amax of the whole
tensor: each rank runs the amax pass on its shard, an all-reduce MAX of the
num_segments floats (NCCL over NVLink) gives every rank the global amax,
and the quantize pass takes it as ``amax_in``.  The result on each rank is
exactly its rows of the unsharded quantization.  MXFP4 and guided
quantization need no exchange (no tensor scale / recorded scales).

Stochastic rounding is not offered sharded: its counter is the element
index within the call, so shards would draw from different positions of the
stream than the unsharded tensor.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as B

# indirection so that the exchange logic can be exercised without a GPU
_ops = {"segment_amax": B.tf4_segment_amax, "quantize_capture": B.tf4_quantize_capture,
        "quantize_rtn": B.tf4_quantize_rtn}


def global_amax(x_shard: torch.Tensor, seg_off=None, group=None) -> torch.Tensor:
    """Per-segment amax of the whole row-sharded tensor (all ranks call this)."""
    amax = _ops["segment_amax"](x_shard, seg_off)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def sharded_capture(x_shard: torch.Tensor, seg_off=None, guidance=True, group=None):
    """Rollout-side capture of this rank's rows under the tensor-wide scale."""
    amax = global_amax(x_shard, seg_off, group)
    return _ops["quantize_capture"](x_shard, seg_off=seg_off, guidance=guidance, amax_in=amax)


def sharded_rtn(x_shard: torch.Tensor, seg_off=None, group=None):
    amax = global_amax(x_shard, seg_off, group)
    return _ops["quantize_rtn"](x_shard, seg_off=seg_off, amax_in=amax)


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous row range [begin, end) of `rank` (balanced, first ranks one larger)."""
    q, r = divmod(rows, world)
    begin = rank * q + min(rank, r)
    return begin, begin + q + (1 if rank < r else 0)


def shard_segments(seg_off, begin: int, end: int):
    """Segment row offsets of rows [begin, end), keeping every segment (empty
    ones included) so that all ranks reduce the same num_segments values."""
    return [min(max(int(o), begin), end) - begin for o in seg_off]
