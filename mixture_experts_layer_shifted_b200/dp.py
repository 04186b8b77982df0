"""Data-parallel replicas of the layer: the one exchange step.

Tokens shard across replicas with no data-path collective; each replica runs
the whole forward on its own batch.  The bias controller is the only state that
must agree: before each controller step the replicas sum their per-expert
selection counts and token counts (one all-reduce of E+1 int64), so every
replica applies the same bit-exact update and keeps an identical bias.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def controller_step(layer, counts_buf: torch.Tensor, group=None, **gains):
    """read accumulators -> all-reduce(sum) over `group` -> write back -> update_bias.

    `layer` provides read_counts(buf), write_counts(buf), update_bias(**gains)
    (ZcMoE does); `counts_buf` is an int64 tensor of E+1 elements on the device
    the collective uses."""
    layer.read_counts(counts_buf)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts_buf, op=dist.ReduceOp.SUM, group=group)
    layer.write_counts(counts_buf)
    layer.update_bias(**gains)
