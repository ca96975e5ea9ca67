"""The combine of the all_reduce form of the layer on W GPUs, one process
per GPU.

Source: Transformers docs, "Expert parallelism", "Choosing an
implementation", the all_reduce row: no token moves and there is no host
synchronisation; every rank holds the same batch, runs its own experts over
it, and an all-reduce sums the ranks' per-token outputs.

Every rank routes the same logits, so the layout (and its rank slabs) comes
out the same on every rank.  Rank r runs moe_grouped_gemm on its experts
(expert_begin = r * E / W, n_experts = E / W) and then calls
``combine_all_reduce``: its fp32 partial (moe_combine_rank), the sum of the
partials across the process group (torch.distributed.all_reduce; NCCL on
GPUs), and one rounding to the output dtype (moe_reduce_partials with a
single partial).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe


def all_reduce_partial(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sums each rank's fp32 partial across the group, in place (a no-op
    without a process group of more than one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


def combine_all_reduce(y, slot_of_pair, topk_w, rank_offsets, rank, partial, out,
                       y_scales=None, group=None, stream=None):
    """This rank's share of the all_reduce form's combine; ``out`` ends up
    the same on every rank."""
    moe.moe_combine_rank(y, slot_of_pair, topk_w, rank_offsets, rank, partial, stream=stream,
                         y_scales=y_scales)
    all_reduce_partial(partial, group)
    moe.moe_reduce_partials(partial.unsqueeze(0), out, stream=stream)
    return out
