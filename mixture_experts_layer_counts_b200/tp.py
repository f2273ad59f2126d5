"""Tensor parallelism over the intermediate dimension I (host side).

Rank g of G holds rows [g I/G, (g+1) I/G) of every expert's gate and up
projections and the matching columns of its down projection.  Each rank runs
the layer on its slice (``layer.moe_forward_partial``, fp32 partial output),
the partials are all-gathered into every rank's memory with the process
group's collective (NCCL on GPUs), and ``layer.sum_partials`` adds them in
rank order and rounds once, so every rank ends with the same bf16 output.
Routing is computed on every rank from replicated inputs and is
deterministic.  The expert-parallel alternative (experts split across ranks)
is unbalanced under skewed routing; the split over I streams 1/G of every
active expert on every rank.
"""
from __future__ import annotations

import torch


def shard_bounds(I: int, rank: int, world: int) -> tuple[int, int]:
    """[lo, hi) of the intermediate columns rank `rank` of `world` holds.
    I / world must be a multiple of 128 (the library's tile of I)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the group")
    if I % world or (I // world) % 128:
        raise ValueError(f"I={I} does not split into {world} slices of a multiple of 128")
    n = I // world
    return rank * n, (rank + 1) * n


def shard_expert_weights(w13: torch.Tensor, w2: torch.Tensor, rank: int, world: int):
    """(w13_shard [E, 2 I/G, H], w2_shard [E, H, I/G]) of one rank, contiguous.

    w13 [E, 2I, H] stacks the gate rows [0, I) and the up rows [I, 2I); the
    shard stacks this rank's gate rows and then its up rows.  Per-expert FP8
    scales are unchanged by slicing."""
    E, I2, H = w13.shape
    I = I2 // 2
    lo, hi = shard_bounds(I, rank, world)
    w13_s = torch.cat([w13[:, lo:hi], w13[:, I + lo:I + hi]], dim=1).contiguous()
    w2_s = w2[:, :, lo:hi].contiguous()
    return w13_s, w2_s


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """[G, T, H] fp32 on every rank: the all-gather of the ranks' partials in
    rank order (into local memory)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(partial.shape), dtype=partial.dtype, device=partial.device)
    dist.all_gather_into_tensor(out, partial.contiguous(), group=group)
    return out


def moe_forward_tp(hidden, router_w, router_bias, w13_shard, w2_shard, top_k, w13_scale=None, w2_scale=None,
                   group=None, workspace=None):
    """The layer under tensor parallelism over I: bf16 [T, H], identical on every rank."""
    from . import layer

    part = layer.moe_forward_partial(hidden, router_w, router_bias, w13_shard, w2_shard, top_k,
                                     w13_scale, w2_scale, workspace=workspace)
    return layer.sum_partials(gather_partials(part, group))
