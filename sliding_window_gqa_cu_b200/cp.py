"""Context-parallel forward over the ranks of one node (one process per GPU).

The Magi plans of the "muse_spark.magi_cp" page shard a packed microbatch's
tokens over the context-parallel ranks and let the attention engine exchange
keys and values.  Here rank r owns the contiguous query rows
``shard_bounds(T, world)[r]`` of the pack and its slice of K and V; one
all-gather over NCCL (torch.distributed, NVLink / NVSwitch) assembles the
whole pack's K and V on every rank, and the local step
(:func:`thd_attn_fwd_range`, one kernel launch) computes the rank's rows
against them.  The union of the ranks' outputs is exactly thd_attn_fwd's
result (same arithmetic per row).
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


def shard_bounds(T: int, world: int) -> list[tuple[int, int]]:
    """Contiguous token ranges of the ranks: ceil(T / world) tokens each, the
    last rank takes the remainder (possibly empty ranges when T < world)."""
    chunk = -(-T // world) if world > 0 else T
    return [(min(T, r * chunk), min(T, (r + 1) * chunk)) for r in range(world)]


def gather_kv(k_local: torch.Tensor, v_local: torch.Tensor, T: int, group=None):
    """All-gather the ranks' K/V slices into the whole pack's [T, Hkv, D]
    tensors (slices padded to equal length for the collective)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return k_local, v_local
    world = dist.get_world_size(group)
    chunk = -(-T // world)
    outs = []
    for x in (k_local, v_local):
        pad = chunk - x.shape[0]
        xp = torch.nn.functional.pad(x, (0, 0, 0, 0, 0, pad)) if pad else x.contiguous()
        full = torch.empty((chunk * world,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(full, xp, group=group)
        else:
            dist.all_gather(list(full.chunk(world)), xp, group=group)
        outs.append(full[:T])
    return outs[0].contiguous(), outs[1].contiguous()


def cp_attention_fwd(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                     cu_seqlens, window: int = 0, scale: Optional[float] = None, sinks=None,
                     group=None):
    """This rank's rows of the packed-THD attention forward.

    q_local / k_local / v_local: the rank's rows ``shard_bounds(T, world)[rank]``
    of q, k, v; cu_seqlens: host boundaries of the WHOLE pack.  Returns
    ``(out_local, lse_local)`` for the same rows.
    """
    from . import thd_attn_fwd_range

    T = int(cu_seqlens[-1])
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    b, e = shard_bounds(T, world)[rank]
    if q_local.shape[0] != e - b or k_local.shape[0] != e - b:
        raise ValueError(f"rank {rank} owns rows [{b}, {e}) of the pack")
    k_full, v_full = gather_kv(k_local, v_local, T, group)
    return thd_attn_fwd_range(q_local, k_full, v_full, cu_seqlens, b, e, window, scale, sinks)
