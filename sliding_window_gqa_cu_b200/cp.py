"""Multi-GPU forms of the forward over the ranks of one node (one process per GPU).

Head sharding (no collective): the kv-head groups of the repeat_kv mapping
("muse_glimmer.model" page) are independent problems, so rank r computes the
query heads :func:`head_shard` gives it -- whole kv groups when the kv heads
divide evenly over the ranks, else an even slice of one group's query heads
with that group's K/V replicated -- on the whole pack, and writes exactly those
heads of the output.  :func:`head_sharded_attention_fwd` is the local call.

Context parallelism:

The Magi plans of the "muse_spark.magi_cp" page shard a packed microbatch's
tokens over the context-parallel ranks and let the attention engine exchange
keys and values.  Here rank r owns the contiguous query rows
``shard_bounds(T, world)[r]`` of the pack and its slice of K and V; one
all-gather over NCCL (torch.distributed, NVLink / NVSwitch) assembles the
whole pack's K and V on every rank, and the local step
(:func:`thd_attn_fwd_range`, one kernel launch) computes the rank's rows
against them.  The union of the ranks' outputs is exactly thd_attn_fwd's
result (same arithmetic per row).

:func:`cp_attention_fwd_overlapped` hides the all-gather behind compute: a
rank's rows split their keys into those at or after its first row b (its own
slice: every row of the range can use them at once) and those before b (only
the rows of the one document that crosses b have any).  While the all-gather
runs on NCCL's stream, the rank computes its slice as a pack of its own
(``local_cu_seqlens``: documents cut at b, sinks included); once K/V have
arrived, the crossing document's rows are computed against the keys before b
(:func:`thd_attn_fwd_range` with ``k_end = b``, no sinks) and the two parts
are merged by their log-sum-exps (``thd_attn_merge``).  Same rows as
cp_attention_fwd up to the rounding of the merge.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
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


def gather_kv_async(k_local: torch.Tensor, v_local: torch.Tensor, T: int, group=None):
    """Start the all-gather of :func:`gather_kv` without waiting for it.
    Returns ``(k_full, v_full, finish)``: the output tensors and a callable
    that waits for the collective (with NCCL: makes the current stream wait
    for it) and returns them trimmed to T rows.  A single rank gets its own
    tensors back and a no-op."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return k_local, v_local, lambda: (k_local, v_local)
    world = dist.get_world_size(group)
    chunk = -(-T // world)
    fulls, works = [], []
    for x in (k_local, v_local):
        pad = chunk - x.shape[0]
        xp = torch.nn.functional.pad(x, (0, 0, 0, 0, 0, pad)) if pad else x.contiguous()
        full = torch.empty((chunk * world,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        if dist.get_backend(group) == "nccl":
            works.append(dist.all_gather_into_tensor(full, xp, group=group, async_op=True))
        else:
            works.append(dist.all_gather(list(full.chunk(world)), xp, group=group, async_op=True))
        fulls.append(full)

    def finish():
        for w in works:
            w.wait()
        return fulls[0][:T], fulls[1][:T]

    return fulls[0][:T], fulls[1][:T], finish


def local_cu_seqlens(cu_seqlens, b: int, e: int) -> np.ndarray:
    """Document boundaries of the rows [b, e) as a pack of their own (relative
    to b): the pack's boundaries inside the range, with b and e added, so a
    document that started before b restarts at 0."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    inner = cu[(cu > b) & (cu < e)] - b
    return np.concatenate([[0], inner, [e - b]]).astype(np.int32)


def crossing_rows(cu_seqlens, b: int, e: int) -> int:
    """End of the rows of [b, e) that have keys before b: the rows of the
    document that contains row b and started before it (b when there is none,
    i.e. b is a document start or the range is empty)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if e <= b:
        return b
    d = int(np.searchsorted(cu, b, side="right")) - 1  # cu[d] <= b < cu[d + 1]
    if cu[d] == b:
        return b
    return int(min(cu[d + 1], e))


def cp_rank_parts(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                  cu_seqlens, b: int, e: int, window: int = 0, scale: Optional[float] = None,
                  sinks=None, kv_before=None):
    """The rows [b, e) of the pack from their two key parts.  ``kv_before`` is
    a callable returning the whole pack's (k, v) -- at least its rows before
    b -- and is called only after the own-slice part has been queued, so a
    pending all-gather can run under it.  Returns ``(out, lse)``."""
    from . import thd_attn_fwd, thd_attn_fwd_range, thd_attn_merge

    D = q_local.shape[2]
    if scale is None:
        scale = D ** -0.5
    if e == b:  # an empty shard still takes part in the collective
        kv_before()
        Hq = q_local.shape[1]
        return (torch.empty((0, Hq, D), dtype=q_local.dtype, device=q_local.device),
                torch.empty((0, Hq), dtype=torch.float32, device=q_local.device))
    out, lse = thd_attn_fwd(q_local, k_local, v_local, local_cu_seqlens(cu_seqlens, b, e), window,
                            scale, sinks)
    x = crossing_rows(cu_seqlens, b, e)
    k_full, v_full = kv_before()
    if x > b:
        n = x - b
        out_r, lse_r = thd_attn_fwd_range(q_local[:n], k_full, v_full, cu_seqlens, b, x, window, scale,
                                          None, k_end=b)
        thd_attn_merge(out[:n], lse[:n], out_r, lse_r, out=out[:n], lse=lse[:n])
    return out, lse


def cp_attention_fwd_overlapped(q_local: torch.Tensor, k_local: torch.Tensor,
                                v_local: torch.Tensor, cu_seqlens, window: int = 0,
                                scale: Optional[float] = None, sinks=None, group=None):
    """:func:`cp_attention_fwd` with the K/V all-gather overlapped with the
    part of the rows that needs only this rank's slice (module docstring).
    Same arguments and result."""
    T = int(cu_seqlens[-1])
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    b, e = shard_bounds(T, world)[rank]
    if q_local.shape[0] != e - b or k_local.shape[0] != e - b:
        raise ValueError(f"rank {rank} owns rows [{b}, {e}) of the pack")
    _, _, finish = gather_kv_async(k_local, v_local, T, group)
    return cp_rank_parts(q_local, k_local, v_local, cu_seqlens, b, e, window, scale, sinks, finish)


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


def head_shard(Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int, int, int]:
    """Heads of ``rank`` in the head-sharded forward: ``(q_lo, q_hi, kv_lo,
    kv_hi)``, the query heads [q_lo, q_hi) and the kv heads [kv_lo, kv_hi)
    they read (query head h reads kv head h // (Hq / Hkv)).

    Hkv % world == 0: whole kv groups, Hkv / world of them per rank.
    world % Hkv == 0 and Hq % world == 0: world / Hkv ranks share a group,
    each with Hq / world of its query heads and a copy of its K/V.
    Anything else raises ValueError."""
    if world <= 0 or not (0 <= rank < world) or Hkv <= 0 or Hq % Hkv:
        raise ValueError("need 0 <= rank < world and Hq a multiple of Hkv")
    G = Hq // Hkv
    if Hkv % world == 0:
        n = Hkv // world
        return rank * n * G, (rank + 1) * n * G, rank * n, (rank + 1) * n
    if world % Hkv == 0 and Hq % world == 0:
        per = Hq // world  # query heads per rank, inside one group
        q_lo = rank * per
        g = q_lo // G
        return q_lo, q_lo + per, g, g + 1
    raise ValueError(f"{Hq} query / {Hkv} kv heads do not split evenly over {world} ranks")


def head_sharded_attention_fwd(q_local: torch.Tensor, k_local: torch.Tensor,
                               v_local: torch.Tensor, cu_seqlens, window: int = 0,
                               scale: Optional[float] = None, sinks_local=None):
    """This rank's heads of the packed-THD attention forward: q_local
    [T, q_hi - q_lo, D] and k_local / v_local [T, kv_hi - kv_lo, D] are the
    head slices of :func:`head_shard` (dense, contiguous), sinks_local the
    same query heads' sink logits.  No collective: the result is those heads
    of the whole forward, [T, q_hi - q_lo, D] and [T, q_hi - q_lo]."""
    from . import thd_attn_fwd

    return thd_attn_fwd(q_local, k_local, v_local, cu_seqlens, window, scale, sinks_local)
