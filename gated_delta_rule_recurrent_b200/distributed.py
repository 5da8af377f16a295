"""Multi-GPU plumbing for the decode step: one process per GPU, no data-path
collective.

Every (item, value head) of the decode step is independent, so one logical
call splits across N GPUs with no exchange step: by batch item (each rank
holds the pool slots its items name) or by value head (each rank holds its
heads of every slot, as tensor-parallel serving does). ``shard_call`` cuts
one call's arguments into a rank's share and ``gather_call`` puts the ranks'
results back together; a multi-GPU step runs each share on its own GPU. The
only cross-rank traffic of the benchmark is timing bookkeeping: a barrier
around the timed region, the maximum of the per-rank elapsed times, and the
sum of the units processed. These helpers work with any torch.distributed
backend (NCCL on GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

__all__ = ["rank_env", "rank_seed", "max_over_ranks", "sum_over_ranks", "throughput",
           "Shard", "shard_bounds", "shard_call", "gather_call"]

# Argument names of one call (the op page's, plus the fused gate's inputs).
_ITEM_AXIS0 = ("query", "key", "value", "beta", "g", "gk", "a", "b", "actual_seq_lengths",
               "ssm_state_indices", "num_accepted_tokens")


@dataclasses.dataclass(frozen=True)
class Shard:
    """One rank's share of a call: items [lo, hi) (by="item") or value heads
    [lo, hi) with query/key heads [qk_lo, qk_hi) (by="head"). For an item
    shard, ``slots`` lists the slots of the full pool that the rank's compact
    pool holds, row by row."""

    by: str
    world: int
    rank: int
    lo: int
    hi: int
    qk_lo: int = 0
    qk_hi: int = 0
    slots: Optional[torch.Tensor] = None


def shard_bounds(n: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of rank ``rank`` in a contiguous split of n units over ``world``
    ranks; the first n % world ranks take one unit more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_call(x: Dict[str, object], world: int, rank: int,
               by: str = "item") -> Tuple[Dict[str, object], Shard]:
    """Rank ``rank``'s share of the call whose arguments are ``x`` (the names of
    ``workloads.make_inputs``; tensors on any device).

    by="item": items [lo, hi) of a contiguous split, with a compact pool of the
    slots those items name (indices remapped; an index outside the pool stays
    outside, so the item is still skipped). by="head": value heads [lo, hi)
    and the query/key heads they read; needs H_v and H_qk divisible by
    ``world`` (value head h reads query/key head h // (H_v / H_qk), so equal
    blocks of both line up). Returns (the share's arguments, the Shard)."""
    B, H_qk = x["query"].shape[0], x["query"].shape[1]
    H_v = x["value"].shape[1]
    pool = x["state_pool"]
    out: Dict[str, object] = dict(x)
    if by == "item":
        lo, hi = shard_bounds(B, world, rank)
        for k in _ITEM_AXIS0:
            if x.get(k) is not None:
                out[k] = x[k][lo:hi]
        idx = x["ssm_state_indices"][lo:hi].to(torch.int64)
        P = pool.shape[0]
        valid = (idx >= 0) & (idx < P)
        slots = torch.unique(idx[valid])
        remap = torch.full((P,), -1, dtype=torch.int64, device=idx.device)
        remap[slots] = torch.arange(slots.numel(), device=idx.device)
        # keep out-of-pool indices out of the compact pool too
        local = torch.where(valid, remap[idx.clamp(0, P - 1)], torch.full_like(idx, -1))
        out["ssm_state_indices"] = local.to(x["ssm_state_indices"].dtype)
        out["state_pool"] = pool[slots].clone() if slots.numel() else pool[:1].clone()
        return out, Shard("item", world, rank, lo, hi, slots=slots)
    if by == "head":
        if H_v % world or H_qk % world:
            raise ValueError("a head split needs H_v and H_qk divisible by the world size")
        lo, hi = rank * H_v // world, (rank + 1) * H_v // world
        qlo, qhi = rank * H_qk // world, (rank + 1) * H_qk // world
        for k in ("query", "key"):
            out[k] = x[k][:, qlo:qhi].contiguous()
        for k in ("value", "beta", "g", "gk"):
            if x.get(k) is not None:
                out[k] = x[k][:, lo:hi].contiguous()
        for k in ("a", "b"):  # [B, T, H_v]: heads last
            if x.get(k) is not None:
                out[k] = x[k][:, :, lo:hi].contiguous()
        for k in ("dt_bias", "decay_scale"):
            if x.get(k) is not None:
                out[k] = x[k][lo:hi].contiguous()
        out["state_pool"] = pool[:, lo:hi].contiguous()
        return out, Shard("head", world, rank, lo, hi, qlo, qhi)
    raise ValueError('by must be "item" or "head"')


def gather_call(outs: Sequence[torch.Tensor], pools: Sequence[torch.Tensor],
                shards: Sequence[Shard], pool_before: torch.Tensor
                ) -> Tuple[torch.Tensor, torch.Tensor]:
    """The whole call's (out, state pool) from every rank's share, in rank order.

    Item shards: outputs stacked along the items, and each rank's compact pool
    written back to the slots it holds (slots no rank holds keep
    ``pool_before``'s values). Head shards: both stacked along the heads."""
    order = sorted(range(len(shards)), key=lambda i: shards[i].rank)
    shards = [shards[i] for i in order]
    outs = [outs[i] for i in order]
    pools = [pools[i] for i in order]
    if any(s.by != shards[0].by for s in shards):
        raise ValueError("all shards must split the same way")
    if shards[0].by == "item":
        pool = pool_before.clone()
        for s, p in zip(shards, pools):
            if s.slots is not None and s.slots.numel():
                pool[s.slots.to(pool.device)] = p.to(pool.device, pool.dtype)
        return torch.cat(list(outs), dim=0), pool
    return torch.cat(list(outs), dim=1), torch.cat(list(pools), dim=1)


def rank_env() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s batch: distinct per rank, equal to ``base_seed`` on rank 0."""
    return base_seed + 7919 * rank


def _reduce(value: float, op, device: Optional[torch.device]) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The maximum of ``value`` over all ranks (the value itself without a process group)."""
    return _reduce(value, dist.ReduceOp.MAX, device)


def sum_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The sum of ``value`` over all ranks (the value itself without a process group)."""
    return _reduce(value, dist.ReduceOp.SUM, device)


def throughput(local_units: float, local_seconds: float,
               device: Optional[torch.device] = None) -> Tuple[float, float]:
    """Whole-job throughput: units processed by all ranks over the slowest rank's time.

    Returns (units per second, slowest time in seconds).
    """
    units = sum_over_ranks(local_units, device)
    seconds = max_over_ranks(local_seconds, device)
    return units / seconds, seconds
