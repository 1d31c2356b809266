"""Data-parallel host logic for the Atom W4A4 path (one process per GPU).

The path shards over tokens: every rank quantizes and multiplies its own rows
of the activations against its own copy of the quantized weights, so no data
moves between GPUs during the computation. This module holds the little that
the ranks do agree on -- which rows are whose, the slowest rank's time, and
collecting the output rows when a caller wants all of Y on one rank -- written
against torch.distributed so that it runs on NCCL (GPUs) and on gloo (CPU
tests) alike.
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def _world() -> Tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def token_shard(M: int, world: int, rank: int) -> Tuple[int, int]:
    """Row range [start, stop) of rank `rank` when M token rows are split over
    `world` ranks: contiguous, sizes differing by at most one, the larger
    shards first, every row in exactly one shard."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and M >= 0")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's);
    `value` itself when torch.distributed is not initialised or has one rank."""
    world, _ = _world()
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    """Sum of `value` over all ranks (work units processed by the whole job)."""
    world, _ = _world()
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def gather_rows(y_local: torch.Tensor, M: int) -> torch.Tensor:
    """All ranks' output rows, in token order, on every rank: rank r holds the
    rows token_shard(M, world, r) of an [M, N] result in `y_local`. Shards are
    padded to the largest one for the collective and trimmed afterwards."""
    world, rank = _world()
    start, stop = token_shard(M, world, rank)
    if y_local.shape[0] != stop - start:
        raise ValueError(f"rank {rank} holds {y_local.shape[0]} rows, its shard has {stop - start}")
    if world == 1:
        return y_local
    rows = token_shard(M, world, 0)[1]   # the largest shard
    padded = torch.zeros((rows,) + tuple(y_local.shape[1:]), dtype=y_local.dtype,
                         device=y_local.device)
    padded[:stop - start] = y_local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded)
    out = [parts[r][:token_shard(M, world, r)[1] - token_shard(M, world, r)[0]]
           for r in range(world)]
    return torch.cat(out, dim=0)
