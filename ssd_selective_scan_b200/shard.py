"""Data-parallel sharding of the layer over ranks (one process per GPU).

The prefill and decode work of the Mamba-2 layer splits into independent
sequences: every (sequence, head) chain carries its own state, and no step
reads another sequence's tokens or state.  A global batch is therefore split
by sequence across ranks; each rank runs the layer on its own sequences and
the data path needs no collective.  Only timing crosses ranks: a step takes
as long as its slowest rank.
"""
from __future__ import annotations

import torch


def batch_shard(b_global: int, rank: int, world: int) -> tuple[int, int]:
    """The sequences [start, stop) that rank `rank` of `world` owns out of
    `b_global`: contiguous, in rank order, sizes differing by at most one."""
    if world <= 0 or not 0 <= rank < world or b_global < 0:
        raise ValueError(f"bad shard request: b={b_global} rank={rank} world={world}")
    base, extra = divmod(b_global, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic batch (weak scaling: every rank runs a
    full batch of different sequences)."""
    return base_seed + rank


def max_over_ranks(value: float, device: torch.device | str | None = None) -> float:
    """Maximum of `value` over the ranks of the default process group, or
    `value` itself without one.  `device` must suit the backend: a CUDA
    device for NCCL, the CPU for gloo."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput of a weak-scaled step: all ranks' tokens over the
    step time taken as the maximum over ranks."""
    if ms_per_step <= 0:
        raise ValueError("step time must be positive")
    return world * tokens_per_rank / (ms_per_step * 1e-3)
