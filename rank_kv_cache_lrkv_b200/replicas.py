"""Data-parallel replicas: one process per GPU, each owning its own sequences.

Every (sequence, KV head) unit is independent, so the decode path shards by
sequence with no exchange on the data path.  Rank r of N owns the B
sequences with global indices r*B .. r*B + B - 1 (weak scaling: the work per
GPU is fixed as N grows).  The only collective is the timing reduction: the
job's time is the maximum over ranks of each rank's device time.
"""
from __future__ import annotations


def shard(wl, rank: int, world: int):
    """The workload of `rank`: the same shapes, sequences offset by rank * B."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    return wl.with_(seq0=wl.seq0 + rank * wl.B)


def owned_sequences(wl, rank: int, world: int) -> range:
    """Global sequence indices owned by `rank`."""
    s = shard(wl, rank, world)
    return range(s.seq0, s.seq0 + s.B)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of `x` over all ranks (x itself when world == 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(B: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job decode tokens/s: every rank decodes B tokens per step."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return B * steps * world / (max_ms * 1e-3)
