"""Replica bookkeeping for running the layer on several GPUs at once.

The decode layer does not shard (its one possible exchange, an all-reduce of y,
costs as much as the layer), so N GPUs run N independent replicas. Each rank
draws its own token streams, times its own steps on its own device, and the job
is as fast as its slowest rank: the device timings are reduced with MAX, and the
throughput counts every rank's tokens over that time.
"""
from __future__ import annotations

import torch

STREAM_STRIDE = 1_000_003  # token-stream ids of different ranks never overlap


def token_streams(rank: int, n: int) -> list[int]:
    """Stream ids of the n token batches rank ``rank`` processes."""
    if rank < 0 or n < 0 or n >= STREAM_STRIDE:
        raise ValueError("rank must be >= 0 and 0 <= n < %d" % STREAM_STRIDE)
    return [rank * STREAM_STRIDE + s for s in range(n)]


def max_over_ranks(values_ms, device=None) -> list[float]:
    """Element-wise maximum of per-rank timings (every rank must call it, in the
    same order, with the same number of values)."""
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values_ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(tokens_per_rank: int, world: int, slowest_ms: float) -> float:
    """Whole-job tokens per second: all ranks' tokens over the slowest rank's time."""
    if slowest_ms <= 0 or world <= 0:
        raise ValueError("time and world size must be positive")
    return world * tokens_per_rank / (slowest_ms / 1e3)
