"""Host logic for running the front end on several GPUs of one node, one process per GPU.

Frames are independent, so the path needs no exchange between GPUs: each rank runs its own
batch (weak scaling) or its share of one batch's clips (shard_clips, strong scaling). The only
collectives are for measurement: a barrier around the timed region and the maximum of the
ranks' elapsed times (the job is as slow as its slowest rank)."""
from __future__ import annotations

import numpy as np


def shard_clips(sample_offsets, rank: int, world: int):
    """Contiguous share of the clips of one batch for `rank`, balanced by frame count.
    Returns (first clip, last clip + 1, sample offsets of the share rebased to 0)."""
    so = np.asarray(sample_offsets, np.int64)
    n = so.shape[0] - 1
    frames = (so[1:] - so[:-1]) // 800
    cum = np.concatenate([[0], np.cumsum(frames)])
    total = int(cum[-1])
    lo_target = total * rank // world
    hi_target = total * (rank + 1) // world
    c0 = int(np.searchsorted(cum, lo_target, side="left")) if rank > 0 else 0
    c1 = int(np.searchsorted(cum, hi_target, side="left")) if rank < world - 1 else n
    c0 = min(c0, n)
    c1 = max(min(c1, n), c0)
    return c0, c1, so[c0:c1 + 1] - so[c0]


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over all ranks (the identity for one rank)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(frames_per_rank, max_seconds: float) -> float:
    """Tokens per second of the whole job: all ranks' frames over the slowest rank's time."""
    return float(np.sum(frames_per_rank)) / max_seconds
