"""Multi-GPU plumbing for the recurrence (one process per GPU, torch.distributed).

Every (sequence, head) chain of the gated delta rule is independent, and documents of a
packed stream are independent after the state reset.  Eqs. (1)-(4) of the Qwen3.8-Flash-Next
summary (picx.dev, "Theoretical foundations") are per head.  So the path shards across GPUs
with no exchange step: each rank runs its own share, and only timing or results are reduced.

- ``shard_documents`` splits the documents of a varlen batch across ranks, balancing token
  counts (longest first onto the least-loaded rank).
- ``shard_range`` splits a dense axis (sequences or heads) into contiguous blocks.
- ``max_over_ranks`` takes a scalar's maximum over ranks.  It uses NCCL (CUDA tensor) or
  gloo (CPU tensor), depending on the process group's backend.
"""
from __future__ import annotations

from typing import List, Sequence

import torch
import torch.distributed as dist


def shard_documents(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Document indices per rank, balancing the summed lengths (greedy, longest first).
    Every document lands on exactly one rank; ranks may receive none when there are fewer
    documents than ranks."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda j: (load[j], j))
        out[r].append(i)
        load[r] += int(lengths[i])
    for r in range(world):
        out[r].sort()
    return out


def shard_range(n: int, world: int, rank: int):
    """Contiguous block [start, stop) of range(n) for ``rank``; sizes differ by at most one."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(x: float, group=None) -> float:
    """Maximum of a Python float over all ranks (identity without an initialised group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(x)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
