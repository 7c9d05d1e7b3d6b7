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

One case does need an exchange: a single sequence split along time across ranks
(``context_parallel_prefill``).  By eqs. (1)-(3) a token maps the state affinely,
S -> alpha (I - beta kh kh^T) S + beta kh v^T, so a rank's run of tokens is one map
S -> M S + N, computable from its own tokens alone.  The ranks all-gather their maps (one
dk x dk and one dk x dv matrix per sequence and head), each composes the maps of the ranks
before it from S0 to get its start state, and runs its tokens from there.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

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


def _kernel_prefill(q, k, v, alpha, beta, s0, scale, l2norm_qk):
    from . import api
    return api.gdn_prefill(q, k, v, alpha, beta, s0, scale=scale, l2norm_qk=l2norm_qk)


def segment_map(q, k, v, alpha, beta, scale=1.0, l2norm_qk=True,
                prefill: Optional[Callable] = None):
    """The affine map S -> M S + N of a run of tokens (q, k [B,T,H,d], v [B,T,H,d], alpha,
    beta [B,T,H], T >= 1), from two kernel runs: v = 0 from S0 = I gives M, S0 = 0 gives N.
    Returns (M [B,H,d,d], N [B,H,d,d]) fp32."""
    run = prefill or _kernel_prefill
    B, T, H, dk = q.shape
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    _, M = run(q, k, torch.zeros_like(k), alpha, beta, eye, scale, l2norm_qk)
    _, N = run(q, k, v, alpha, beta, None, scale, l2norm_qk)
    return M.contiguous(), N.contiguous()


def start_states(Ms, Ns, S0):
    """The state before every segment, given the segments' maps in order: S^(0) = S0,
    S^(p+1) = M_p S^(p) + N_p.  Returns the list [S^(0), .., S^(P)] (the last one is the state
    after the last segment)."""
    out = [S0]
    for M, N in zip(Ms, Ns):
        out.append(torch.matmul(M, out[-1]) + N)
    return out


def context_parallel_prefill(q, k, v, alpha, beta, s0=None, scale=1.0, l2norm_qk=True,
                             group=None, prefill: Optional[Callable] = None):
    """Prefill of ONE batch of sequences split along time across the ranks of ``group``, in rank
    order: this rank holds tokens [t_r, t_{r+1}) as q, k [B,T_r,H,dk], v [B,T_r,H,dv] and
    alpha, beta [B,T_r,H] (T_r may be 0).  ``s0`` [B,H,dk,dv] (or None for zero) is the state
    before the first token and must be the same on every rank.  Returns this rank's y
    [B,T_r,H,dv] and the state after its last token (on the last rank: the sequence's final
    state).

    Needs dk == dv (the map's M part runs through the same kernels as a dk-column state).  Per
    rank: one run with v = 0 from S0 = I gives M, one from S0 = 0 gives N, an all-gather
    exchanges (M, N), the maps of the earlier ranks are composed from s0 (small GEMMs), and a
    third run from that start state gives y.  ``prefill(q, k, v, alpha, beta, s0, scale,
    l2norm_qk) -> (y, s_final)`` is the kernel call (``api.gdn_prefill`` by default)."""
    run = prefill or _kernel_prefill
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if dk != dv:
        raise ValueError("context-parallel prefill needs dk == dv")
    f32 = dict(dtype=torch.float32, device=q.device)
    S0 = torch.zeros((B, H, dk, dv), **f32) if s0 is None else s0.to(torch.float32)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world == 1:
        if T == 0:
            return v.new_zeros((B, 0, H, dv)), S0.clone()
        return run(q, k, v, alpha, beta, S0, scale, l2norm_qk)
    rank = dist.get_rank(group)
    # 1. this rank's map S -> M S + N, from its own tokens
    if T > 0:
        M, N = segment_map(q, k, v, alpha, beta, scale, l2norm_qk, run)
    else:
        M = torch.eye(dk, **f32).expand(B, H, dk, dk).contiguous()
        N = torch.zeros((B, H, dk, dv), **f32)
    # 2. the exchange: every rank's map
    Ms = [torch.empty_like(M) for _ in range(world)]
    Ns = [torch.empty_like(N) for _ in range(world)]
    dist.all_gather(Ms, M, group=group)
    dist.all_gather(Ns, N, group=group)
    # 3. start state: the maps of ranks 0 .. rank-1 applied to S0 in order
    S = start_states(Ms[:rank], Ns[:rank], S0)[-1]
    # 4. this rank's tokens from their start state
    if T == 0:
        return v.new_zeros((B, 0, H, dv)), S
    return run(q, k, v, alpha, beta, S.contiguous(), scale, l2norm_qk)
