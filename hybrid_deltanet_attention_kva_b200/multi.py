"""Host-side plumbing for running the path on several GPUs of one node.

The path partitions into independent sequences (their DeltaNet states, conv tails
and KV caches never meet), so N GPUs run N disjoint sets of sequences with no data
exchange.  The only collectives are the ones that measurement needs: a barrier and
the maximum of the per-rank device times.  One process per GPU, launched by torchrun
(RANK / LOCAL_RANK / WORLD_SIZE in the environment); NCCL on GPUs, gloo on CPU.
"""
from __future__ import annotations

import datetime
import os
from typing import List, Optional

import torch
import torch.distributed as dist


def env_rank() -> tuple:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0, device: Optional[torch.device] = None) -> None:
    """Join the process group (no-op for a single process)."""
    rank, _, world = env_rank()
    if world == 1 or dist.is_initialized():
        return
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def rank_sequences(n_seq: int, rank: int, world: int) -> List[int]:
    """The contiguous block of sequence ids this rank owns (sizes differ by at most one)."""
    base, extra = divmod(n_seq, world)
    lo = rank * base + min(rank, extra)
    return list(range(lo, lo + base + (1 if rank < extra else 0)))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own inputs: distinct per rank, stable across runs."""
    return seed * 1009 + rank


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(x: float, device: Optional[torch.device] = None) -> float:
    """Maximum of a per-rank scalar (the job's time is its slowest rank's time)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
