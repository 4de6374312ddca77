"""Multi-process plumbing for replicas of the layer (one process per GPU).

The layer is token-parallel: every rank runs its own replica on its own tokens
and nothing crosses ranks on the data path.  Ranks only agree on timing: the
job's step time is the slowest rank's, and the job's throughput is all ranks'
tokens over that time (weak scaling).  Works with the "nccl" backend on GPUs
and "gloo" on CPU.
"""
from __future__ import annotations

import os
from datetime import timedelta


def env_ranks():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, timeout_s: int = 300, device=None):
    """Initialise the default process group when more than one rank runs."""
    import torch.distributed as dist
    _, world, _ = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest `value` over all ranks (the job's step time)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, step_s_max: float) -> float:
    """Whole-job tokens per second: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / step_s_max


def finish():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
