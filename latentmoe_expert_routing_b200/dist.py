"""Multi-process plumbing of the layer (one process per GPU).

Replicas: the layer is token-parallel, every rank runs its own replica on its
own tokens and nothing crosses ranks on the data path.  Ranks only agree on
timing: the job's step time is the slowest rank's, and the job's throughput is
all ranks' tokens over that time (weak scaling).

Expert parallelism (the pages' LatentMoE remark: tokens reach their experts in
the d_latent-wide latent, a quarter of d_model, so that is what crosses GPUs):
rank r holds experts [r E/n, (r+1) E/n); every rank routes all T tokens and
writes its partial latent combine [T, d_latent] fp32; one all-gather brings
every rank's part to every rank; each rank then sums the parts in rank order
and finishes its token shard (fc2 and the shared expert).  Works with the
"nccl" backend on GPUs and "gloo" on CPU.
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


def ep_expert_range(rank: int, n_ranks: int, E: int):
    """Experts [first, last) held by `rank` of `n_ranks` (E % n_ranks == 0)."""
    if E % n_ranks:
        raise ValueError("n_experts must be a multiple of the expert-parallel ranks")
    per = E // n_ranks
    return rank * per, (rank + 1) * per


def ep_token_shard(rank: int, n_ranks: int, T: int):
    """Token rows [t0, t0 + Ts) whose output `rank` finishes: contiguous,
    sizes differing by at most one."""
    base, extra = divmod(T, n_ranks)
    t0 = rank * base + min(rank, extra)
    return t0, base + (1 if rank < extra else 0)


def ep_exchange(part):
    """The latent exchange: every rank's partial combine [T, L] gathered into
    [n_ranks, T, L] on every rank, rank r's part at index r (one all-gather).
    One rank (no process group): the part itself, as [1, T, L]."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return part.unsqueeze(0)
    n = dist.get_world_size()
    out = torch.empty((n * part.shape[0],) + tuple(part.shape[1:]), dtype=part.dtype,
                      device=part.device)
    dist.all_gather_into_tensor(out, part.contiguous())     # rank r's rows at r*T
    return out.view((n,) + tuple(part.shape))


def ep_forward(layer, x, rank: int, n_ranks: int):
    """One expert-parallel layer forward on this rank: partial combine of the
    held experts, the exchange, then this rank's token shard of the output.
    `layer` provides ep_partial(x) -> (zc_part, topk_idx, topk_w) and
    ep_finish(parts, t0, Ts) -> out rows [t0, t0 + Ts).  Returns
    (t0, out_shard, topk_idx, topk_w)."""
    zc, idx, w = layer.ep_partial(x)
    parts = ep_exchange(zc)
    t0, ts = ep_token_shard(rank, n_ranks, x.shape[0])
    return t0, layer.ep_finish(parts, t0, ts), idx, w
