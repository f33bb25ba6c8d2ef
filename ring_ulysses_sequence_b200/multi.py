"""Process-group plumbing for running one replica of the workload per GPU.

The simulated ring needs no exchange between GPUs: each process runs its own
P-rank ring on its own batch (weak scaling), so the only collectives are the
timing barrier and the max-over-ranks reduction of the measured time.
"""
import os
from datetime import timedelta


def env_ranks():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, timeout_s: float = 120.0, device=None):
    """Initialise the default process group when WORLD_SIZE > 1."""
    import torch.distributed as dist
    rank, world, _ = env_ranks()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        kw = {}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=timedelta(seconds=timeout_s), **kw)
    return rank, world


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (x itself when alone)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shutdown():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
