"""Independent per-GPU replicas: process-group plumbing for the benchmark.

The attention path has no exchange between GPUs, so N GPUs run N independent
copies of the workload.  What crosses processes is only timing: every rank
times its own K steps on the device, the job's time is the maximum over ranks,
and the job's throughput is the work of all ranks divided by that time.
"""
from __future__ import annotations

import datetime
import os

import torch


def env_world():
    """(rank, world_size, local_rank) from the torchrun environment (1 process if unset)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, ws, local


def init(backend: str = "nccl", timeout_s: int = 120):
    """Join the process group when WORLD_SIZE > 1; returns (rank, world_size, local_rank)."""
    rank, ws, local = env_world()
    if ws <= 1:
        return rank, ws, local
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, **kw)
    return rank, ws, local


def barrier(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int, device=None) -> float:
    """Maximum of a per-rank scalar (e.g. a timed duration) across the job."""
    if ws <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, steps: int, max_ms: float, ws: int) -> float:
    """Units per second for the whole job: all ranks' units over the slowest rank's time."""
    return ws * units_per_rank * steps / (max_ms * 1e-3)


def shutdown(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
