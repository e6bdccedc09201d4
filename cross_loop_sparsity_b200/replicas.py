"""One independent replica per GPU: the rank plumbing of the benchmark.

A decode step of a batch has no exchange between GPUs, so N GPUs run N
independent replicas (weak scaling).  The only collectives are the barriers
around the timed region and the max over ranks of the measured time; no
collective sits on the data path.  Works with NCCL (one GPU per rank) and with
gloo (CPU tensors), so the logic is testable without GPUs.
"""
from __future__ import annotations

import datetime
import os


def env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str | None = None, timeout_s: int = 120):
    """Join the process group when WORLD_SIZE > 1; returns (world, rank, local_rank)."""
    world, rank, local = env()
    if world > 1:
        import torch
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def _device():
    import torch
    import torch.distributed as dist
    return torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world: int, value: float) -> float:
    """The largest of every rank's value (the job's time is its slowest rank's)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


def finish(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
