"""Process-group plumbing for running the GLA forward on several GPUs.

The forward has no exchange step: every (batch, head) sequence is an
independent problem, so N GPUs run N independent batches (weak scaling) and
the only collectives are host-side bookkeeping: a barrier around the timed
region and the max of the per-rank times.  One process per GPU, launched by
torchrun; RANK, LOCAL_RANK, WORLD_SIZE and MASTER_* come from the
environment.  With WORLD_SIZE unset or 1 nothing is initialised.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_world():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def local_device() -> int:
    return int(os.environ.get("LOCAL_RANK", "0"))


def active() -> bool:
    return dist.is_available() and dist.is_initialized()


def init_from_env(backend="nccl", timeout_s=120):
    rank, world = rank_world()
    if world > 1 and not active():
        if backend == "nccl":
            torch.cuda.set_device(local_device())
        dist.init_process_group(backend=backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier():
    if active():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def _reduce_device():
    if dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def max_over_ranks(x: float) -> float:
    """Max of a per-rank scalar (a time) over all ranks."""
    if not active():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not active():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard(n_units: int, rank: int, world: int):
    """Contiguous [start, stop) share of n_units for `rank` (sizes differ by at most one)."""
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def finalize():
    if active():
        dist.destroy_process_group()
