"""One process per GPU: process-group set-up, barrier, the max over ranks.

The SAS hot path partitions into independent problems: sequences and kv
groups share nothing, so N ranks run N replicas of the workload and no
collective sits on the data path. The collectives here only align the
timed regions and take the slowest rank's time, so the whole-job rate is
(units per rank x ranks) / max-over-ranks time (weak scaling).

The backend is NCCL on GPUs and gloo on CPU (multi-process tests). Every
process group gets a short timeout, so a rank that fails or never joins
turns the next collective of the others into an error instead of a hang.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_world() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup(backend: str | None = None, timeout_s: float = 120.0) -> tuple[int, int, int]:
    """Join the process group when launched with more than one rank.

    backend: "nccl" (GPU ranks, the default when CUDA is present) or "gloo".
    Returns (world, rank, local rank); with one rank no group is created.
    """
    world, rank, local = env_world()
    use_cuda = torch.cuda.is_available() and backend != "gloo"
    if use_cuda:
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        backend = backend or ("nccl" if use_cuda else "gloo")
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(world: int, x: float) -> float:
    """The largest x over all ranks (a time: the slowest rank's)."""
    if world == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units processed by all ranks per second, over the max-over-ranks time."""
    return units_per_rank * world / (ms * 1e-3)


def teardown(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
