"""Host plumbing for running the conv path as independent replicas, one
process per GPU (launched by torch.distributed.run).

The causal conv has no exchange step between GPUs in this library: each
rank runs the same per-GPU workload on its own inputs ("weak" scaling), and
the only collectives are the timing barrier and the max-over-ranks reduction
of the measured time.  The same functions run over NCCL on GPUs and over
gloo on CPU (the tests use the latter).
"""
from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_rank():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Join the process group if WORLD_SIZE > 1 (a short timeout, so ranks
    that wait on a missing peer end with an error instead of hanging)."""
    _, world, _ = env_rank()
    if world <= 1 or dist.is_initialized():
        return
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def world() -> int:
    return dist.get_world_size() if dist.is_initialized() else 1


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device="cpu") -> float:
    """The slowest rank's value (all ranks get it)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, seconds_local: float, device="cpu") -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's
    time."""
    slowest = max_over_ranks(seconds_local, device)
    return world() * units_per_rank / slowest


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own synthetic inputs."""
    return base + 1000 * rank


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
