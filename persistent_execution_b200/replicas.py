"""Multi-GPU use of the runtime: independent replicas, one process per GPU.

The method has no exchange step between GPUs: each GPU runs its own
persistent kernel over its own op streams (the pages keep the queue on one
device and name no collective). With N processes every rank runs the same
workload on its own GPU (weak scaling); the only collectives are the ones
that time the run: a barrier on both sides of the timed region and a maximum
of the elapsed times, so that the slowest rank sets the job's time.

Launched by torchrun (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR/PORT in the
environment). Every rank takes the same collective steps in the same order.
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass
class Ranks:
    rank: int
    local: int
    world: int


def from_env() -> Ranks:
    return Ranks(int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
                 int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, timeout_s: float = 600.0) -> Ranks:
    """Joins the process group when WORLD_SIZE > 1 (nccl for GPU ranks, gloo on CPU)."""
    r = from_env()
    if r.world > 1:
        import torch.distributed as dist
        if not dist.is_initialized():
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return r


def barrier(r: Ranks) -> None:
    if r.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(r: Ranks, value: float, device: str = "cpu") -> float:
    """The maximum of `value` over all ranks (every rank gets it)."""
    if r.world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, r: Ranks, elapsed_max_s: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * r.world / elapsed_max_s


def finalize(r: Ranks) -> None:
    if r.world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
