"""Host-side plumbing for running the forward path on several GPUs.

Heads are independent (each has its own codebook and statistics, paper §4.1),
so the path shards with no data-path collective: each rank runs the whole
forward pass on its own batch (weak scaling). The only collectives are the
ones that time the job: a barrier around the timed region and a MAX
all-reduce of the per-rank times, so that the reported time is the slowest
rank's. These helpers work with any torch.distributed backend (nccl on the
GPUs, gloo on the CPU for tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

from . import synthetic as syn


def env_rank_world() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, device: torch.device | None = None, timeout_s: float = 120.0) -> None:
    """Initialise the default process group (short timeout: ranks that wait
    for a dead peer fail instead of hanging)."""
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def rank_workload(wl: syn.Workload, rank: int) -> syn.Workload:
    """The batch rank `rank` processes under weak scaling: same sizes, its own seed."""
    return wl.with_(seed=wl.seed + rank)


def barrier(device: torch.device | None = None) -> None:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(values, device: torch.device | None = None) -> list[float]:
    """Element-wise maximum of `values` over all ranks (identity on one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device or "cpu")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_value(rows_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: all ranks' query rows per second of the slowest rank."""
    return rows_per_rank * world / (ms_per_step / 1e3)
