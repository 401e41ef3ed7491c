"""Host-side plumbing for running the forward path on several GPUs.

Heads are independent (each has its own codebook and statistics, paper §4.1),
so the path shards with no data-path collective: each rank runs the whole
forward pass on its own batch (weak scaling). The only collectives are the
ones that time the job: a barrier around the timed region and a MAX
all-reduce of the per-rank times, so that the reported time is the slowest
rank's.

For few, long sequences the keys and queries of each (b,h) can instead be
split along N (``sequence_sharded_forward``, and
``sequence_sharded_forward_deep`` for a depth-L tree): every rank assigns its own keys,
one SUM all-reduce of the counts and value sums makes the statistics global,
and every rank attends its own queries. Selection depends only on the global
statistics and on tiles, so tiles must not straddle ranks.

These helpers work with any torch.distributed backend (nccl on the GPUs, gloo
on the CPU for tests).
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


def shard_rows(N: int, world: int, rank: int, tile: int) -> tuple[int, int]:
    """Rows [n0, n1) of a length-N sequence held by `rank` when the sequence is
    split along N into `world` runs of whole tiles (the last rank takes the
    ragged end)."""
    ntiles = (N + tile - 1) // tile
    t0, t1 = (ntiles * rank) // world, (ntiles * (rank + 1)) // world
    return min(N, t0 * tile), min(N, t1 * tile)


def sequence_sharded_forward(K, V, Q, codebook, M0: int, C: int, P: int, tile: int, scale: float,
                             *, precompute=None, attention=None, group=None):
    """The forward path with the keys and queries of every (b,h) split along N
    across the ranks of `group` (``shard_rows`` gives each rank's rows; every
    local N but the last must be a whole number of tiles, so that local tiles
    are global tiles). K, V, Q: this rank's [B,H,n,d]; codebook: the full
    [H,Mtot,d]. Returns (assign of the local keys, global counts, global vsum,
    O of the local queries, selected of the local tiles).

    `precompute` / `attention` default to the library calls of ``binding``
    (callables with their signatures may be passed instead, e.g. by tests)."""
    if precompute is None or attention is None:
        from . import binding
        precompute = precompute or binding.precompute
        attention = attention or binding.attention
    assign, counts, vsum = precompute(K, V, codebook, M0, C)
    _global_statistics(counts, vsum, group)
    O, selected = attention(Q, codebook, counts, vsum, M0, C, P, tile, scale)
    return assign, counts, vsum, O, selected


def sequence_sharded_forward_deep(K, V, Q, codebook, M0: int, C: int, L: int, P, tile: int, scale: float,
                                  *, precompute=None, attention=None, group=None):
    """``sequence_sharded_forward`` over a depth-L codebook tree (the depth-L
    calls; P: one budget per expanded level, L - 1 of them). A node's count
    and value sum are sums over the keys whose path passes through it, so the
    same single SUM all-reduce makes them global; the tile-level selections
    of every level depend only on those and on the tile's own queries.
    codebook: the full [H, Mtot, d] tree. Returns what
    ``sequence_sharded_forward`` returns."""
    if precompute is None or attention is None:
        from . import binding
        precompute = precompute or binding.precompute_deep
        attention = attention or binding.attention_deep
    assign, counts, vsum = precompute(K, V, codebook, M0, C, L)
    _global_statistics(counts, vsum, group)
    O, selected = attention(Q, codebook, counts, vsum, M0, C, L, P, tile, scale)
    return assign, counts, vsum, O, selected


def _global_statistics(counts, vsum, group=None) -> None:
    """Sum the ranks' per-node counts and value sums in place (the one
    exchange step of sequence sharding; nothing on one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(vsum, op=dist.ReduceOp.SUM, group=group)
