"""The multi-rank host logic with world_size-2 gloo process groups on CPU:
per-rank batches, max-over-ranks timing and the whole-job value. No GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from adaptive_vector_quantized_avq_b200 import multigpu as mg
from adaptive_vector_quantized_avq_b200 import synthetic as syn


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        r, lr, w = mg.env_rank_world()
        assert (r, lr, w) == (rank, rank, world)
        mg.init("gloo", timeout_s=30)
        wl = syn.small_workload(N=64, d=8, M0=4, C=2, dtype="bf16")
        mine = mg.rank_workload(wl, rank)
        inp = syn.generate(mine)
        # each rank times a different amount of "work"; the job time is the max
        fake_ms = [10.0 + rank, 3.0 * (world - rank)]
        mg.barrier()
        mx = mg.max_over_ranks(fake_ms)
        # every rank sees the same maxima
        gathered = [None] * world
        dist.all_gather_object(gathered, (mx, int(inp.K.astype(np.int64).sum()), mine.seed))
        dist.destroy_process_group()
        q.put((rank, "ok", gathered))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, f"error: {e!r}", None))


@pytest.mark.parametrize("world", [2])
def test_gloo_two_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, status, gathered in res:
        assert status == "ok", status
        maxima = [g[0] for g in gathered]
        assert all(m == [10.0 + world - 1, 3.0 * world] for m in maxima)
        # weak scaling: ranks process different seeded batches
        seeds = [g[2] for g in gathered]
        assert seeds == list(range(world))
        sums = [g[1] for g in gathered]
        assert len(set(sums)) == world


def test_single_rank_helpers_without_process_group():
    assert mg.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    mg.barrier()
    assert mg.weak_scaling_value(1000, 4, 2.0) == pytest.approx(2e6)
    wl = syn.WORKLOADS["max-64k"]
    assert mg.rank_workload(wl, 3).seed == wl.seed + 3
    assert mg.rank_workload(wl, 3).rows == wl.rows
