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


def test_shard_rows_cover_the_sequence_in_whole_tiles():
    for N, world, tile in [(1000, 2, 128), (65536, 8, 128), (300, 4, 64), (64, 3, 64)]:
        spans = [mg.shard_rows(N, world, r, tile) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == N
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 == b0
        assert all(s0 % tile == 0 for s0, _ in spans)


def _oracle_calls(oracle):
    """The oracle behind the library calls' signatures (tensors in and out),
    so that the host plumbing can be run on CPU ranks."""
    def pre(K, V, cb, M0, C):
        r = oracle.precompute(K.numpy(), V.numpy(), cb.numpy(), M0, C)
        return (torch.from_numpy(r["assign"]), torch.from_numpy(r["counts"]),
                torch.from_numpy(r["vsum"]))

    def att(Q, cb, counts, vsum, M0, C, P, tile, scale):
        r = oracle.attention(Q.numpy(), cb.numpy(), counts.numpy(), vsum.numpy(), M0, C, P, tile, scale)
        return torch.from_numpy(r["O_full"]), torch.from_numpy(r["selected_full"])
    return pre, att


SHARD_WL = dict(B=1, H=2, N=640, d=8, M0=8, C=2, tile=64, dtype="f32", seed=31, n_components=8)


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        from oracle import oracle as orc
        mg.init("gloo", timeout_s=60)
        wl = syn.small_workload(**SHARD_WL)
        inp = syn.generate(wl)
        n0, n1 = mg.shard_rows(wl.N, world, rank, wl.tile)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(inp.f64(a)[:, :, n0:n1]))
        pre, att = _oracle_calls(orc.get())
        out = mg.sequence_sharded_forward(t("K"), t("V"), t("Q"), torch.from_numpy(inp.f64("codebook")),
                                          wl.M0, wl.C, 4, wl.tile, wl.softmax_scale,
                                          precompute=pre, attention=att)
        dist.destroy_process_group()
        q.put((rank, "ok", (n0, n1), [x.numpy() for x in out]))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, f"error: {e!r}", None, None))


def test_sequence_sharded_forward_equals_one_rank(oracle):
    """Two gloo ranks, each with half of every sequence, reproduce the
    single-rank forward pass: global statistics, every local assignment,
    output row and tile selection."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = syn.small_workload(**SHARD_WL)
    inp = syn.generate(wl)
    full_pre = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)
    full_att = oracle.attention(inp.f64("Q"), inp.f64("codebook"), full_pre["counts"], full_pre["vsum"],
                                wl.M0, wl.C, 4, wl.tile, wl.softmax_scale)
    for rank, status, (n0, n1), (assign, counts, vsum, O, sel) in res:
        assert status == "ok", status
        np.testing.assert_array_equal(counts, full_pre["counts"])
        np.testing.assert_allclose(vsum, full_pre["vsum"], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(assign, full_pre["assign"][:, :, n0:n1])
        np.testing.assert_allclose(O, full_att["O_full"][:, :, n0:n1], rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(sel, full_att["selected_full"][:, :, n0 // wl.tile:n1 // wl.tile])


def _deep_oracle_calls(deep):
    """The depth-L oracle behind the depth-L calls' signatures; selected as
    [B, H, ntiles, sum P] (each level's expanded row ids by rank)."""
    def pre(K, V, cb, M0, C, L):
        r = deep.precompute(K.numpy(), V.numpy(), cb.numpy(), M0, C, L)
        return (torch.from_numpy(r["assign"]), torch.from_numpy(r["counts"]),
                torch.from_numpy(r["vsum"]))

    def att(Q, cb, counts, vsum, M0, C, L, P, tile, scale):
        r = deep.attention(Q.numpy(), cb.numpy(), counts.numpy(), vsum.numpy(), M0, C, L, list(P), tile, scale)
        B, H, N, _ = Q.shape
        ntiles = (N + tile - 1) // tile
        sel = np.full((B * H * ntiles, sum(P)), -1, dtype=np.int64)
        for j, levels in enumerate(r["selected"]):
            flat = np.concatenate([np.asarray(x, dtype=np.int64) for x in levels])
            sel[j, :flat.size] = flat
        return torch.from_numpy(r["O_full"]), torch.from_numpy(sel.reshape(B, H, ntiles, sum(P)))
    return pre, att


DEEP_SHARD_WL = dict(B=1, H=2, N=640, d=8, M0=4, C=2, L=3, P=((2, 3),), tile=64, dtype="f32", seed=37,
                     n_components=8)


def _deep_shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        from oracle import deep
        mg.init("gloo", timeout_s=60)
        wl = syn.small_workload(**DEEP_SHARD_WL)
        inp = syn.generate(wl)
        n0, n1 = mg.shard_rows(wl.N, world, rank, wl.tile)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(inp.f64(a)[:, :, n0:n1]))
        pre, att = _deep_oracle_calls(deep)
        out = mg.sequence_sharded_forward_deep(t("K"), t("V"), t("Q"), torch.from_numpy(inp.f64("codebook")),
                                               wl.M0, wl.C, wl.L, wl.P[0], wl.tile, wl.softmax_scale,
                                               precompute=pre, attention=att)
        dist.destroy_process_group()
        q.put((rank, "ok", (n0, n1), [x.numpy() for x in out]))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, f"error: {e!r}", None, None))


def test_sequence_sharded_deep_forward_equals_one_rank():
    """Two gloo ranks, each with half of every sequence, reproduce the
    single-rank depth-3 forward pass: global node statistics, every local
    assignment, output row and per-level tile selection."""
    from oracle import deep
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_deep_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = syn.small_workload(**DEEP_SHARD_WL)
    inp = syn.generate(wl)
    pre, att = _deep_oracle_calls(deep)
    f = lambda a: torch.from_numpy(inp.f64(a))
    assign_f, counts_f, vsum_f = (x.numpy() for x in pre(f("K"), f("V"), f("codebook"), wl.M0, wl.C, wl.L))
    O_f, sel_f = (x.numpy() for x in att(f("Q"), f("codebook"), torch.from_numpy(counts_f),
                                         torch.from_numpy(vsum_f), wl.M0, wl.C, wl.L, wl.P[0], wl.tile,
                                         wl.softmax_scale))
    assert (assign_f >= wl.M0 + wl.M0 * wl.C).any(), "no key reached the deepest level"
    for rank, status, (n0, n1), (assign, counts, vsum, O, sel) in res:
        assert status == "ok", status
        np.testing.assert_array_equal(counts, counts_f)
        np.testing.assert_allclose(vsum, vsum_f, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(assign, assign_f[:, :, n0:n1])
        np.testing.assert_allclose(O, O_f[:, :, n0:n1], rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(sel, sel_f[:, :, n0 // wl.tile:n1 // wl.tile])
