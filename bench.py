#!/usr/bin/env python
"""Throughput of the AVQ-attention forward path on B200.

One step = the whole hot path over one batch of synthetic input:
``avq_precompute`` (assignment + full-tree statistics) then ``avq_attention``
(parent attention, importance, top-P, child correction, output), through the
C ABI. Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--P P]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

Multi-GPU (N > 1, launched by torch.distributed.run): every rank runs the
same workload on its own seeded batch (heads are independent, no data-path
collective): weak scaling, value = all ranks' query rows / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from adaptive_vector_quantized_avq_b200 import synthetic as syn  # noqa: E402

METRIC = "AVQ forward queries/sec and % of roofline (HBM/tensor) at N=64k, 1×B200"
UNIT = "queries/s"
DEFAULT_WORKLOAD = "max-64k"
L2_BYTES = 126 * 2 ** 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


# ----------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def algorithmic(wl: syn.Workload, P):
    """Per-call algorithmic bytes and tensor FLOPs (paper Table 1 cost model):
    precompute reads K and V and evaluates M0 + C distances per key;
    attention reads Q, writes O and evaluates M0 + P*C logits and weighted
    sums per query. A depth-L tree (P one budget per expanded level) takes
    M0 + (L-1) C distances per key and M0 + C sum_l P_l logits per query."""
    s = 2 if wl.dtype == "bf16" else 4
    R, d = wl.rows, wl.d
    if wl.L > 2:
        dist = wl.M0 + (wl.L - 1) * wl.C
        logits = wl.M0 + wl.C * sum(P)
    else:
        dist = wl.M0 + wl.C
        logits = wl.M0 + P * wl.C
    return {
        "precompute": {"bytes": 2 * R * d * s, "flops": 2 * R * dist * d},
        "attention": {"bytes": 2 * R * d * s, "flops": 4 * R * logits * d},
    }


def default_P(wl: syn.Workload, P_arg=None):
    """The refinement budget a run uses: --P, else the workload's default
    (the largest of refine-d128's sweep; the per-level tuple of a deep tree)."""
    if wl.L > 2:
        return tuple(wl.P[0])
    if P_arg is not None:
        return P_arg
    return wl.P[-1 if wl.name == "refine-d128" else 0]


def n_selected(P) -> int:
    return sum(P) if isinstance(P, tuple) else P


def call_precompute(bd, wl, shape, K, V, cb, assign, counts, vsum, ws, stream):
    if wl.L > 2:
        return bd.avq_precompute_deep(shape, wl.L, K, V, cb, assign, counts, vsum, stream)
    return bd.avq_precompute(shape, K, V, cb, assign, counts, vsum, ws, ws.numel(), stream)


def call_attention(bd, wl, shape, Q, cb, counts, vsum, P, scale, O, sel, ws, stream):
    if wl.L > 2:
        return bd.avq_attention_deep(shape, wl.L, P, Q, cb, counts, vsum, wl.tile, scale, O, sel, ws, ws.numel(),
                                     stream)
    return bd.avq_attention(shape, Q, cb, counts, vsum, P, wl.tile, scale, O, sel, ws, ws.numel(), stream)


def attention_ws_bytes(bd, wl, shape, P) -> int:
    if wl.L > 2:
        return bd.avq_attention_deep_workspace_bytes(shape, wl.L)
    return bd.avq_attention_workspace_bytes(shape, P, wl.tile)


def roofline_for(kind, alg, ms, peaks, sustained):
    hbm = peaks["hbm_gbs"]
    tf = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_hbm = alg["bytes"] / (hbm * 1e9)
    t_ten = alg["flops"] / (tf * 1e12)
    sec = ms / 1e3
    if t_ten > t_hbm:
        ach = alg["flops"] / sec / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": tf, "unit": "TFLOP/s", "frac": ach / tf,
                "roofline_us": t_ten * 1e6}
    ach = alg["bytes"] / sec / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
            "roofline_us": t_hbm * 1e6}


# the sources the two calls' kernels are built from (tree, flat and depth-L
# paths, with the shared headers and the entry points); other kernels of the
# library do not change their traffic
KERNEL_SOURCES = ("avq_api.cu", "avq_internal.cuh", "avq_sm100.cuh", "avq_tma.cu", "avq_precompute_tc.cu",
                  "avq_attention_tree.cu", "avq_attention_tc.cu", "avq_deep.cu")


def kernel_source_hash(kind: str, deep: bool = False) -> str:
    """Hash of the sources a call's kernels are built from (to invalidate stored
    ncu traffic): the depth-L kernels for a deeper tree, else the others."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "adaptive_vector_quantized_avq_b200", "csrc")
    shared = ("avq_api.cu", "avq_internal.cuh", "avq_sm100.cuh")
    names = shared + (("avq_deep.cu",) if deep else tuple(n for n in KERNEL_SOURCES if n not in shared + ("avq_deep.cu",)))
    for n in sorted(names):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def stored_traffic(kind: str, workload: str, P: int):
    """DRAM bytes per launch from a committed ncu capture, if the kernel sources
    are unchanged since it was taken; else None."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    e = d.get(f"{kind}/{workload}/P{P}")
    if not e or e.get("source_hash") != kernel_source_hash(kind, syn.WORKLOADS[workload].L > 2):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the GPU works."""

    Q = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
         "utilization.gpu")

    def __init__(self, bus_id: str | None, period_ms: int = 50):
        self.bus_id = bus_id
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                   f"-lms={self.period_ms}", f"--filename={self.path}"]
            if self.bus_id:
                cmd.insert(1, f"--id={self.bus_id}")
            self.proc = subprocess.Popen(cmd, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(self.period_ms / 1000 * 2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 11:
                    continue
                try:
                    rows.append({"sm": float(p[2]), "max": float(p[3]), "power": float(p[4]),
                                 "hw": p[6], "hwt": p[7], "swt": p[8], "pcap": p[9],
                                 "util": float(p[10])})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(busy), "power_w_max": max(r["power"] for r in busy)}


def bus_id_of(torch, dev: int) -> str | None:
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ------------------------------------------------------- CPU oracle timing
class OracleSampler:
    """The fp64 oracle timed on a bounded sample of the workload: whole (b,h)
    sequences (keys through the precompute, then every query tile through the
    attention with that sequence's statistics), as many as fit the time budget;
    when even one sequence does not fit, the first whole tiles of one. Inputs
    and the statistics the attention reads are prepared untimed, like inputs
    already resident. A depth-L tree uses the numpy depth-L oracle."""

    def __init__(self, wl: syn.Workload, P):
        self.wl, self.P = wl, P
        if wl.L > 2:
            from oracle import deep
            self.deep = deep
            self.threads = 1
        else:
            from oracle import oracle as orc
            self.O = orc.get()
            self.deep = None
            self.threads = self.O.max_threads()
        self.one = wl.with_(B=1, H=1)
        self.ntiles = self.one.ntiles
        self.heads = [self._head(0)]
        self.n_heads, self.n_tiles = 1, self.ntiles

    def _pre(self, K, V, cb):
        wl = self.wl
        if self.deep is not None:
            return self.deep.precompute(K, V, cb, wl.M0, wl.C, wl.L)
        return self.O.precompute(K, V, cb, wl.M0, wl.C, nthreads=self.threads)

    def _head(self, i: int):
        inp = syn.generate(self.one.with_(seed=self.wl.seed + 7919 * i))
        K, V, Q, cb = (inp.f64(n) for n in ("K", "V", "Q", "codebook"))
        return K, V, Q, cb, self._pre(K, V, cb)

    def _one(self, h, n_tiles: int) -> int:
        wl = self.wl
        K, V, Q, cb, full = h
        n = min(wl.N, n_tiles * wl.tile)
        self._pre(K[:, :, :n], V[:, :, :n], cb)
        if self.deep is not None:
            self.deep.attention(Q, cb, full["counts"], full["vsum"], wl.M0, wl.C, wl.L, self.P, wl.tile,
                                wl.softmax_scale, tile_ids=np.arange(n_tiles))
        else:
            self.O.attention(Q, cb, full["counts"], full["vsum"], wl.M0, wl.C, self.P, wl.tile,
                             wl.softmax_scale, tile_ids=np.arange(n_tiles), nthreads=self.threads)
        return n

    def plan(self, seconds: float) -> None:
        """Choose the sample for a budget of about `seconds` of oracle work."""
        t0 = time.perf_counter()
        self._one(self.heads[0], 2)
        per_row = (time.perf_counter() - t0) / min(self.wl.N, 2 * self.wl.tile)
        per_head = per_row * self.wl.N
        if per_head > seconds:
            self.n_heads = 1
            self.n_tiles = int(max(1, min(self.ntiles, math.ceil(seconds / per_row / self.wl.tile))))
        else:
            self.n_heads = int(max(1, min(self.wl.B * self.wl.H, seconds // per_head)))
            self.n_tiles = self.ntiles
            while len(self.heads) < self.n_heads:
                self.heads.append(self._head(len(self.heads)))

    def run(self):
        t0 = time.perf_counter()
        rows = sum(self._one(h, self.n_tiles) for h in self.heads[:self.n_heads])
        return rows, time.perf_counter() - t0

    def describe(self) -> str:
        wl = self.wl
        if self.n_heads > 1 or self.n_tiles == self.ntiles:
            what = (f"{self.n_heads} whole (b,h) sequence(s) of {wl.N} keys and {wl.N} queries "
                    f"of {wl.name} ({self.n_heads * wl.N} rows)")
        else:
            n = min(wl.N, self.n_tiles * wl.tile)
            what = (f"{n} keys precomputed + {n} queries attended ({self.n_tiles} tiles of {wl.tile}) "
                    f"of one (b,h) sequence of {wl.name}")
        if self.deep is not None:
            return f"{what}; fp64 depth-L oracle (numpy, one thread)"
        return f"{what}; fp64 oracle, {self.threads} OpenMP threads"


# --------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from adaptive_vector_quantized_avq_b200 import binding as bd
    from adaptive_vector_quantized_avq_b200 import multigpu as mg

    rank, local, world = mg.env_rank_world()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        mg.init("nccl", dev)

    wl = syn.WORKLOADS[args.workload]
    P = default_P(wl, args.P)
    wl_rank = mg.rank_workload(wl, rank)
    inp = syn.generate(wl_rank)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def to_dev(a):
        if wl.dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16) if wl.dtype == "bf16" else a)
        return t.pin_memory()

    K, V, Q, cb = (to_dev(getattr(inp, n)) for n in ("K", "V", "Q", "codebook"))
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    Mtot = wl.Mtot
    shape = bd.make_shape(B, H, N, d, wl.M0, wl.C, tdt)
    # Inputs read per step (Q, K, V). When they would fit in L2 several copies
    # rotate from step to step, so that every step reads its inputs from HBM:
    # between two uses of a copy at least twice the L2 of other data is read.
    in_bytes = 3 * wl.rows * d * (2 if wl.dtype == "bf16" else 4)
    nrot = 1 if in_bytes >= 2 * L2_BYTES else int(math.ceil(3 * L2_BYTES / in_bytes))
    sets = [(K, V, Q)] + [(K.clone(), V.clone(), Q.clone()) for _ in range(nrot - 1)]
    if nrot == 1:
        l2_note = (f"no flush: Q+K+V = {in_bytes / 1e6:.0f} MB per step >= 2x the "
                   f"{L2_BYTES / 1e6:.0f} MB L2")
    else:
        l2_note = (f"{nrot} input copies rotated step to step: Q+K+V = {in_bytes / 1e6:.0f} MB per step "
                   f"< 2x the {L2_BYTES / 1e6:.0f} MB L2, {nrot * in_bytes / 1e6:.0f} MB cycled")
    assign = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    counts = torch.empty((B, H, Mtot), dtype=torch.int32, device=dev)
    vsum = torch.empty((B, H, Mtot, d), dtype=torch.float32, device=dev)
    O = torch.empty_like(Q)
    sweep_P = list(wl.P) if (wl.L == 2 and len(wl.P) > 1) else []
    Pmax = max([n_selected(P)] + sweep_P)
    sel_buf = torch.empty((B, H, wl.ntiles, max(Pmax, 1)), dtype=torch.int32, device=dev)
    ws_pre = bd.workspace(bd.avq_precompute_workspace_bytes(shape) if wl.L == 2 else 256, dev)
    ws_att = bd.workspace(max(attention_ws_bytes(bd, wl, shape, p_) for p_ in sweep_P + [P]), dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = wl.softmax_scale

    ncalls = [0]   # precompute calls so far (its status block sums the fp64 re-decisions)

    def step(i, P_, ev=None):
        ncalls[0] += 1
        Ki, Vi, Qi = sets[i % nrot]
        k_ = n_selected(P_)
        sel = sel_buf[..., :k_] if k_ > 0 else None
        if ev is not None:
            ev[0].record(stream)
        rc = call_precompute(bd, wl, shape, Ki, Vi, cb, assign, counts, vsum, ws_pre, sp)
        if ev is not None:
            ev[1].record(stream)
        rc2 = call_attention(bd, wl, shape, Qi, cb, counts, vsum, P_, scale, O, sel, ws_att, sp)
        if ev is not None:
            ev[2].record(stream)
        if rc or rc2:
            raise RuntimeError(f"avq call failed: {rc} {rc2}")

    def barrier():
        mg.barrier(dev)

    def timed(P_, nsteps):
        """Times nsteps steps at refinement budget P_ (after the warm-up):
        (total ms, per-call precompute ms, per-call attention ms, launches)."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nsteps)]
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        launches0 = bd.avq_kernel_launches()
        start.record(stream)
        for i in range(nsteps):
            step(i, P_, evs[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        launches = bd.avq_kernel_launches() - launches0
        barrier()
        return (start.elapsed_time(stop), [e[0].elapsed_time(e[1]) for e in evs],
                [e[1].elapsed_time(e[2]) for e in evs], launches)

    # warm-up
    for i in range(args.warmup):
        step(i, P)
    torch.cuda.synchronize(dev)
    if bd.avq_device_status(ws_pre, sp) or bd.avq_device_status(ws_att, sp):
        raise RuntimeError("device status error after warm-up")

    clocks = ClockSampler(bus_id_of(torch, local))
    clocks.start()
    ms_total, pre_ms, att_ms, launches = timed(P, args.steps)
    clk = clocks.stop()
    if bd.avq_device_status(ws_pre, sp) or bd.avq_device_status(ws_att, sp):
        raise RuntimeError("device status error after timing")
    # throughput against the refinement budget (a workload that lists several
    # P): the same step timed at each of them
    sweep = []
    if sweep_P:
        for P_ in sweep_P:
            for i in range(args.warmup):
                step(i, P_)
            t_, pre_, att_, _ = timed(P_, args.steps)
            sweep.append((P_, t_ / args.steps, statistics.mean(pre_), statistics.mean(att_)))
        if bd.avq_device_status(ws_pre, sp) or bd.avq_device_status(ws_att, sp):
            raise RuntimeError("device status error in the P sweep")
    # keys whose parent / leaf the fp32 bounds could not certify, re-decided in
    # fp64 by the precompute kernel (counters in its status block, summed over
    # the warm-up and timed calls)
    diag = ws_pre[:16].view(torch.int32).cpu().tolist()
    redecided = [diag[2] / ncalls[0], diag[3] / ncalls[0]]

    # end to end through the public API: pinned host inputs in, output out.
    # The (b,h) sequences are independent, so the step is cut into chunks of
    # whole batches (or heads, when B == 1) issued round-robin on a few
    # streams: a chunk's inputs go up while an earlier chunk computes and its
    # output comes down (the two copy directions overlap on the link).
    hK, hV, hQ, hcb = (pinned(getattr(inp, n)) for n in ("K", "V", "Q", "codebook"))
    hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    nsel = n_selected(P)
    sel = sel_buf[..., :nsel].contiguous() if nsel > 0 else None
    hsel = torch.empty(sel.shape, dtype=sel.dtype).pin_memory() if nsel > 0 else None
    e2e_steps = max(3, min(args.steps, 20))
    along_b = B > 1
    n_units = B if along_b else H
    n_chunks = min(4, n_units)
    bounds = [round(i * n_units / n_chunks) for i in range(n_chunks + 1)]
    streams = [torch.cuda.Stream(dev) for _ in range(min(3, n_chunks))]
    ws_chunks = []
    for i in range(n_chunks):
        u = bounds[i + 1] - bounds[i]
        cshape = bd.make_shape(u if along_b else 1, H if along_b else u, N, d, wl.M0, wl.C, tdt)
        ws_chunks.append((cshape, bd.workspace(bd.avq_precompute_workspace_bytes(cshape) if wl.L == 2 else 256, dev),
                          bd.workspace(attention_ws_bytes(bd, wl, cshape, P), dev)))

    def sl(t, i):
        a, b_ = bounds[i], bounds[i + 1]
        return t[a:b_] if along_b else t[:, a:b_]

    def e2e_step():
        ev_cb = torch.cuda.Event()
        with torch.cuda.stream(streams[0]):
            streams[0].wait_stream(stream)
            cb.view(hcb.dtype).copy_(hcb, non_blocking=True)
            ev_cb.record(streams[0])
        for i in range(n_chunks):
            s_ = streams[i % len(streams)]
            cshape, wsp, wsa = ws_chunks[i]
            with torch.cuda.stream(s_):
                s_.wait_stream(stream)
                s_.wait_event(ev_cb)
                for h_, d_ in ((hK, K), (hV, V), (hQ, Q)):
                    sl(d_, i).view(h_.dtype).copy_(sl(h_, i), non_blocking=True)
                hc = (slice(None),) if along_b else (slice(bounds[i], bounds[i + 1]),)
                cbi = cb if along_b else cb[hc]
                sel_i = sl(sel, i) if nsel > 0 else None
                rc = call_precompute(bd, wl, cshape, sl(K, i), sl(V, i), cbi, sl(assign, i), sl(counts, i),
                                     sl(vsum, i), wsp, s_.cuda_stream)
                rc2 = call_attention(bd, wl, cshape, sl(Q, i), cbi, sl(counts, i), sl(vsum, i), P, scale,
                                     sl(O, i), sel_i, wsa, s_.cuda_stream)
                if rc or rc2:
                    raise RuntimeError(f"avq call failed: {rc} {rc2}")
                sl(hO, i).copy_(sl(O, i), non_blocking=True)
                if nsel > 0:
                    sl(hsel, i).copy_(sel_i, non_blocking=True)
        for s_ in streams:
            stream.wait_stream(s_)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    for _, wsp, wsa in ws_chunks:
        if bd.avq_device_status(wsp, sp) or bd.avq_device_status(wsa, sp):
            raise RuntimeError("device status error in the end-to-end run")
    barrier()
    h2d = sum(t.numel() * t.element_size() for t in (hK, hV, hQ, hcb))
    d2h = hO.numel() * hO.element_size() + (hsel.numel() * hsel.element_size() if nsel > 0 else 0)

    # max over ranks
    ms_total, e2e_ms, pre_avg, att_avg = mg.max_over_ranks(
        [ms_total, e2e_ms, statistics.mean(pre_ms), statistics.mean(att_ms)], dev)
    ms_step = ms_total / args.steps
    rows_all = wl.rows * world
    value = mg.weak_scaling_value(wl.rows, world, ms_step)

    out = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        alg = algorithmic(wl, P)
        kern = {"precompute": pre_avg, "attention": att_avg}
        dom = max(kern, key=kern.get)
        # each call is a single launch of a fraction of a millisecond, timed on
        # its own events: rated against the burst tensor peak; the sustained
        # peak is shown beside it
        rl = {k: roofline_for(k, alg[k], kern[k], peaks, sustained=False) for k in kern}
        for k in kern:
            rl[k]["frac_of_sustained_peak"] = roofline_for(k, alg[k], kern[k], peaks, sustained=True)["frac"]
        roof = dict(rl[dom])
        roof["kernel"] = dom
        roof["peak_source"] = f"{peak_src} ({'bf16_tflops (burst)' if roof['bound'] == 'tensor' else 'hbm_gbs'})"
        roof["traffic"] = stored_traffic(dom, wl.name, P)
        roof["algorithmic_per_launch"] = alg[dom]["bytes"] if roof["bound"] == "hbm" else alg[dom]["flops"]
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "B": B, "H": H, "N": N, "d": d, "M0": wl.M0,
                       "C": wl.C, "P": P, "tile": wl.tile, "scale": scale,
                       "query_rows_per_gpu": wl.rows, "l2": l2_note, **({"L": wl.L} if wl.L > 2 else {}),
                       "seed": f"{wl.seed}+rank"},
            "kernels": {k: {"ms_avg": kern[k], "ms_min": min(pre_ms if k == 'precompute' else att_ms),
                            "roofline": rl[k]} for k in kern},
            "fp64_redecided_per_call": {"parent": redecided[0], "leaf": redecided[1]},
            "roofline": roof,
            "clocks": clk,
            "e2e": {"value": rows_all / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
            "gpu_launches": int(launches),
        }
        if sweep:
            out["p_sweep"] = []
            for P_, ms_, pre_, att_ in sweep:
                a_ = algorithmic(wl, P_)
                out["p_sweep"].append({
                    "P": P_, "ms_per_step": ms_, "queries_per_s": wl.rows / (ms_ / 1e3),
                    "precompute_ms": pre_, "attention_ms": att_,
                    "attention_queries_per_s": wl.rows / (att_ / 1e3),
                    "attention_roofline": roofline_for("attention", a_["attention"], att_, peaks, sustained=False)})
    if world > 1:
        mg.barrier(dev)
        dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleSampler(wl, P)
        smp.plan(args.cpu_budget)
        n, secs = smp.run()
        out["cpu_baseline"] = {"value": n / secs, "unit": UNIT, "cores": smp.threads,
                               "kind": "oracle", "sample": smp.describe(), "seconds": secs}
    if rank == 0:
        print(json.dumps(out), flush=True)


# --------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = syn.WORKLOADS[args.workload]
    P = default_P(wl, args.P)
    smp = OracleSampler(wl, P)
    per_step = 150.0 / max(1, args.steps + args.warmup)
    smp.plan(per_step)                    # calibration and input preparation, untimed
    for _ in range(args.warmup):
        smp.run()
    times = []
    for _ in range(args.steps):
        n, dt = smp.run()
        times.append(dt)
    rows = n
    cores, desc = smp.threads, smp.describe()
    ms = 1e3 * statistics.mean(times)
    value = rows / (ms / 1e3)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "M0": wl.M0,
                   "C": wl.C, "P": P, "tile": wl.tile, "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


KERNEL_NAMES = {"precompute": ("precompute_tc_kernel", "flat_precompute_kernel", "deep_precompute_rows_kernel"),
                "attention": ("attention_tree_kernel", "flat_attention_kernel", "deep_attention_kernel")}


def ingest_ncu(csv_path: str, workload: str, P: int):
    """Record per-launch DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum)
    of each kernel from an ncu --csv capture of this workload into
    profiles/traffic.json, stamped with the current kernel-source hash."""
    import csv
    import collections
    rows = list(csv.reader(open(csv_path)))
    hdr = None
    per = collections.defaultdict(lambda: collections.defaultdict(float))
    for r in rows:
        if r and r[0] == "ID":
            hdr = r
            continue
        if hdr is None or len(r) != len(hdr):
            continue
        d = dict(zip(hdr, r))
        name, metric, val, unit = d["Kernel Name"], d["Metric Name"], d["Metric Value"], d["Metric Unit"]
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(unit, 1)
        per[(d["ID"], name)][metric] = float(val.replace(",", "")) * scale
    out = json.load(open(PROFILE_TRAFFIC)) if os.path.exists(PROFILE_TRAFFIC) else {}
    for kind, kname in KERNEL_NAMES.items():
        launches = [m for (i, n), m in per.items() if any(k in n for k in kname) and "dram__bytes_read.sum" in m]
        if not launches:
            continue
        b = [m["dram__bytes_read.sum"] + m.get("dram__bytes_write.sum", 0.0) for m in launches]
        out[f"{kind}/{workload}/P{P}"] = {
            "bytes_per_launch": sum(b) / len(b), "launches": len(b),
            "source_hash": kernel_source_hash(kind, syn.WORKLOADS[workload].L > 2), "from": os.path.basename(csv_path)}
    os.makedirs(os.path.dirname(PROFILE_TRAFFIC), exist_ok=True)
    with open(PROFILE_TRAFFIC, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
    print(json.dumps(out, indent=1))


def run_capture(args):
    """Times the top-P capture diagnostic (`avq_capture`, an exact-attention
    pass) on the workload's synthetic inputs, with the assignment and the
    selection from the forward calls; prints one JSON line of its own (not
    the benchmark line): ms per call and logits per second."""
    import torch

    from adaptive_vector_quantized_avq_b200 import binding as bd

    wl = syn.WORKLOADS[args.workload]
    P = default_P(wl, args.P)
    if wl.dtype != "bf16" or wl.C == 0 or wl.L != 2:
        raise SystemExit("capture needs a bf16 tree workload")
    dev = torch.device("cuda", 0)
    inp = syn.generate(wl)
    K, V, Q, cb = (torch.from_numpy(getattr(inp, n).view(np.int16)).to(dev).view(torch.bfloat16)
                   for n in ("K", "V", "Q", "codebook"))
    assign, counts, vsum = bd.precompute(K, V, cb, wl.M0, wl.C)
    _, sel = bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, wl.tile, wl.softmax_scale)
    shape = bd.make_shape(wl.B, wl.H, wl.N, wl.d, wl.M0, wl.C, Q.dtype)
    ws = bd.workspace(bd.avq_capture_workspace_bytes(shape, P, wl.tile), dev)
    out = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        rc = bd.avq_capture(shape, Q, K, assign, sel, P, wl.tile, wl.softmax_scale, out, ws, ws.numel(),
                            stream.cuda_stream)
        if rc:
            raise RuntimeError(f"avq_capture failed: {rc}")

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    if bd.avq_device_status(ws) != 0:
        raise RuntimeError("avq_capture device status")
    times = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = float(np.median(times))
    logits = wl.B * wl.H * wl.N * wl.N
    print(json.dumps({"metric": "top-P capture logits/s", "workload": args.workload, "P": P,
                      "ms_per_call": ms, "value": logits / (ms * 1e-3), "unit": "logits/s",
                      "mean_capture": float(out.mean()), "steps": args.steps, "warmup": args.warmup}))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(syn.WORKLOADS))
    ap.add_argument("--P", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--ingest-ncu", metavar="CSV", help="record DRAM traffic per launch from an ncu CSV")
    ap.add_argument("--capture", action="store_true",
                    help="time the top-P capture diagnostic instead (its own JSON line)")
    args = ap.parse_args(argv)
    if args.ingest_ncu:
        wl = syn.WORKLOADS[args.workload]
        P = default_P(wl, args.P)
        ingest_ncu(args.ingest_ncu, args.workload, P)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.capture:
        run_capture(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
