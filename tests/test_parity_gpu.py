"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
import json
import os

import numpy as np
import pytest
import torch

from adaptive_vector_quantized_avq_b200 import synthetic as syn

import parity

pytestmark = pytest.mark.gpu

SMALL = [
    # name, workload, P values
    ("tiny-fp32", syn.WORKLOADS["tiny-fp32"], (0, 4, 16)),
    ("bf16-ragged", syn.small_workload(B=2, H=3, N=1000, d=64, M0=64, C=4, tile=128, dtype="bf16",
                                       seed=3, n_components=64), (0, 8, 64)),
    ("bf16-d128", syn.small_workload(B=1, H=2, N=700, d=128, M0=32, C=8, tile=128, dtype="bf16",
                                     seed=4, n_components=40), (0, 4, 32)),
    ("bf16-tile64", syn.small_workload(B=1, H=2, N=333, d=64, M0=128, C=8, tile=64, dtype="bf16",
                                       seed=5, n_components=160, zipf_s=1.1), (16, 128)),
    ("bf16-sparse-parents", syn.small_workload(B=1, H=2, N=500, d=64, M0=128, C=2, tile=128,
                                               dtype="bf16", seed=6, n_components=128,
                                               zipf_s=1.1), (0, 5, 128)),
    ("f32-d128", syn.small_workload(B=2, H=1, N=300, d=128, M0=16, C=3, tile=64, dtype="f32",
                                    seed=7, n_components=16), (0, 3, 16)),
    ("bf16-scale1", syn.small_workload(B=1, H=1, N=512, d=64, M0=16, C=4, tile=128, dtype="bf16",
                                       seed=8, n_components=16, scale=1.0), (0, 4)),
    ("one-key", syn.small_workload(B=1, H=1, N=1, d=64, M0=4, C=2, tile=64, dtype="bf16",
                                   seed=9, n_components=4), (0, 1, 4)),
    ("one-parent", syn.small_workload(B=1, H=2, N=300, d=64, M0=1, C=1, tile=128, dtype="bf16",
                                      seed=10, n_components=1), (0, 1)),
    # flat codebooks (C = 0): nearest codeword among up to 512, attention with P = 0
    ("flat-256", syn.small_workload(B=1, H=2, N=1000, d=64, M0=256, C=0, tile=128, dtype="bf16",
                                    seed=13, n_components=300), (0,)),
    ("flat-100-ragged", syn.small_workload(B=2, H=1, N=333, d=64, M0=100, C=0, tile=128,
                                           dtype="bf16", seed=14, n_components=100, zipf_s=1.1), (0,)),
    ("flat-512", syn.small_workload(B=1, H=2, N=1500, d=64, M0=512, C=0, tile=128, dtype="bf16",
                                    seed=15, n_components=600), (0,)),
    ("flat-3", syn.small_workload(B=1, H=1, N=200, d=64, M0=3, C=0, tile=128, dtype="bf16",
                                  seed=16, n_components=3), (0,)),
    # head dim 128 (two 64-column blocks per row, 128 output columns in TMEM)
    ("flat-d128-512", syn.small_workload(B=1, H=2, N=700, d=128, M0=512, C=0, tile=128,
                                         dtype="bf16", seed=17, n_components=600), (0,)),
    ("flat-d128-200", syn.small_workload(B=2, H=1, N=257, d=128, M0=200, C=0, tile=128,
                                         dtype="bf16", seed=18, n_components=200), (0,)),
    # dispatch paths: a bf16 tree whose codebook image does not fit the
    # tensor-core precompute's shared memory runs the CUDA-core precompute
    # (d = 64 with M0 = 128, C = 16; d = 128 with M0 = 128, C = 8); C = 16 on
    # both tensor-core kernels; a bf16 C outside {1, 2, 4, 8, 16} runs the
    # CUDA-core attention
    ("bf16-simt-pre-c16", syn.small_workload(B=1, H=2, N=1100, d=64, M0=128, C=16, tile=128,
                                             dtype="bf16", seed=19, n_components=160,
                                             zipf_s=1.1), (0, 3, 8, 128)),
    ("bf16-simt-pre-d128", syn.small_workload(B=1, H=2, N=900, d=128, M0=128, C=8, tile=128,
                                              dtype="bf16", seed=20, n_components=140), (0, 16, 128)),
    ("bf16-tc-c16", syn.small_workload(B=2, H=1, N=650, d=64, M0=32, C=16, tile=128, dtype="bf16",
                                       seed=21, n_components=40), (0, 5, 32)),
    ("bf16-tc-c16-d128", syn.small_workload(B=1, H=2, N=400, d=128, M0=16, C=16, tile=128,
                                            dtype="bf16", seed=22, n_components=20), (0, 7, 16)),
    ("bf16-c3", syn.small_workload(B=1, H=2, N=530, d=64, M0=24, C=3, tile=128, dtype="bf16",
                                   seed=23, n_components=30), (0, 5, 24)),
]


@pytest.fixture(scope="module")
def lib_built():
    from adaptive_vector_quantized_avq_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return True


def _run_case(wl, Ps, oracle):
    inp = syn.generate(wl)
    gpu = parity.run_gpu(wl, inp, Ps)
    ora = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)
    reports = {"precompute": parity.check_precompute(wl, inp, gpu, ora, oracle)}
    for P in Ps:
        O, sel = gpu["att"][P]
        reports[P] = parity.check_attention(wl, inp, P, O, sel, ora["counts"], ora["vsum"], oracle)
    return reports


@pytest.mark.parametrize("name,wl,Ps", SMALL, ids=[c[0] for c in SMALL])
def test_small_parity(lib_built, oracle, name, wl, Ps):
    rep = _run_case(wl, Ps, oracle)
    print(name, rep)


def test_empty_sequence(lib_built):
    from adaptive_vector_quantized_avq_b200 import binding as bd
    K = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    cb = torch.zeros(2, 16 * 5, 64, dtype=torch.bfloat16, device="cuda")
    a, c, v = bd.precompute(K, K, cb, 16, 4)
    assert a.numel() == 0 and int(c.abs().sum()) == 0 and float(v.abs().sum()) == 0.0
    O, sel = bd.attention(K, cb, c, v, 16, 4, 4, 128)
    assert O.numel() == 0 and sel.numel() == 0


def _record(name, rep):
    """Append a workload's parity figures to the JSON file named by
    AVQ_PARITY_RECORD (when set): per P the O max-abs error, the tiles
    compared and the tie-band tiles, plus the precompute's value-sum error
    and fp64 re-decision counts."""
    path = os.environ.get("AVQ_PARITY_RECORD")
    if not path:
        return
    data = json.load(open(path)) if os.path.exists(path) else {}
    data[name] = {str(k): dict(v) for k, v in rep.items()}
    with open(path, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)


@pytest.mark.parametrize("name", ["tiny-fp32", "vit-b", "long-16k", "max-64k", "refine-d128", "flat-512"])
def test_full_size_parity(lib_built, oracle, name):
    """The workloads at full size, in the launch configuration the benchmark
    times: assignments, counts and value sums compared everywhere, and every
    query tile's selection and output compared with the oracle's."""
    wl = syn.WORKLOADS[name]
    rep = _run_case(wl, wl.P, oracle)
    for P in wl.P:
        assert rep[P]["tiles"] == wl.B * wl.H * wl.ntiles
    _record(name, rep)
    print(name, rep)


def test_duplicate_parents_exact_ties(lib_built, oracle):
    """Parents 0 and 1 (and their children) are the same codewords, so every
    key of that cluster is an exact parent tie that no fp32 bound separates:
    the keys go through the exact fp64 decision, which must keep the lower
    index (paper §4.2 argmin; ties to the lowest index)."""
    wl = syn.small_workload(B=1, H=2, N=900, d=64, M0=16, C=4, tile=128, dtype="bf16", seed=11,
                            n_components=16)
    inp = syn.generate(wl)
    cb = inp.codebook.copy()
    for h in range(wl.H):
        cb[h, 1] = cb[h, 0]
        cb[h, wl.M0 + wl.C:wl.M0 + 2 * wl.C] = cb[h, wl.M0:wl.M0 + wl.C]
    inp = syn.Inputs(wl, inp.K, inp.V, inp.Q, cb)
    gpu = parity.run_gpu(wl, inp, (0, 4))
    ora = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)
    rep = parity.check_precompute(wl, inp, gpu, ora, oracle)
    # every key of the duplicated cluster was re-decided, and none landed on parent 1's subtree
    assert gpu["redecided"][0] > 0
    sub1 = (gpu["assign"] == 1) | ((gpu["assign"] >= wl.M0 + wl.C) & (gpu["assign"] < wl.M0 + 2 * wl.C))
    assert not sub1.any()
    for P in (0, 4):
        O, sel = gpu["att"][P]
        parity.check_attention(wl, inp, P, O, sel, ora["counts"], ora["vsum"], oracle)
    print(rep)


def test_far_child_moves_the_shift(lib_built, oracle):
    """A non-empty child whose logit lies about 127 octaves above every parent
    logit of the queries: the row's shift moves up (the running accumulators
    are rescaled by an exact power of two, paper §4.3) and the output and
    selection are still the oracle's, with no overflow and no device error."""
    d, M0, C, N = 64, 16, 2, 256
    rng = np.random.default_rng(12)
    grid = 1.0 / 32
    par = np.round(rng.standard_normal((M0, d)) * 0.1 / grid) * grid   # parents near 0 ...
    par[0] = 0.25                                                       # ... parent 0 a little out
    ch = np.repeat(par, C, axis=0).copy()
    ch[0] = 3.0                                                         # child 0 of parent 0: far out
    cb = np.concatenate([par, ch])[None]                                # [1, Mtot, d]
    K = np.round(rng.standard_normal((1, 1, N, d)) * 0.1 / grid) * grid
    K[0, 0, 0] = 3.0                                                    # a key on the far child
    V = rng.standard_normal((1, 1, N, d))
    # q . child0 = 96 against q . parent0 = 8 (scale 1): ~127 octaves above the shift
    Q = np.full((1, 1, N, d), 0.5)
    wl = syn.small_workload(B=1, H=1, N=N, d=d, M0=M0, C=C, tile=128, dtype="bf16", P=(M0, 3),
                            scale=1.0)
    store = lambda a: syn.f64_to_bf16_bits(a)
    inp = syn.Inputs(wl, store(K), store(V), store(Q), store(cb))
    gpu = parity.run_gpu(wl, inp, wl.P)   # asserts a clean device status
    assert int(gpu["assign"][0, 0, 0]) == M0   # the far key sits on child 0 of parent 0
    ora = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), M0, C)
    parity.check_precompute(wl, inp, gpu, ora, oracle)
    for P in wl.P:
        O, sel = gpu["att"][P]
        rep = parity.check_attention(wl, inp, P, O, sel, ora["counts"], ora["vsum"], oracle)
        print(P, dict(rep))


def test_timeout_status_and_recovery(lib_built, oracle):
    """The failure path of a bounded wait, without a GPU fault: the test hook
    gives the attention kernel's first hand-over wait a limit of zero. The call
    reports AVQ_ETIMEOUT through the device status (every CTA stopped, drained
    its loads and contractions and freed its tensor memory), and the next call
    on the same context is correct and clean."""
    from adaptive_vector_quantized_avq_b200 import binding as bd
    wl = syn.small_workload(B=1, H=2, N=700, d=64, M0=32, C=4, tile=128, dtype="bf16", seed=24,
                            n_components=40, P=(6,))
    inp = syn.generate(wl)
    K, V, Q, cb = (parity.to_device(getattr(inp, n), wl.dtype) for n in ("K", "V", "Q", "codebook"))
    _, counts, vsum = bd.precompute(K, V, cb, wl.M0, wl.C)
    shape = bd.make_shape(wl.B, wl.H, wl.N, wl.d, wl.M0, wl.C, Q.dtype)
    ws = bd.workspace(bd.avq_attention_workspace_bytes(shape, 6, 128), Q.device)
    assert bd.avq_test_fail_next_wait() == 0
    bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, 6, 128, wl.softmax_scale, ws=ws)
    assert bd.avq_device_status(ws) == -4          # AVQ_ETIMEOUT
    O, sel = bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, 6, 128, wl.softmax_scale, ws=ws)
    assert bd.avq_device_status(ws) == 0
    ora = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)
    parity.check_attention(wl, inp, 6, parity.from_device(O), sel.cpu().numpy(), ora["counts"], ora["vsum"],
                           oracle)
