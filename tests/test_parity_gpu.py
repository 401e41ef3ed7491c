"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
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
]


@pytest.fixture(scope="module")
def lib_built():
    from adaptive_vector_quantized_avq_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return True


def _run_case(wl, Ps, oracle, tile_ids_fn=None):
    inp = syn.generate(wl)
    gpu = parity.run_gpu(wl, inp, Ps)
    ora = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)
    reports = {"precompute": parity.check_precompute(wl, inp, gpu, ora, oracle)}
    for P in Ps:
        O, sel = gpu["att"][P]
        ids = tile_ids_fn(wl) if tile_ids_fn else None
        reports[P] = parity.check_attention(wl, inp, P, O, sel, ora["counts"], ora["vsum"], oracle,
                                            tile_ids=ids)
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


def _sample_tiles(wl, n=24, seed=0):
    total = wl.B * wl.H * wl.ntiles
    rng = np.random.default_rng(seed)
    ids = set(rng.choice(total, size=min(n, total), replace=False).tolist())
    ids |= {0, total - 1}
    return np.array(sorted(ids))


@pytest.mark.parametrize("name", ["tiny-fp32", "vit-b", "long-16k", "max-64k", "refine-d128"])
def test_full_size_parity(lib_built, oracle, name):
    """The five workloads at full size: assignments/counts/value sums compared
    everywhere, attention on a sample of tiles (plus the first and last)."""
    wl = syn.WORKLOADS[name]
    rep = _run_case(wl, wl.P, oracle, tile_ids_fn=_sample_tiles)
    print(name, rep)
