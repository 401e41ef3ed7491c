"""Depth-L trees on the GPU (avq_precompute_deep / avq_attention_deep)
against the fp64 depth-L oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

from adaptive_vector_quantized_avq_b200 import binding as bd
from adaptive_vector_quantized_avq_b200 import synthetic as syn

import parity
from test_deep_oracle import _deep_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib_built():
    from adaptive_vector_quantized_avq_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return True


def _storage(a, dtype):
    bits = syn.to_storage(np.asarray(a, dtype=np.float64), dtype)
    return bits, syn.storage_to_f64(bits, dtype)


def _run(name, Q, K, V, cb, M0, C, L, Ps, T, scale, dtype):
    (Qs, Qf), (Ks, Kf), (Vs, Vf), (cbs, cbf) = (_storage(x, dtype) for x in (Q, K, V, cb))
    dev = lambda a: parity.to_device(a, dtype)
    tQ, tK, tV, tcb = dev(Qs), dev(Ks), dev(Vs), dev(cbs)
    assign, counts, vsum = bd.precompute_deep(tK, tV, tcb, M0, C, L)
    O, sel = bd.attention_deep(tQ, tcb, counts, vsum, M0, C, L, Ps, T, scale)
    torch.cuda.synchronize()
    return parity.check_deep(name, dtype, assign.cpu().numpy(), counts.cpu().numpy(), vsum.cpu().numpy(),
                             parity.from_device(O), sel.cpu().numpy(), Qf, Kf, Vf, cbf, M0, C, L, list(Ps), T,
                             scale)


# name, (M0, C, L, N, d), Ps, T, dtype, B, H, seed
TREE_CASES = [
    ("L3-d64", (16, 4, 3, 1500, 64), (4, 8), 128, "bf16", 1, 2, 2),
    ("L3-ragged", (8, 4, 3, 700, 64), (2, 4), 128, "bf16", 2, 1, 1),
    ("L4", (4, 2, 4, 500, 64), (2, 2, 2), 128, "bf16", 1, 2, 3),
    ("L3-d128", (32, 8, 3, 4096, 128), (8, 16), 128, "bf16", 1, 2, 4),
    ("L3-f32-tile64", (8, 4, 3, 700, 64), (2, 4), 64, "f32", 1, 2, 5),
    ("L3-f32-tile128", (16, 4, 3, 900, 64), (4, 8), 128, "f32", 1, 2, 10),
    ("L3-all", (8, 4, 3, 600, 64), (8, 32), 128, "bf16", 1, 1, 6),
    ("L3-none", (8, 4, 3, 600, 64), (0, 0), 128, "bf16", 1, 1, 7),
    ("L2", (16, 4, 2, 900, 64), (5,), 64, "bf16", 1, 2, 8),
    ("L3-C1", (32, 1, 3, 800, 64), (12, 7), 128, "bf16", 1, 1, 9),
]


@pytest.mark.parametrize("name,dims,Ps,T,dtype,B,H,seed", TREE_CASES, ids=[c[0] for c in TREE_CASES])
def test_deep_tree_parity(lib_built, name, dims, Ps, T, dtype, B, H, seed):
    M0, C, L, N, d = dims
    Q, K, V, cb = _deep_inputs(seed, N, d, M0, C, L, H=H, B=B)
    rep = _run(name, Q, K, V, cb, M0, C, L, Ps, T, 0.125, dtype)
    if C > 1:
        assert rep["max_depth"] == L - 1, "no key reached the deepest level"
    print(name, dict(rep))


@pytest.mark.parametrize("name", ["deep3-small", "deep3-16k"])
def test_deep_synthetic_workloads(lib_built, name):
    """The seeded synthetic depth-3 workloads (mixture keys and queries, a
    codebook whose every node is the exact mean of its children)."""
    wl = syn.WORKLOADS[name] if name in syn.WORKLOADS else syn.small_workload(
        B=1, H=2, N=1000, d=64, M0=32, C=4, L=3, P=((4, 8),), tile=128, dtype="bf16", seed=41, n_components=40)
    inp = syn.generate(wl)
    Ps = wl.P[0]
    rep = _run(wl.name, inp.f64("Q"), inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C, wl.L, Ps,
               wl.tile, wl.softmax_scale, wl.dtype)
    print(name, dict(rep))


def test_deep_rescale_far_child(lib_built):
    """A grandchild whose logit lies far above every level-0 logit of the
    queries (about 90 octaves): the row's shift moves up and the output is
    still the oracle's (no overflow)."""
    M0, C, L, N, d = 4, 2, 3, 256, 64
    rng = np.random.default_rng(13)
    grid = 1.0 / 32
    lv0 = np.round(rng.standard_normal((1, M0, d)) * 0.1 / grid) * grid
    lv0[0, 0] = 0.25                      # node 0 a little out: the nearest for the far keys
    lv1 = np.repeat(lv0, C, axis=1)
    lv1[0, 0] = 1.5                       # its child 0 further out
    lv2 = np.repeat(lv1, C, axis=1)
    lv2[0, 0] = 3.0                       # and that child's child 0 far out
    cb = np.concatenate([lv0, lv1, lv2], axis=1)
    K = np.round(rng.standard_normal((1, 1, N, d)) * 0.1 / grid) * grid
    K[0, 0, 0] = 3.0
    K[0, 0, 1] = 1.5
    Q = np.full((1, 1, N, d), 1.0)
    V = rng.standard_normal((1, 1, N, d))
    rep = _run("rescale", Q, K, V, cb, M0, C, L, (M0, M0 * C), 128, 1.0, "bf16")
    print(dict(rep))
