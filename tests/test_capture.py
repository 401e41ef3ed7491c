"""Top-P capture (paper §5.2 "Elastic Inference", Table 6; Figure 7): the
oracle's definition pinned on CPU, the C-ABI argument checks, and the GPU
kernel against the oracle (marked gpu)."""
import math

import numpy as np
import pytest

from adaptive_vector_quantized_avq_b200 import synthetic as syn
from oracle import oracle as orc


def _tree_case(seed, N=37, d=4, M0=5, C=2, tile=16, P=2, B=1, H=1):
    wl = syn.small_workload(B=B, H=H, N=N, d=d, M0=M0, C=C, tile=tile, seed=seed, n_components=M0)
    inp = syn.generate(wl)
    return wl, inp


def _brute_capture(Q, K, cb, M0, sel, tile, scale):
    """Pure-Python loops for one head: each key's parent by its own nearest-
    parent search (squared distances, first index on ties), true softmax
    weights with math.exp, and the weight on keys of the tile's parents."""
    N, d = len(K), len(K[0])
    parent = []
    for k in K:
        best, arg = math.inf, -1
        for p in range(M0):
            dist = sum((k[j] - cb[p][j]) ** 2 for j in range(d))
            if dist < best:
                best, arg = dist, p
        parent.append(arg)
    out = []
    for i, q in enumerate(Q):
        s = [scale * sum(q[j] * k[j] for j in range(d)) for k in K]
        mx = max(s)
        w = [math.exp(v - mx) for v in s]
        chosen = set(sel[i // tile])
        out.append(sum(wk for wk, pk in zip(w, parent) if pk in chosen) / sum(w))
    return out


def test_capture_matches_brute_force(oracle):
    """Children take some keys, so the leaf -> parent mapping is exercised."""
    for seed in (31, 32):
        wl, inp = _tree_case(seed)
        Q, K, V, cb = inp.f64("Q"), inp.f64("K"), inp.f64("V"), inp.f64("codebook")
        pre = oracle.precompute(K, V, cb, wl.M0, wl.C)
        assert (pre["assign"] >= wl.M0).any(), "no key on a child: the case does not test the mapping"
        att = oracle.attention(Q, cb, pre["counts"], pre["vsum"], wl.M0, wl.C, 2, wl.tile, wl.softmax_scale)
        sel = att["selected"].reshape(1, 1, -1, 2)
        got = orc.capture(Q, K, pre["assign"], sel, wl.M0, wl.C, wl.tile, wl.softmax_scale)
        ref = _brute_capture(Q[0, 0].tolist(), K[0, 0].tolist(), cb[0].tolist(), wl.M0,
                             sel[0, 0].tolist(), wl.tile, wl.softmax_scale)
        np.testing.assert_allclose(got[0, 0], ref, rtol=0, atol=1e-12)


def test_capture_all_and_no_parents(oracle):
    """Every parent selected: all the weight is captured; none: nothing."""
    wl, inp = _tree_case(33, N=200, d=8, M0=6, C=3, tile=64, B=2, H=2)
    Q, K, V, cb = inp.f64("Q"), inp.f64("K"), inp.f64("V"), inp.f64("codebook")
    pre = oracle.precompute(K, V, cb, wl.M0, wl.C)
    nt = wl.ntiles
    full = np.broadcast_to(np.arange(wl.M0, dtype=np.int32), (2, 2, nt, wl.M0)).copy()
    np.testing.assert_allclose(orc.capture(Q, K, pre["assign"], full, wl.M0, wl.C, wl.tile, 0.3), 1.0,
                               rtol=0, atol=1e-12)
    none = np.zeros((2, 2, nt, 0), np.int32)
    assert np.all(orc.capture(Q, K, pre["assign"], none, wl.M0, wl.C, wl.tile, 0.3) == 0.0)


def test_capture_uniform_keys_closed_form(oracle):
    """Identical keys make the true attention uniform, so the capture is the
    share of keys whose parent is selected."""
    rng = np.random.default_rng(34)
    N, d, M0, C, T = 150, 8, 4, 2, 64
    K = np.tile(rng.standard_normal(d), (1, 1, N, 1))
    Q = rng.standard_normal((1, 1, N, d))
    assign = rng.integers(0, M0 * (1 + C), size=(1, 1, N)).astype(np.int32)
    sel = np.array([[[[0, 3], [1, 2], [3, 1]]]], dtype=np.int32)          # ceil(150/64) = 3 tiles
    parent = np.where(assign < M0, assign, (assign - M0) // C)[0, 0]
    got = orc.capture(Q, K, assign, sel, M0, C, T, 1.0)[0, 0]
    for i in range(N):
        want = np.isin(parent, sel[0, 0, i // T]).mean()
        assert abs(got[i] - want) < 1e-12


def test_capture_additive_over_disjoint_selections(oracle):
    """Capture is linear in the set of parents: disjoint sets add up, and a
    parent repeated in the list counts once."""
    wl, inp = _tree_case(35, N=300, d=8, M0=8, C=2, tile=128)
    Q, K, V, cb = inp.f64("Q"), inp.f64("K"), inp.f64("V"), inp.f64("codebook")
    pre = oracle.precompute(K, V, cb, wl.M0, wl.C)
    nt = wl.ntiles
    a = np.tile(np.array([0, 5, 2], np.int32), (1, 1, nt, 1))
    b = np.tile(np.array([7, 1], np.int32), (1, 1, nt, 1))
    ab = np.concatenate([a, b], axis=3)
    args = (pre["assign"], )
    ca = orc.capture(Q, K, *args, a, wl.M0, wl.C, wl.tile, 0.5)
    cb_ = orc.capture(Q, K, *args, b, wl.M0, wl.C, wl.tile, 0.5)
    cab = orc.capture(Q, K, *args, ab, wl.M0, wl.C, wl.tile, 0.5)
    np.testing.assert_allclose(cab, ca + cb_, rtol=0, atol=1e-12)
    rep = np.concatenate([a, a[..., :1]], axis=3)
    np.testing.assert_array_equal(orc.capture(Q, K, *args, rep, wl.M0, wl.C, wl.tile, 0.5), ca)
