"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle it is given
disagrees with something the paper or the mathematics fixes:

* ``pin_brute``      -- the pure-Python per-key brute force (different algebra),
                        on random and on integer-grid inputs with exact ties;
* ``pin_p0``         -- P = 0 is flat VQ-attention over the parents, i.e. exact
                        softmax attention with every key replaced by its parent
                        codeword (paper §3.2), computed with dense numpy;
* ``pin_pmax``       -- P = M0 is VQ-attention over the tree leaf of every key;
* ``pin_exact``      -- one codeword per key reduces to exact softmax attention
                        (paper §3.1);
* ``pin_invariants`` -- count/value-sum bookkeeping and score normalisation;
* ``pin_scale``      -- the logit scale acts as a factor on Q (paper §3.1 writes
                        exp(Q K^T) with any scale folded into Q);
* ``pin_flat``       -- a flat codebook (no children) is VQ-attention with every
                        key replaced by its nearest codeword (paper §3.2), by
                        numpy argmin and dense softmax, and the brute force;
* ``pin_worked``     -- the worked example's codeword and interaction counts
                        (papernotes summary, "A Worked Example") and Table 1's
                        per-key distance count.

The mutation tests call the same functions on deliberately broken copies of
the oracle and require each copy to fail at least one pin.
"""
from __future__ import annotations

import json
import os

import numpy as np

from adaptive_vector_quantized_avq_b200 import synthetic as syn
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers
def _dense_softmax_attention(Q, Khat, V, scale):
    """Exact softmax attention (paper §3.1) for one head, numpy fp64."""
    S = scale * (Q @ Khat.T)
    S = S - S.max(axis=1, keepdims=True)
    E = np.exp(S)
    return (E @ V) / E.sum(axis=1, keepdims=True)


def _numpy_tree_assignment(K, cb, M0, C):
    """Library argmin over numpy distance matrices: nearest parent (first index
    on ties), then the strictly-closer child rule. Only used on inputs whose
    distances are far from ties or exact (integer grid)."""
    D = ((K[:, None, :] - cb[None, :, :]) ** 2).sum(axis=2)     # [N, Mtot]
    parent = np.argmin(D[:, :M0], axis=1)
    leaf = parent.copy()
    if C > 0:
        rows = np.arange(K.shape[0])
        ch = M0 + parent[:, None] * C + np.arange(C)[None, :]
        dch = D[rows[:, None], ch]
        cbest = np.argmin(dch, axis=1)
        move = dch[rows, cbest] < D[rows, parent]
        leaf = np.where(move, ch[rows, cbest], parent)
    return parent, leaf, D


def _grid_inputs(seed, N, d, M0, C, span=2):
    """Integer-valued keys, queries, values and codebook: exact fp64 arithmetic,
    so distance ties are exact and frequent."""
    rng = np.random.default_rng(seed)
    K = rng.integers(-span, span + 1, size=(1, 1, N, d)).astype(np.float64)
    Q = rng.integers(-span, span + 1, size=(1, 1, N, d)).astype(np.float64) * 0.25
    V = rng.integers(-3, 4, size=(1, 1, N, d)).astype(np.float64)
    cb = rng.integers(-span, span + 1, size=(1, M0 * (1 + C), d)).astype(np.float64)
    return K, V, Q, cb


def _close_selection(sel_a, sel_b, score, P, band=1e-12):
    """Selections agree exactly, except that parents whose score is within
    ``band`` of the P-th score may be exchanged."""
    if P == 0:
        return True
    if list(sel_a) == list(sel_b):
        return True
    kth = np.sort(score)[::-1][P - 1]
    sure = set(np.nonzero(score > kth + band)[0].tolist())
    return sure <= set(sel_a) and sure <= set(sel_b)


# -------------------------------------------------------------------- pins
BRUTE_CASES = [
    # (N, d, M0, C, T, seed)
    (1, 4, 1, 1, 16, 0),
    (17, 4, 3, 2, 16, 1),
    (100, 8, 6, 3, 64, 2),
    (256, 8, 8, 4, 64, 3),
    (130, 4, 5, 1, 32, 4),
]


def pin_brute(orc, cases=BRUTE_CASES, grid=True):
    for (N, d, M0, C, T, seed) in cases:
        wl = syn.small_workload(N=N, d=d, M0=M0, C=C, P=(0,), tile=T, seed=seed)
        inp = syn.generate(wl)
        sets = [(inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook"), wl.softmax_scale)]
        if grid:
            gK, gV, gQ, gcb = _grid_inputs(seed + 100, N, d, M0, C)
            sets.append((gK, gV, gQ, gcb, 0.5))
        for (K, V, Q, cb, scale) in sets:
            pre = orc.precompute(K, V, cb, M0, C)
            ref_parent = None
            for P in sorted({0, 1, M0 // 2, M0}):
                att = orc.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, P, T, scale)
                bf = brute.brute_force(Q[0, 0].tolist(), K[0, 0].tolist(), V[0, 0].tolist(),
                                       cb[0].tolist(), M0, C, P, T, scale)
                if ref_parent is None:
                    ref_parent = np.array(bf["parent"])
                    leaf = np.array(bf["leaf"])
                    assert np.array_equal(leaf, pre["assign"][0, 0]), "assignment differs from brute force"
                    cnt = np.zeros(M0 * (1 + C), dtype=np.int64)
                    np.add.at(cnt, ref_parent, 1)
                    moved = leaf != ref_parent
                    np.add.at(cnt, leaf[moved], 1)
                    assert np.array_equal(cnt, pre["counts"][0, 0]), "counts differ from brute force"
                sc = np.array(bf["score"])
                assert np.allclose(att["score"], sc, rtol=0, atol=1e-12), "importance differs"
                for t in range(len(bf["selected"])):
                    assert _close_selection(att["selected"][t], bf["selected"][t], sc[t], P), \
                        f"selection differs in tile {t}: {att['selected'][t]} vs {bf['selected'][t]}"
                O = att["O_full"][0, 0]
                err = np.abs(O - np.array(bf["O"])).max() if N else 0.0
                assert err <= 1e-12 * max(1.0, np.abs(O).max()), f"output differs by {err}"


def pin_p0(orc, seed=7):
    wl = syn.small_workload(N=1024, d=16, M0=16, C=4, tile=64, seed=seed, zipf_s=1.1,
                            n_components=24)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    pre = orc.precompute(K, V, cb, wl.M0, wl.C)
    parent, leaf, _ = _numpy_tree_assignment(K[0, 0], cb[0], wl.M0, wl.C)
    assert np.array_equal(leaf, pre["assign"][0, 0]), "assignment differs from numpy argmin"
    att = orc.attention(Q, cb, pre["counts"], pre["vsum"], wl.M0, wl.C, 0, wl.tile, wl.softmax_scale)
    ref = _dense_softmax_attention(Q[0, 0], cb[0][parent], V[0, 0], wl.softmax_scale)
    err = np.abs(att["O_full"][0, 0] - ref).max()
    assert err < 1e-10, f"P=0 differs from flat VQ attention by {err}"


def pin_pmax(orc, seed=8):
    wl = syn.small_workload(N=1024, d=16, M0=16, C=4, tile=128, seed=seed)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    pre = orc.precompute(K, V, cb, wl.M0, wl.C)
    parent, leaf, _ = _numpy_tree_assignment(K[0, 0], cb[0], wl.M0, wl.C)
    assert np.array_equal(leaf, pre["assign"][0, 0])
    att = orc.attention(Q, cb, pre["counts"], pre["vsum"], wl.M0, wl.C, wl.M0, wl.tile,
                        wl.softmax_scale)
    ref = _dense_softmax_attention(Q[0, 0], cb[0][leaf], V[0, 0], wl.softmax_scale)
    err = np.abs(att["O_full"][0, 0] - ref).max()
    assert err < 1e-10, f"P=M0 differs from full-tree VQ attention by {err}"
    for t in range(att["selected"].shape[0]):
        assert sorted(att["selected"][t].tolist()) == list(range(wl.M0))


def pin_exact(orc, seed=9, N=192, d=8, C=2, T=64):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((1, 1, N, d))
    Q = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    M0 = N
    cb = np.empty((1, M0 * (1 + C), d))
    cb[0, :M0] = K[0, 0]
    cb[0, M0:] = np.repeat(K[0, 0], C, axis=0)          # children = copies: constraint holds
    pre = orc.precompute(K, V, cb, M0, C)
    assert np.array_equal(pre["assign"][0, 0], np.arange(N)), "a key left its own codeword"
    ref = _dense_softmax_attention(Q[0, 0], K[0, 0], V[0, 0], 0.75)
    for P in (0, 3, M0):
        att = orc.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, P, T, 0.75)
        err = np.abs(att["O_full"][0, 0] - ref).max()
        assert err < 1e-10, f"one codeword per key differs from exact attention by {err} (P={P})"


def pin_invariants(orc, seed=10):
    wl = syn.small_workload(N=2000, d=16, M0=12, C=4, tile=64, seed=seed, zipf_s=1.1,
                            n_components=20, B=2, H=2)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    M0, C = wl.M0, wl.C
    pre = orc.precompute(K, V, cb, M0, C)
    cnt, vs, asg = pre["counts"], pre["vsum"], pre["assign"]
    assert pre["dist_evals"] == wl.rows * (M0 + C)
    for b in range(wl.B):
        for h in range(wl.H):
            n = cnt[b, h]
            assert n[:M0].sum() == wl.N
            child = n[M0:].reshape(M0, C)
            assert np.all(child.sum(axis=1) <= n[:M0])
            for p in range(M0):
                stay = V[b, h][asg[b, h] == p].sum(axis=0)
                kids = vs[b, h, M0 + p * C: M0 + (p + 1) * C].sum(axis=0)
                assert np.allclose(vs[b, h, p], stay + kids, rtol=0, atol=1e-9)
                assert n[p] - child[p].sum() == int((asg[b, h] == p).sum())
    prev = None
    for P in range(0, M0 + 1):
        att = orc.attention(Q, cb, cnt, vs, M0, C, P, wl.tile, wl.softmax_scale)
        assert np.allclose(att["score"].sum(axis=1), 1.0, atol=1e-12)
        if prev is not None:
            for t in range(att["selected"].shape[0]):
                assert set(prev[t].tolist()) <= set(att["selected"][t].tolist()), "selection does not nest"
        prev = att["selected"]


def pin_scale(orc, seed=11):
    wl = syn.small_workload(N=300, d=8, M0=8, C=3, tile=64, seed=seed)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    pre = orc.precompute(K, V, cb, wl.M0, wl.C)
    for P in (0, 3):
        a = orc.attention(Q, cb, pre["counts"], pre["vsum"], wl.M0, wl.C, P, wl.tile, 0.125)
        b = orc.attention(Q * 0.125, cb, pre["counts"], pre["vsum"], wl.M0, wl.C, P, wl.tile, 1.0)
        assert np.array_equal(a["selected"], b["selected"])
        assert np.abs(a["O"] - b["O"]).max() < 1e-12


def pin_flat(orc, seed=13):
    wl = syn.small_workload(N=700, d=16, M0=40, C=0, tile=128, seed=seed, zipf_s=1.1,
                            n_components=48)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    assert cb.shape[1] == wl.M0
    pre = orc.precompute(K, V, cb, wl.M0, 0)
    nearest, _, _ = _numpy_tree_assignment(K[0, 0], cb[0], wl.M0, 0)
    assert np.array_equal(nearest, pre["assign"][0, 0]), "flat assignment differs from numpy argmin"
    assert np.array_equal(np.bincount(nearest, minlength=wl.M0), pre["counts"][0, 0])
    att = orc.attention(Q, cb, pre["counts"], pre["vsum"], wl.M0, 0, 0, wl.tile, wl.softmax_scale)
    ref = _dense_softmax_attention(Q[0, 0], cb[0][nearest], V[0, 0], wl.softmax_scale)
    err = np.abs(att["O_full"][0, 0] - ref).max()
    assert err < 1e-10, f"flat codebook differs from VQ attention by {err}"
    pin_brute(orc, cases=[(90, 8, 7, 0, 32, seed), (1, 4, 1, 0, 16, seed + 1)])


def pin_worked(orc):
    with open(os.path.join(GOLDEN, "worked_example_64_16_8.json")) as f:
        g = json.load(f)
    wl = syn.small_workload(N=256, d=8, M0=g["M0"], C=g["C"], tile=128, seed=12,
                            n_components=g["M0"])
    inp = syn.generate(wl)
    cb = inp.f64("codebook")
    assert cb.shape[1] == g["stored_codewords"]
    pre = orc.precompute(inp.f64("K"), inp.f64("V"), cb, g["M0"], g["C"])
    assert pre["dist_evals"] == wl.N * g["distance_evaluations_per_key"]
    att = orc.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], g["M0"], g["C"], g["P"],
                        wl.tile, wl.softmax_scale)
    assert att["logit_evals"] == wl.N * g["interactions_per_query"]
    assert att["selected"].shape[1] * g["C"] == g["children_per_tile"]


ALL_PINS = [pin_brute, pin_p0, pin_pmax, pin_exact, pin_invariants, pin_scale, pin_flat, pin_worked]
