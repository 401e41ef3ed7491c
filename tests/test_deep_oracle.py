"""Deeper hierarchies (AVQ-Attention §6 proposes them; the readings taken
are stated in ``oracle/deep.py``): that numpy fp64 reference pinned on CPU
against the two-level C oracle, a per-key brute force, and the exact
special cases."""
import numpy as np
import pytest

from adaptive_vector_quantized_avq_b200 import synthetic as syn
from oracle import brute
from oracle import deep


def _deep_inputs(seed, N, d, M0, C, L, spread=(2.0, 0.6, 0.25, 0.1), key_sigma=0.15, H=1, B=1):
    """A depth-L codebook whose levels tighten around their parents, and keys
    drawn around random deepest nodes, so that descents of every depth occur."""
    rng = np.random.default_rng(seed)
    levels = [rng.standard_normal((H, M0, d)) * spread[0]]
    for l in range(1, L):
        par = np.repeat(levels[-1], C, axis=1)
        levels.append(par + rng.standard_normal(par.shape) * spread[min(l, len(spread) - 1)])
    cb = np.concatenate(levels, axis=1)
    deepest = levels[-1]
    pick = rng.integers(0, deepest.shape[1], size=(B, H, N))
    K = np.stack([np.stack([deepest[h][pick[b, h]] for h in range(H)]) for b in range(B)])
    K = K + rng.standard_normal(K.shape) * key_sigma
    Q = rng.standard_normal((B, H, N, d)) * 0.7
    V = rng.standard_normal((B, H, N, d))
    return Q, K, V, cb


def _sel_close(a, b, score, band=1e-12):
    """Equal selections, except for candidates within `band` of the cut."""
    if list(a) == list(b):
        return True
    vals = sorted(score.values(), reverse=True)
    kth = vals[len(a) - 1]
    sure = {c for c, v in score.items() if v > kth + band}
    return sure <= set(a) and sure <= set(b)


@pytest.mark.parametrize("grid", [False, True])
def test_two_levels_reproduce_the_tree_oracle(oracle, grid):
    """L = 2 is the two-level method: the same assignment and statistics as the
    (pinned) C oracle, the same selections and outputs."""
    wl = syn.small_workload(B=1, H=2, N=300, d=8, M0=6, C=3, tile=64, seed=51, n_components=6)
    inp = syn.generate(wl)
    K, V, Q, cb = inp.f64("K"), inp.f64("V"), inp.f64("Q"), inp.f64("codebook")
    if grid:
        rng = np.random.default_rng(52)
        K = rng.integers(-2, 3, size=K.shape).astype(np.float64)
        cb = rng.integers(-2, 3, size=cb.shape).astype(np.float64)
    a = oracle.precompute(K, V, cb, wl.M0, wl.C)
    b = deep.precompute(K, V, cb, wl.M0, wl.C, 2)
    np.testing.assert_array_equal(b["assign"], a["assign"])
    np.testing.assert_array_equal(b["counts"], a["counts"])
    np.testing.assert_allclose(b["vsum"], a["vsum"], rtol=0, atol=1e-12)
    for P in (0, 2, wl.M0):
        ta = oracle.attention(Q, cb, a["counts"], a["vsum"], wl.M0, wl.C, P, wl.tile, 0.5)
        tb = deep.attention(Q, cb, a["counts"], a["vsum"], wl.M0, wl.C, 2, P, wl.tile, 0.5)
        for j in range(ta["selected"].shape[0]):
            score = {p: s for p, s in enumerate(ta["score"][j])}
            assert _sel_close(tb["selected"][j][0], ta["selected"][j], score)
            np.testing.assert_allclose(tb["score"][j][0], ta["score"][j], rtol=0, atol=1e-13)
        np.testing.assert_allclose(tb["O_full"], ta["O_full"], rtol=0, atol=1e-11)


@pytest.mark.parametrize("L,Ps", [(3, (1, 2)), (3, (2, 1)), (3, (3, 6)), (4, (1, 2, 2))])
def test_deep_matches_per_key_brute_force(L, Ps):
    M0, C, d, N, T = 3, 2, 4, 48, 16
    Q, K, V, cb = _deep_inputs(60 + L + Ps[0], N, d, M0, C, L)
    pre = deep.precompute(K, V, cb, M0, C, L)
    bf = brute.brute_force_deep(Q[0, 0].tolist(), K[0, 0].tolist(), V[0, 0].tolist(), cb[0].tolist(),
                                M0, C, L, list(Ps), T, 0.8)
    np.testing.assert_array_equal(pre["assign"][0, 0], [p[-1] for p in bf["paths"]])
    np.testing.assert_array_equal(pre["depth"][0, 0], [len(p) - 1 for p in bf["paths"]])
    assert pre["depth"].max() == L - 1, "no key reached the deepest level: the case tests too little"
    att = deep.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, L, Ps, T, 0.8)
    for t in range(len(bf["selected"])):
        for l in range(L - 1):
            sc = bf["score"][t][l]
            got = dict(zip(att["candidates"][t][l].tolist(), att["score"][t][l].tolist()))
            assert set(got) == set(sc), f"tile {t} level {l}: candidates differ"
            for c in sc:
                assert abs(got[c] - sc[c]) < 1e-12
            assert _sel_close(att["selected"][t][l].tolist(), bf["selected"][t][l], sc)
    np.testing.assert_allclose(att["O_full"][0, 0], np.array(bf["O"]), rtol=0, atol=1e-12)


def _dense(Q, Khat, V, scale):
    S = scale * (Q @ Khat.T)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    return (E @ V) / E.sum(axis=1, keepdims=True)


def test_full_expansion_is_vq_attention_over_the_leaves():
    """Expanding every candidate at every level represents each key by its
    leaf: exact softmax attention over the keys replaced by their leaves."""
    M0, C, L, d, N, T = 4, 3, 3, 6, 200, 64
    Q, K, V, cb = _deep_inputs(71, N, d, M0, C, L)
    pre = deep.precompute(K, V, cb, M0, C, L)
    att = deep.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, L, (M0, M0 * C), T, 0.6)
    ref = _dense(Q[0, 0], cb[0][pre["assign"][0, 0]], V[0, 0], 0.6)
    np.testing.assert_allclose(att["O_full"][0, 0], ref, rtol=0, atol=1e-10)


def test_no_expansion_is_vq_attention_over_level_zero():
    M0, C, L, d, N, T = 4, 3, 3, 6, 150, 64
    Q, K, V, cb = _deep_inputs(72, N, d, M0, C, L)
    pre = deep.precompute(K, V, cb, M0, C, L)
    att = deep.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, L, (0, 0), T, 0.6)
    top = np.argmin(((K[0, 0][:, None, :] - cb[0][None, :M0, :]) ** 2).sum(axis=2), axis=1)
    ref = _dense(Q[0, 0], cb[0][top], V[0, 0], 0.6)
    np.testing.assert_allclose(att["O_full"][0, 0], ref, rtol=0, atol=1e-10)


def test_statistics_hold_every_key_that_reached_a_node():
    M0, C, L, d, N = 3, 2, 4, 4, 400
    Q, K, V, cb = _deep_inputs(73, N, d, M0, C, L, B=2, H=2)
    pre = deep.precompute(K, V, cb, M0, C, L)
    offs = deep.level_offsets(M0, C, L)
    for b in range(2):
        for h in range(2):
            n = pre["counts"][b, h]
            assert n[:M0].sum() == N
            for l in range(L - 1):
                for j in range(M0 * C ** l):
                    kids = offs[l + 1] + j * C + np.arange(C)
                    stay = int(((pre["assign"][b, h] == offs[l] + j)).sum())
                    assert n[offs[l] + j] == n[kids].sum() + stay
                    np.testing.assert_allclose(
                        pre["vsum"][b, h, offs[l] + j],
                        pre["vsum"][b, h, kids].sum(axis=0) + V[b, h][pre["assign"][b, h] == offs[l] + j].sum(axis=0),
                        rtol=0, atol=1e-9)


def test_importance_normaliser_is_the_current_approximation():
    """At every level the candidates' importance and the unexpanded nodes'
    shares, all under the level's normaliser, account for each query once."""
    M0, C, L, d, N, T = 4, 3, 3, 6, 180, 64
    Q, K, V, cb = _deep_inputs(74, N, d, M0, C, L)
    pre = deep.precompute(K, V, cb, M0, C, L)
    Ps = (2, 3)
    att = deep.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, L, Ps, T, 0.6)
    offs = deep.level_offsets(M0, C, L)
    n = pre["counts"][0, 0].astype(np.float64)
    ntiles = (N + T - 1) // T
    for t in range(ntiles):
        q = Q[0, 0, t * T:min(N, (t + 1) * T)]
        S = 0.6 * (q @ cb[0].T)
        m = np.where(n[None, :M0] > 0, S[:, :M0], -np.inf).max(axis=1)
        A = np.where(n[None, :] > 0, np.exp(S - m[:, None]), 0.0)
        # level 1: children of the level-0 selection, plus every level-0 node's
        # keys that are not represented by those children
        sel0 = att["selected"][t][0]
        z1 = att["zbar"][t][1]
        total = att["score"][t][1].sum() * q.shape[0]
        for p in range(M0):
            kids = offs[1] + p * C + np.arange(C)
            rest = n[p] - (n[kids].sum() if p in sel0 else 0.0)
            total += (A[:, p] * rest / z1).sum()
        assert abs(total - q.shape[0]) < 1e-9
