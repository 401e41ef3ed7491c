"""Randomised agreement of the fp64 C oracle with the per-key brute force
(``oracle/brute.py``) over small shapes drawn by hypothesis: tree sizes,
tile sizes, P from 0 to M0, integer-grid inputs (exact ties) and random ones.
The fixed pins (``oracle_pins.py``) cover chosen cases; this covers the
space between them."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import brute
from oracle import oracle as orc

_ORACLE = orc.get()


@st.composite
def problems(draw):
    M0 = draw(st.integers(1, 6))
    C = draw(st.integers(0, 4))
    N = draw(st.integers(1, 40))
    d = draw(st.sampled_from([2, 3, 4, 8]))
    T = draw(st.sampled_from([4, 8, 16, 64]))
    P = draw(st.integers(0, M0)) if C > 0 else 0
    grid = draw(st.booleans())
    seed = draw(st.integers(0, 2 ** 31 - 1))
    scale = draw(st.sampled_from([0.25, 0.5, 1.0]))
    rng = np.random.default_rng(seed)
    shape_k, shape_cb = (1, 1, N, d), (1, M0 * (1 + C), d)
    if grid:
        K = rng.integers(-2, 3, size=shape_k).astype(np.float64)
        cb = rng.integers(-2, 3, size=shape_cb).astype(np.float64)
        Q = rng.integers(-2, 3, size=shape_k).astype(np.float64) * 0.5
    else:
        K = rng.standard_normal(shape_k)
        cb = rng.standard_normal(shape_cb)
        Q = rng.standard_normal(shape_k)
    V = rng.standard_normal(shape_k)
    return dict(M0=M0, C=C, N=N, d=d, T=T, P=P, K=K, V=V, Q=Q, cb=cb, scale=scale)


def _close_selection(a, b, score, P, band=1e-12):
    if P == 0 or list(a) == list(b):
        return True
    kth = np.sort(score)[::-1][P - 1]
    sure = set(np.nonzero(score > kth + band)[0].tolist())
    return sure <= set(a) and sure <= set(b)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_oracle_agrees_with_brute_force(pb):
    M0, C, P, T = pb["M0"], pb["C"], pb["P"], pb["T"]
    pre = _ORACLE.precompute(pb["K"], pb["V"], pb["cb"], M0, C)
    att = _ORACLE.attention(pb["Q"], pb["cb"], pre["counts"], pre["vsum"], M0, C, P, T, pb["scale"])
    bf = brute.brute_force(pb["Q"][0, 0].tolist(), pb["K"][0, 0].tolist(), pb["V"][0, 0].tolist(),
                           pb["cb"][0].tolist(), M0, C, P, T, pb["scale"])
    assert np.array_equal(pre["assign"][0, 0], np.array(bf["leaf"]))
    sc = np.array(bf["score"])
    np.testing.assert_allclose(att["score"], sc, rtol=0, atol=1e-12)
    for t in range(sc.shape[0]):
        assert _close_selection(att["selected"][t], bf["selected"][t], sc[t], P)
    O = att["O_full"][0, 0]
    assert np.abs(O - np.array(bf["O"])).max() <= 1e-12 * max(1.0, np.abs(O).max())
