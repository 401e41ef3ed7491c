"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle)


def test_oracle_parent_logit_recovery(oracle):
    """Under the parent-child constraint the parent logit equals the mean of its
    children's logits (AVQ-Attention §4.3, "Child attention"), so recovering it
    that way changes the output only by rounding."""
    import numpy as np
    from adaptive_vector_quantized_avq_b200 import synthetic as syn
    wl = syn.small_workload(N=512, d=16, M0=8, C=4, tile=64, seed=21)
    inp = syn.generate(wl)
    cb = inp.f64("codebook")
    par = cb[0, :wl.M0]
    kids = cb[0, wl.M0:].reshape(wl.M0, wl.C, wl.d)
    assert np.array_equal(par, kids.mean(axis=1)), "generator broke the constraint"
    pre = oracle.precompute(inp.f64("K"), inp.f64("V"), cb, wl.M0, wl.C)
    for P in (2, 8):
        a = oracle.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], wl.M0, wl.C, P,
                             wl.tile, wl.softmax_scale)
        b = oracle.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], wl.M0, wl.C, P,
                             wl.tile, wl.softmax_scale, parent_logit_from_children=True)
        assert np.array_equal(a["selected"], b["selected"])
        assert np.abs(a["O"] - b["O"]).max() < 1e-12


def test_oracle_forced_selection(oracle):
    """A forced selection equal to the oracle's own reproduces its output."""
    import numpy as np
    from adaptive_vector_quantized_avq_b200 import synthetic as syn
    wl = syn.small_workload(N=300, d=8, M0=8, C=3, tile=64, seed=22)
    inp = syn.generate(wl)
    cb = inp.f64("codebook")
    pre = oracle.precompute(inp.f64("K"), inp.f64("V"), cb, wl.M0, wl.C)
    a = oracle.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], wl.M0, wl.C, 3, wl.tile, 0.5)
    ids = np.array([0, 2, 4])
    b = oracle.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], wl.M0, wl.C, 3, wl.tile, 0.5,
                         tile_ids=ids, forced=a["selected"][ids])
    assert np.array_equal(a["O"][ids], b["O"])
    c = oracle.attention(inp.f64("Q"), cb, pre["counts"], pre["vsum"], wl.M0, wl.C, 3, wl.tile, 0.5,
                         tile_ids=ids, forced=np.zeros((3, 3), np.int32) + [5, 6, 7])
    assert not np.allclose(a["O"][ids], c["O"])
