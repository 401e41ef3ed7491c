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


def test_capture_argument_errors():
    """Rejected on the host before any CUDA call (no GPU needed)."""
    from adaptive_vector_quantized_avq_b200 import binding as bd
    from adaptive_vector_quantized_avq_b200 import build as bl
    bl.build()
    A = 1 << 20   # an aligned address that is never dereferenced
    ws = bd.avq_capture_workspace_bytes
    shape = bd.make_shape(1, 2, 300, 64, 16, 4, bd.AVQ_BF16)
    assert ws(shape, 4, 128) == 256
    assert ws(shape, 4, 64) == 0                       # 128-query tiles only
    assert ws(bd.make_shape(1, 2, 300, 64, 16, 4, bd.AVQ_F32), 4, 128) == 0
    call = lambda s, P=4, tile=128, out=A, w=A, wsb=256, sel=A: bd.avq_capture(
        s, A, A, A, sel, P, tile, 0.125, out, w, wsb, 0)
    assert call(shape, out=None) == -1                 # no output
    assert call(shape, out=A + 2) == -1                # misaligned output
    assert call(shape, P=17) == -1                     # P > M0
    assert call(shape, sel=None) == -1                 # P > 0 needs the selection
    assert call(shape, tile=64) == -2                  # tile 64: not built
    assert call(shape, wsb=128) == -5                  # workspace too small
    assert call(bd.make_shape(1, 2, 300, 64, 16, 4, bd.AVQ_F32)) == -2
    assert call(bd.make_shape(1, 2, 300, 48, 16, 4, bd.AVQ_BF16)) == -1    # d not in {64, 128}


# --------------------------------------------------------------------- GPU
CAPTURE_TOL = 1e-4   # absolute, on a fraction in [0, 1]


def _gpu_case(oracle, wl, P, rows=None, seed=0):
    import torch
    import parity
    from adaptive_vector_quantized_avq_b200 import binding as bd
    inp = syn.generate(wl)
    Qf, Kf, Vf, cbf = inp.f64("Q"), inp.f64("K"), inp.f64("V"), inp.f64("codebook")
    pre = oracle.precompute(Kf, Vf, cbf, wl.M0, wl.C)
    if P > 0:
        nt = wl.ntiles
        ids = np.arange(wl.B * wl.H * nt) if rows is None else np.unique(np.asarray(rows) // wl.N * nt +
                                                                         (np.asarray(rows) % wl.N) // wl.tile)
        att = oracle.attention(Qf, cbf, pre["counts"], pre["vsum"], wl.M0, wl.C, P, wl.tile,
                               wl.softmax_scale, tile_ids=ids)
        sel = np.zeros((wl.B * wl.H * nt, P), np.int32)
        sel[ids] = att["selected"]
        sel = sel.reshape(wl.B, wl.H, nt, P)
    else:
        sel = np.zeros((wl.B, wl.H, wl.ntiles, 0), np.int32)
    Q, K = (parity.to_device(getattr(inp, n), wl.dtype) for n in ("Q", "K"))
    assign = torch.from_numpy(np.ascontiguousarray(pre["assign"], dtype=np.int32)).cuda()
    selected = torch.from_numpy(np.ascontiguousarray(sel)).cuda()
    got = bd.capture(Q, K, assign, selected, wl.M0, wl.C, P, wl.tile, wl.softmax_scale).cpu().numpy()
    torch.cuda.synchronize()
    ref = orc.capture(Qf, Kf, pre["assign"], sel, wl.M0, wl.C, wl.tile, wl.softmax_scale, rows=rows)
    g = got.reshape(-1) if rows is None else got.reshape(-1)[np.asarray(rows)]
    err = np.abs(g - ref.reshape(-1)).max()
    assert err <= CAPTURE_TOL, f"capture differs by {err}"
    return err, float(ref.mean())


@pytest.mark.gpu
@pytest.mark.parametrize("name,P", [("d64-ragged", 8), ("d128", 4), ("one-tile", 2), ("p0", 0),
                                    ("pmax", 16)])
def test_capture_gpu_small(oracle, name, P):
    wl = {"d64-ragged": syn.small_workload(B=2, H=2, N=1000, d=64, M0=32, C=4, tile=128, dtype="bf16",
                                           seed=36, n_components=40),
          "d128": syn.small_workload(B=1, H=2, N=555, d=128, M0=16, C=8, tile=128, dtype="bf16",
                                     seed=37, n_components=16),
          "one-tile": syn.small_workload(B=1, H=1, N=100, d=64, M0=4, C=2, tile=128, dtype="bf16",
                                         seed=38, n_components=4),
          "p0": syn.small_workload(B=1, H=2, N=300, d=64, M0=16, C=4, tile=128, dtype="bf16",
                                   seed=39, n_components=16),
          "pmax": syn.small_workload(B=1, H=2, N=300, d=64, M0=16, C=4, tile=128, dtype="bf16",
                                     seed=40, n_components=16)}[name]
    err, mean = _gpu_case(oracle, wl, P)
    print(name, P, err, mean)


@pytest.mark.gpu
def test_capture_gpu_max64k_sampled(oracle):
    """The full max-64k workload at its P; 48 sampled queries (with the first
    and last) compared against the oracle."""
    wl = syn.WORKLOADS["max-64k"]
    rng = np.random.default_rng(41)
    rows = np.unique(np.concatenate([[0, wl.rows - 1], rng.choice(wl.rows, 46, replace=False)]))
    err, mean = _gpu_case(oracle, wl, wl.P[-1], rows=rows)
    print("max-64k", err, mean)
