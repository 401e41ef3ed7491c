"""The seeded input generator (no GPU)."""
import numpy as np
import torch

from adaptive_vector_quantized_avq_b200 import synthetic as syn


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        [0.0, -0.0, 1.0, 3.75, -4.0, 1e-30]])
    ours = syn.f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = syn.bf16_bits_to_f64(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_codebook_constraint_exact_in_storage_dtype():
    for name in ("tiny-fp32", "vit-b", "refine-d128"):
        wl = syn.WORKLOADS[name].with_(B=1, N=8)
        inp = syn.generate(wl)
        cb = inp.f64("codebook")
        assert cb.shape == (wl.H, wl.Mtot, wl.d)
        par = cb[:, :wl.M0]
        kids = cb[:, wl.M0:].reshape(wl.H, wl.M0, wl.C, wl.d)
        assert np.array_equal(par * wl.C, kids.sum(axis=2))
        # values are on the 2^-5 grid and survive the storage round trip
        assert np.array_equal(np.rint(cb / syn.GRID) * syn.GRID, cb)
        assert np.array_equal(syn.storage_to_f64(syn.to_storage(cb, wl.dtype), wl.dtype), cb)


def test_generator_is_deterministic_and_seeded():
    wl = syn.small_workload(N=64, d=8, M0=4, C=2, dtype="bf16", B=2, H=3)
    a, b = syn.generate(wl), syn.generate(wl)
    for k in ("K", "V", "Q", "codebook"):
        assert np.array_equal(getattr(a, k), getattr(b, k))
    c = syn.generate(wl.with_(seed=1))
    assert not np.array_equal(a.K, c.K)
    assert a.K.dtype == np.uint16 and a.K.shape == (2, 3, 64, 8)


def test_mixture_statistics():
    wl = syn.small_workload(N=20000, d=16, M0=8, C=2, n_components=8, sigma=0.3, seed=3)
    inp = syn.generate(wl)
    K = inp.f64("K")[0, 0]
    cb = inp.f64("codebook")[0, :8]
    d2 = ((K[:, None, :] - cb[None]) ** 2).sum(-1).min(1)
    # nearest-centre squared distance ~ d*sigma^2 (+ small child-mean offset)
    assert 0.8 * 16 * 0.09 < np.median(d2) < 1.6 * 16 * 0.09


def test_zipf_weights_heavy_first():
    w = syn._mixture_weights(256, 1.1)
    assert np.all(np.diff(w) < 0) and abs(w.sum() - 1) < 1e-12


def test_flat_codebook_is_the_centres_on_the_grid():
    """C = 0: the codebook is M0 codewords (no children), on the bf16-exact grid,
    spread over distinct centres (no divide-by-zero fix-up)."""
    wl = syn.WORKLOADS["flat-512"].with_(N=16, H=2)
    inp = syn.generate(wl)
    cb = inp.f64("codebook")
    assert cb.shape == (2, 512, 64) and wl.Mtot == 512
    assert np.array_equal(np.rint(cb / syn.GRID) * syn.GRID, cb)
    assert np.abs(cb).max() <= 3.75
    assert len(np.unique(cb[0], axis=0)) == 512
    assert np.array_equal(syn.storage_to_f64(syn.to_storage(cb, "bf16"), "bf16"), cb)


def test_deep_codebook_means_exact_at_every_level():
    """Depth-L codebooks: every node is the exact mean of its C children in
    storage (bf16 included), on the grid and within range; L = 2 has the
    two-level layout and constraint."""
    rng = np.random.default_rng(5)
    for (M0, C, L, d) in [(4, 2, 3, 8), (8, 8, 3, 16), (3, 4, 4, 8), (16, 4, 2, 8), (2, 3, 1, 4)]:
        cen = rng.standard_normal((2, M0 + 3, d))
        cb = syn.make_deep_codebook(cen, M0, C, L, 0.1, np.random.default_rng(1))
        offs = [sum(M0 * C ** k for k in range(lv)) for lv in range(L + 1)]
        assert cb.shape == (2, offs[L], d)
        assert np.array_equal(np.rint(cb / syn.GRID) * syn.GRID, cb) and np.abs(cb).max() <= 3.75
        assert np.array_equal(syn.storage_to_f64(syn.to_storage(cb, "bf16"), "bf16"), cb)
        for lv in range(L - 1):
            par = cb[:, offs[lv]:offs[lv + 1]]
            kids = cb[:, offs[lv + 1]:offs[lv + 2]].reshape(2, M0 * C ** lv, C, d)
            assert np.array_equal(par * C, kids.sum(axis=2)), (M0, C, L, lv)
        assert np.abs(cb[:, :M0] - cen[:, :M0]).max() < 1.0      # parents stay near their centres


def test_depth_in_workloads():
    """L = 2 keeps the two-level inputs bit for bit; L = 3 draws a depth-3
    codebook of M0 (1 + C + C^2) rows that the deep oracle accepts."""
    wl2 = syn.small_workload(N=64, d=8, M0=4, C=2, dtype="bf16", seed=7)
    a, b = syn.generate(wl2), syn.generate(wl2.with_(L=2))
    assert np.array_equal(a.codebook, b.codebook) and wl2.Mtot == 12
    wl3 = syn.small_workload(N=300, d=8, M0=4, C=2, dtype="bf16", seed=7, L=3)
    assert wl3.Mtot == 4 * (1 + 2 + 4)
    inp = syn.generate(wl3)
    cb = inp.f64("codebook")
    assert cb.shape == (1, 28, 8)
    assert np.array_equal(cb[:, 4:12] * 2, cb[:, 12:28].reshape(1, 8, 2, 8).sum(axis=2))
    from oracle import deep
    pre = deep.precompute(inp.f64("K"), inp.f64("V"), cb, 4, 2, 3)
    assert pre["counts"][0, 0, :4].sum() == 300
