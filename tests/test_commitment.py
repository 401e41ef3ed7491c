"""Commitment loss (paper, appendix "Per-layer codebook analysis", Table 7):
the oracle's definition pinned on CPU, the C-ABI argument checks, and the
GPU kernel against the oracle (marked gpu)."""
import numpy as np
import pytest

from adaptive_vector_quantized_avq_b200 import synthetic as syn
from oracle import oracle as orc


def _brute(K, cb, assign):
    B, H, N, d = K.shape
    out = np.zeros((B, H))
    for b in range(B):
        for h in range(H):
            for n in range(N):
                c = cb[h, assign[b, h, n]]
                out[b, h] += sum((K[b, h, n, j] - c[j]) ** 2 for j in range(d))
    return out


def test_commitment_matches_per_key_loop(oracle):
    wl = syn.small_workload(B=2, H=2, N=40, d=8, M0=4, C=2, seed=21, n_components=4)
    inp = syn.generate(wl)
    K, cb = inp.f64("K"), inp.f64("codebook")
    r = oracle.precompute(K, inp.f64("V"), cb, wl.M0, wl.C)
    got = orc.commitment(K, cb, r["assign"])
    np.testing.assert_allclose(got, _brute(K, cb, r["assign"]), rtol=1e-12)


def test_children_never_raise_the_commitment(oracle):
    """A child replaces its parent only when strictly closer, so the leaf
    assignment's loss is at most the parent-only loss, and strictly below it
    when any key moved."""
    wl = syn.small_workload(B=1, H=3, N=300, d=16, M0=8, C=4, seed=22, n_components=8)
    inp = syn.generate(wl)
    K, cb = inp.f64("K"), inp.f64("codebook")
    r = oracle.precompute(K, inp.f64("V"), cb, wl.M0, wl.C)
    leaf = r["assign"]
    parent = np.where(leaf < wl.M0, leaf, (leaf - wl.M0) // wl.C)
    lc, pc = orc.commitment(K, cb, leaf), orc.commitment(K, cb, parent)
    assert np.all(lc <= pc)
    moved = (leaf >= wl.M0).reshape(wl.H, -1).any(axis=1)
    assert np.all(lc[0][moved] < pc[0][moved])


def test_commitment_zero_when_keys_are_codewords(oracle):
    rng = np.random.default_rng(23)
    K = rng.standard_normal((1, 1, 6, 8))
    cb = np.concatenate([K[0, 0], np.repeat(K[0, 0], 1, axis=0)])[None]   # parents = keys, one child each
    r = oracle.precompute(K, K, cb, 6, 1)
    assert orc.commitment(K, cb, r["assign"])[0, 0] == 0.0


def test_flat_commitment_is_the_nearest_codeword_distance(oracle):
    """C = 0: the assigned codeword is the nearest one, so the loss is the sum
    of each key's smallest squared distance (a direct numpy minimum)."""
    wl = syn.small_workload(B=1, H=2, N=250, d=8, M0=12, C=0, seed=26, n_components=12)
    inp = syn.generate(wl)
    K, cb = inp.f64("K"), inp.f64("codebook")
    r = oracle.precompute(K, inp.f64("V"), cb, wl.M0, 0)
    got = orc.commitment(K, cb, r["assign"])
    for h in range(2):
        dmin = ((K[0, h][:, None, :] - cb[h][None, :, :]) ** 2).sum(axis=2).min(axis=1)
        assert abs(got[0, h] - dmin.sum()) <= 1e-12 * dmin.sum()


def test_commitment_argument_errors():
    """Rejected on the host before any CUDA call (no GPU needed)."""
    from adaptive_vector_quantized_avq_b200 import binding as bd
    from adaptive_vector_quantized_avq_b200 import build as bl
    bl.build()
    A = 1 << 20   # an aligned address that is never dereferenced
    shape = bd.make_shape(1, 2, 128, 64, 16, 4, bd.AVQ_BF16)
    assert bd.avq_commitment(shape, A, A, A, None, stream=0) == -1         # no output
    assert bd.avq_commitment(shape, A + 2, A, A, A, stream=0) == -1        # misaligned K
    assert bd.avq_commitment(shape, A, A, A, A + 4, stream=0) == -1        # misaligned output
    bad = bd.make_shape(1, 2, 128, 48, 16, 4, bd.AVQ_BF16)
    assert bd.avq_commitment(bad, A, A, A, A, stream=0) == -1              # d not in {64, 128}
    big = bd.make_shape(1, 2, 128, 64, 256, 4, bd.AVQ_BF16)
    assert bd.avq_commitment(big, A, A, A, A, stream=0) == -2              # M0 beyond the kernels


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["bf16-small", "f32-small", "max-64k"])
def test_commitment_gpu(oracle, name):
    import torch
    import parity
    from adaptive_vector_quantized_avq_b200 import binding as bd
    wl = {"bf16-small": syn.small_workload(B=2, H=3, N=777, d=128, M0=32, C=4, tile=128, dtype="bf16",
                                           seed=24, n_components=32),
          "f32-small": syn.small_workload(B=1, H=2, N=500, d=64, M0=16, C=8, tile=64, dtype="f32",
                                          seed=25, n_components=16),
          "max-64k": syn.WORKLOADS["max-64k"]}[name]
    inp = syn.generate(wl, with_q=False)
    K, cb = (parity.to_device(getattr(inp, n), wl.dtype) for n in ("K", "codebook"))
    # both sides take the oracle's assignment (no oracle input from the CUDA path)
    ora_assign = oracle.precompute(inp.f64("K"), inp.f64("V"), inp.f64("codebook"), wl.M0, wl.C)["assign"]
    assign = torch.from_numpy(np.ascontiguousarray(ora_assign, dtype=np.int32)).cuda()
    got = bd.commitment(K, cb, assign, wl.M0, wl.C).cpu().numpy()
    ref = orc.commitment(inp.f64("K"), inp.f64("codebook"), ora_assign)
    np.testing.assert_allclose(got, ref, rtol=2e-6)
    torch.cuda.synchronize()
