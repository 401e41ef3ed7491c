"""Seeded synthetic inputs for AVQ-attention: keys, queries, values and a
frozen two-level tree codebook.

This module holds no step of the method's arithmetic. It only draws random
numbers, rounds them to the storage dtype and builds a codebook that satisfies
the parent-child constraint of AVQ-Attention (§4.1 "Parent-child constraint":
every parent equals the arithmetic mean of its children). It is the one piece
shared by the CUDA path's tests and benchmark and by the CPU oracle's tests;
it imports neither of them.

Recipe (all draws from ``numpy.random.default_rng`` sub-streams of one seed):

* per head, ``n_components`` mixture centres ~ N(0, I_d);
* mixture weights uniform, or Zipf with exponent ``zipf_s`` over the
  component rank (component 0 is the heaviest);
* keys and queries are independent draws from the same per-head mixture:
  centre + N(0, sigma^2 I), sigma = 0.3;
* values ~ N(0, 1);
* codebook parents are the first ``M0`` components by rank; each parent gets
  ``C`` children = centre + N(0, 0.1^2 I) (the 0.1 child-initialisation scale
  of AVQ-Attention, Appendix F "ImageNet-1k"), rounded to the grid 2^-5;
  per coordinate, the first r children are moved down by one grid unit so that
  the child sum is a multiple of C grid units, and the parent is then set to
  the exact child mean. Every codebook value is an integer multiple of 2^-5
  with magnitude below 4, hence exact in bf16 and fp32, and the constraint
  holds exactly in the storage dtype;
* bf16 tensors are rounded from the fp64 draws (through fp32, round to
  nearest even at each step).

Codebook layout: ``[H, M0 * (1 + C), d]`` in tree order: parents ``0..M0-1``,
then child ``c`` of parent ``p`` at row ``M0 + p * C + c``.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

GRID = 2.0 ** -5          # codebook value grid (exact in bf16 for |x| < 8)
_GRID_LIMIT_UNITS = 120   # clamp |x| <= 120 * 2^-5 = 3.75 before the sum fix-up


# --------------------------------------------------------------------------
# dtype helpers (storage format <-> exact fp64 values)
# --------------------------------------------------------------------------
def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 (nearest even) -> bf16 (nearest even); return uint16 bits."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to fp64 exactly."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return f64_to_bf16_bits(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def storage_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    """One synthetic AVQ-attention problem (all heads share the sizes)."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str            # "f32" or "bf16"
    M0: int
    C: int
    P: tuple              # refinement budgets to run (first one is the default)
    tile: int
    n_components: int
    zipf_s: float | None  # None -> uniform mixture weights
    sigma: float = 0.3
    child_sigma: float = 0.1
    seed: int = 0
    scale: float | None = None   # None -> 1/sqrt(d)
    note: str = field(default="", compare=False)
    L: int = 2                   # codebook depth (2: parents and children)

    @property
    def Mtot(self) -> int:
        return self.M0 * sum(self.C ** k for k in range(self.L))   # M0 (1 + C) at depth 2

    @property
    def rows(self) -> int:
        return self.B * self.H * self.N

    @property
    def ntiles(self) -> int:
        return (self.N + self.tile - 1) // self.tile

    @property
    def softmax_scale(self) -> float:
        return float(self.scale) if self.scale is not None else 1.0 / float(np.sqrt(self.d))

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads the method is measured and checked on.
WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny-fp32", 1, 1, 1024, 64, "f32", 16, 4, (4,), 64, 16, None,
                 note="16-component isotropic mixture, fp32, correctness case"),
        Workload("vit-b", 8, 12, 4096, 64, "bf16", 64, 4, (8,), 128, 64, None,
                 note="ViT-B-like self-attention shape"),
        Workload("long-16k", 2, 16, 16384, 64, "bf16", 128, 4, (16,), 128, 128, 1.1,
                 note="long sequence, Zipf(1.1) cluster sizes"),
        Workload("max-64k", 1, 16, 65536, 64, "bf16", 128, 8, (16,), 128, 256, 1.1,
                 note="maximum length, 256-component Zipf mixture"),
        Workload("refine-d128", 1, 8, 16384, 128, "bf16", 64, 8, (0, 4, 16, 64), 128, 64, None,
                 note="refinement sweep over P at head dim 128"),
        Workload("flat-512", 1, 16, 16384, 64, "bf16", 512, 0, (0,), 128, 512, None,
                 note="flat VQ attention (no tree, nothing selected) over 512 codewords"),
        Workload("deep3-16k", 1, 8, 16384, 64, "bf16", 64, 4, ((8, 16),), 128, 64, None,
                 note="depth-3 tree (64 / 256 / 1024 nodes), 8 then 16 nodes expanded per tile", L=3),
    ]
}


# --------------------------------------------------------------------------
# generation
# --------------------------------------------------------------------------
def _mixture_weights(n: int, zipf_s: float | None) -> np.ndarray:
    if zipf_s is None:
        return np.full(n, 1.0 / n)
    w = 1.0 / np.arange(1, n + 1, dtype=np.float64) ** zipf_s
    return w / w.sum()


def make_tree_codebook(centres: np.ndarray, M0: int, C: int, child_sigma: float,
                       rng: np.random.Generator) -> np.ndarray:
    """Tree codebook ``[H, M0*(1+C), d]`` (fp64 values on the 2^-5 grid).

    Parents are ``centres[:, :M0]`` moved to the exact mean of their children;
    with C == 0 (a flat codebook) they are the centres on the grid.
    """
    H, _, d = centres.shape
    par = centres[:, :M0, :]                                       # [H, M0, d]
    if C == 0:
        return np.clip(np.rint(par / GRID), -_GRID_LIMIT_UNITS, _GRID_LIMIT_UNITS) * GRID
    noise = rng.standard_normal((H, M0, C, d))
    child = par[:, :, None, :] + child_sigma * noise               # [H, M0, C, d]
    units = np.clip(np.rint(child / GRID), -_GRID_LIMIT_UNITS, _GRID_LIMIT_UNITS).astype(np.int64)
    r = np.mod(units.sum(axis=2), C)                               # [H, M0, d] in 0..C-1
    cidx = np.arange(C)[None, None, :, None]
    units = units - (cidx < r[:, :, None, :]).astype(np.int64)     # first r children -1 unit
    psum = units.sum(axis=2)
    assert np.all(np.mod(psum, C) == 0)
    parent_units = psum // C
    cb = np.empty((H, M0 * (1 + C), d), dtype=np.float64)
    cb[:, :M0, :] = parent_units * GRID
    cb[:, M0:, :] = (units * GRID).reshape(H, M0 * C, d)
    return cb


def make_deep_codebook(centres: np.ndarray, M0: int, C: int, L: int, child_sigma: float,
                       rng: np.random.Generator) -> np.ndarray:
    """Depth-L codebook ``[H, M0*(1+C+...+C^(L-1)), d]`` (fp64 values on the
    2^-5 grid), levels stored one after another, node j of level l with the
    children j*C + c of level l+1.

    Level l+1 nodes are drawn around their parents with spread
    ``child_sigma * 2^-l``; then every node is set to the exact mean of its
    deepest descendants, so that each node is the exact mean of its children
    in storage (bf16 included). The deepest nodes' grid units are adjusted
    first so that every subtree's unit sum divides by its size: a node at
    level l needs divisibility by C^(L-1-l); the remainder is a multiple of
    C^(L-2-l) (its child subtrees already divide) and is removed one step of
    that size at a time from distinct deepest descendants, which keeps every
    deeper constraint. L = 2 gives the two-level layout."""
    H, _, d = centres.shape
    assert L >= 1 and C >= 1
    nodes = [centres[:, :M0, :]]
    for l in range(1, L):
        par = np.repeat(nodes[-1], C, axis=1)
        nodes.append(par + child_sigma * 2.0 ** (1 - l) * rng.standard_normal(par.shape))
    headroom = sum(C ** k for k in range(L - 1))              # largest total adjustment of one unit
    units = np.clip(np.rint(nodes[-1] / GRID), -(_GRID_LIMIT_UNITS - headroom),
                    _GRID_LIMIT_UNITS - headroom).astype(np.int64)   # [H, M0*C^(L-1), d]
    for l in range(L - 2, -1, -1):
        size = C ** (L - 1 - l)                                # deepest nodes under a level-l node
        step = size // C
        sub = units.reshape(H, -1, size, d)                    # [H, M0*C^l, size, d] (a view)
        rem = np.mod(sub.sum(axis=2), size)                    # multiple of step, < size
        k = rem // step                                        # steps to remove, 0 .. C-1
        # remove one step from the first k deepest descendants of distinct child subtrees
        first = np.arange(C) * step                            # the first deepest node of each child subtree
        take = np.arange(C)[None, None, :, None] < k[:, :, None, :]
        sub[:, :, first, :] -= step * take
    assert np.all(np.mod(units.reshape(H, M0, -1, d).sum(axis=2), C ** (L - 1)) == 0)
    levels = []
    for l in range(L):
        size = C ** (L - 1 - l)
        sums = units.reshape(H, M0 * C ** l, size, d).sum(axis=2)
        levels.append((sums // size) * GRID)
    return np.concatenate(levels, axis=1)


@dataclass
class Inputs:
    """Storage-format arrays (fp32, or bf16 as uint16 bits) plus their sizes."""

    wl: Workload
    K: np.ndarray          # [B,H,N,d]
    V: np.ndarray          # [B,H,N,d]
    Q: np.ndarray          # [B,H,N,d]
    codebook: np.ndarray   # [H,Mtot,d]

    def f64(self, name: str) -> np.ndarray:
        return storage_to_f64(getattr(self, name), self.wl.dtype)


def generate(wl: Workload, *, with_q: bool = True, with_kv: bool = True) -> Inputs:
    """Draw the seeded inputs of ``wl`` (deterministic in ``wl.seed``)."""
    ss = np.random.SeedSequence(wl.seed)
    s_centre, s_lab_k, s_lab_q, s_k, s_q, s_v, s_cb = ss.spawn(7)
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    centres = np.random.default_rng(s_centre).standard_normal((H, wl.n_components, d))
    if wl.L == 2:
        cb = make_tree_codebook(centres, wl.M0, wl.C, wl.child_sigma, np.random.default_rng(s_cb))
    else:
        cb = make_deep_codebook(centres, wl.M0, wl.C, wl.L, wl.child_sigma, np.random.default_rng(s_cb))
    weights = _mixture_weights(wl.n_components, wl.zipf_s)

    def mixture_draw(s_lab, s_pt):
        rl = np.random.default_rng(s_lab)
        rp = np.random.default_rng(s_pt)
        out = np.empty((B, H, N, d), dtype=np.float32 if wl.dtype == "f32" else np.uint16)
        for b in range(B):
            for h in range(H):
                lab = rl.choice(wl.n_components, size=N, p=weights)
                x = centres[h, lab, :] + wl.sigma * rp.standard_normal((N, d))
                out[b, h] = to_storage(x, wl.dtype)
        return out

    empty = np.empty((B, H, 0, d), dtype=np.float32 if wl.dtype == "f32" else np.uint16)
    K = mixture_draw(s_lab_k, s_k) if with_kv else empty
    Q = mixture_draw(s_lab_q, s_q) if with_q else empty
    if with_kv:
        rv = np.random.default_rng(s_v)
        V = np.empty_like(K)
        for b in range(B):
            for h in range(H):
                V[b, h] = to_storage(rv.standard_normal((N, d)), wl.dtype)
    else:
        V = empty
    return Inputs(wl, K, V, Q, to_storage(cb, wl.dtype))


def small_workload(N: int = 256, d: int = 8, M0: int = 8, C: int = 4, P=(2,), tile: int = 64,
                   B: int = 1, H: int = 1, dtype: str = "f32", n_components: int | None = None,
                   zipf_s: float | None = None, seed: int = 0, scale: float | None = None,
                   sigma: float = 0.3, L: int = 2) -> Workload:
    """A small workload for oracle and parity checks (L: codebook depth)."""
    return Workload(f"small-{B}x{H}x{N}x{d}-{M0}-{C}" + (f"-L{L}" if L != 2 else ""), B, H, N, d, dtype, M0, C,
                    tuple(P) if not isinstance(P, int) else (P,), tile,
                    n_components if n_components is not None else M0, zipf_s,
                    sigma=sigma, seed=seed, scale=scale, L=L)
