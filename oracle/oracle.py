"""ctypes wrapper around the fp64 C oracle (``avq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does. The shared library is compiled with gcc (``-O2 -ffp-contract=off
-fopenmp``) into ``oracle/_build`` on first use, or by ``build()``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "avq_oracle.c")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(BUILD_DIR, "libavq_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(src: str = SRC, out: str = LIB, extra: tuple = ()) -> str:
    """Compile ``src`` into the shared library ``out`` (returns ``out``)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _needs_build(src: str, out: str) -> bool:
    return not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src)


_P = np.ctypeslib.ndpointer
_f64 = _P(dtype=np.float64, flags="C_CONTIGUOUS")
_i32 = _P(dtype=np.int32, flags="C_CONTIGUOUS")
_i64 = _P(dtype=np.int64, flags="C_CONTIGUOUS")


def _opt(ptr_type):
    """ndpointer that also accepts None."""

    class _Opt(ptr_type):  # type: ignore[misc, valid-type]
        @classmethod
        def from_param(cls, obj):
            if obj is None:
                return None
            return super().from_param(obj)

    return _Opt


class Oracle:
    """The fp64 oracle. ``lib`` overrides the library path (mutation tests)."""

    def __init__(self, lib: str | None = None):
        if lib is None:
            if _needs_build(SRC, LIB):
                build()
            lib = LIB
        self.path = lib
        self._lib = ctypes.CDLL(lib)
        c = ctypes
        self._lib.oracle_precompute.restype = c.c_int
        self._lib.oracle_precompute.argtypes = [
            c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
            _f64, _f64, _f64, _i32, _i64, _f64, c.POINTER(c.c_int64), c.c_int]
        self._lib.oracle_attention.restype = c.c_int
        self._lib.oracle_attention.argtypes = [
            c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
            _f64, _f64, _i64, _f64, c.c_int, c.c_int, c.c_double,
            _opt(_i32), c.c_int, _opt(_i32), c.c_int,
            _f64, _i32, _f64, c.POINTER(c.c_int64), c.c_int]
        self._lib.oracle_max_threads.restype = c.c_int
        self._lib.oracle_max_threads.argtypes = []

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())

    def precompute(self, K: np.ndarray, V: np.ndarray, codebook: np.ndarray, M0: int, C: int,
                   nthreads: int | None = None) -> dict:
        """Assignment + full-tree statistics. K, V: [B,H,N,d]; codebook: [H,Mtot,d] (fp64)."""
        K = np.ascontiguousarray(K, dtype=np.float64)
        V = np.ascontiguousarray(V, dtype=np.float64)
        cb = np.ascontiguousarray(codebook, dtype=np.float64)
        B, H, N, d = K.shape
        Mtot = M0 * (1 + C)
        assert cb.shape == (H, Mtot, d), (cb.shape, (H, Mtot, d))
        assign = np.empty((B, H, N), dtype=np.int32)
        counts = np.empty((B, H, Mtot), dtype=np.int64)
        vsum = np.empty((B, H, Mtot, d), dtype=np.float64)
        evals = ctypes.c_int64(0)
        rc = self._lib.oracle_precompute(B, H, N, d, M0, C, K, V, cb, assign, counts, vsum,
                                         ctypes.byref(evals), nthreads or self.max_threads())
        if rc != 0:
            raise RuntimeError(f"oracle_precompute failed: {rc}")
        return {"assign": assign, "counts": counts, "vsum": vsum, "dist_evals": int(evals.value)}

    def attention(self, Q: np.ndarray, codebook: np.ndarray, counts: np.ndarray, vsum: np.ndarray,
                  M0: int, C: int, P: int, T: int, scale: float, tile_ids=None, forced=None,
                  parent_logit_from_children: bool = False, nthreads: int | None = None) -> dict:
        """Adaptive attention over all tiles, or over the listed global tile ids.

        Returns per listed tile: ``O`` [n,T,d], ``selected`` [n,P], ``score`` [n,M0];
        for a full run also ``O_full`` [B,H,N,d].
        """
        Q = np.ascontiguousarray(Q, dtype=np.float64)
        cb = np.ascontiguousarray(codebook, dtype=np.float64)
        counts = np.ascontiguousarray(counts, dtype=np.int64)
        vsum = np.ascontiguousarray(vsum, dtype=np.float64)
        B, H, N, d = Q.shape
        ntiles = (N + T - 1) // T
        if tile_ids is None:
            ids = None
            n = B * H * ntiles
        else:
            ids = np.ascontiguousarray(tile_ids, dtype=np.int32)
            n = int(ids.size)
        f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32).reshape(n, P)
        O = np.empty((n, T, d), dtype=np.float64)
        sel = np.empty((n, P), dtype=np.int32)
        score = np.empty((n, M0), dtype=np.float64)
        evals = ctypes.c_int64(0)
        rc = self._lib.oracle_attention(B, H, N, d, M0, C, Q, cb, counts, vsum, P, T,
                                        float(scale), ids, n, f, int(bool(parent_logit_from_children)),
                                        O, sel, score, ctypes.byref(evals),
                                        nthreads or self.max_threads())
        if rc != 0:
            raise RuntimeError(f"oracle_attention failed: {rc}")
        out = {"O": O, "selected": sel, "score": score, "logit_evals": int(evals.value)}
        if ids is None:
            out["O_full"] = O.reshape(B, H, ntiles * T, d)[:, :, :N, :]
            out["selected_full"] = sel.reshape(B, H, ntiles, P)
            out["score_full"] = score.reshape(B, H, ntiles, M0)
        return out


def commitment(K: np.ndarray, codebook: np.ndarray, assign: np.ndarray) -> np.ndarray:
    """Per-(b,h) sum over the keys of ||k - codebook[h, assign]||^2 in fp64
    (paper, appendix "Per-layer codebook analysis", Table 7: the commitment
    loss is this sum divided by N; the assigned codeword is the key's leaf).
    K [B,H,N,d], codebook [H,Mtot,d], assign [B,H,N] -> [B,H]."""
    K = np.asarray(K, dtype=np.float64)
    cb = np.asarray(codebook, dtype=np.float64)
    B, H, N, d = K.shape
    out = np.zeros((B, H))
    for b in range(B):
        for h in range(H):
            diff = K[b, h] - cb[h][assign[b, h]]
            out[b, h] = float((diff * diff).sum())
    return out


def capture(Q: np.ndarray, K: np.ndarray, assign: np.ndarray, selected: np.ndarray, M0: int, C: int,
            tile: int, scale: float, rows=None) -> np.ndarray:
    """Top-P capture of every query (paper §5.2 "Elastic Inference", Table 6,
    and Figure 7): the share of the query's true softmax attention weight,
    softmax_k(scale * Q_i . K_k) over all N keys of its (b,h), that falls on
    keys whose parent is among the P parents selected for the query's tile.
    A key's parent is its leaf when the leaf is a parent (id < M0), else the
    parent of that child ((id - M0) // C); ids outside [0, M0*(1+C)) and
    selected entries outside [0, M0) never count towards the numerator.

    Q, K [B,H,N,d]; assign [B,H,N]; selected [B,H,ceil(N/tile),P].
    Returns fp64 [B,H,N], or, with ``rows`` (flat indices b*H*N + h*N + i),
    the values of those queries only."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    B, H, N, d = Q.shape
    Mtot = M0 * (1 + C)
    a = np.asarray(assign).reshape(B * H, N).astype(np.int64)
    parent = np.where(a < M0, a, (a - M0) // max(C, 1))
    parent = np.where((a >= 0) & (a < Mtot), parent, -1)
    ntiles = (N + tile - 1) // tile
    sel = np.asarray(selected).reshape(B * H, ntiles, -1) if N else None
    Qf, Kf = Q.reshape(B * H, N, d), K.reshape(B * H, N, d)
    want = np.arange(B * H * N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros(want.size)
    for j, r in enumerate(want):
        bh, i = divmod(int(r), N)
        s = scale * (Kf[bh] @ Qf[bh, i])                  # logits over all keys
        w = np.exp(s - s.max())
        w /= w.sum()                                       # true attention weights
        chosen = [int(v) for v in sel[bh, i // tile] if 0 <= v < M0]
        on = np.isin(parent[bh], chosen)
        out[j] = float(w[on].sum())
    return out.reshape(B, H, N) if rows is None else out


_DEFAULT: Oracle | None = None


def get() -> Oracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
