"""Deeper codebook hierarchies (more than one level of children): fp64
reference in plain numpy.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does.

The pages propose deeper hierarchies without defining or testing them
(AVQ-Attention, §6 "Discussion and Conclusion": each further level adds P·C
codes to the attention cost and multiplies the codebook's resolution by C).
This module carries the two-level method's steps (§4.2 assignment and
full-tree aggregation, §4.3 importance, child spawning and the correction
of the replaced parent share) down every level:

* a codebook of depth L has M0 nodes at level 0 and M0·C^l at level l; node j
  of level l has the children j·C + c (c < C) at level l + 1; rows are stored
  level after level, so that L = 2 is the two-level layout
  [parents | M0 + p·C + c];
* assignment: the nearest level-0 node (first index on ties), then, level by
  level, the nearest child of the current node (first on ties) replaces it
  only when strictly closer; the descent stops at the first level where no
  child is closer; the key's leaf is the last node reached;
* statistics: every node on a key's path counts the key and sums its value,
  so a node holds all keys that reached it;
* attention, per query tile, one shift m_i per row (the largest level-0 logit
  among non-empty nodes): level-0 attention A = exp(S - m) over non-empty
  nodes, Zbar = sum A n, Xbar = sum A vsum; then for l = 0 .. L-2 the
  candidates (level 0: every level-0 node; level l >= 1: the children of the
  nodes expanded at level l - 1) get the importance sum_i A_ic n_c / Zbar_i,
  with the Zbar of the approximation so far, and the P_l candidates of
  largest importance (ties to the lower row id) are expanded: every child g
  of an expanded node f adds (A_g - A_f) [vsum_g, n_g] to Xbar and Zbar.
  O = Xbar / Zbar.

Distances are summed in index order with each square rounded before the add,
as the two-level C oracle does, so that L = 2 reproduces its assignment bit
for bit.
"""
from __future__ import annotations

import numpy as np


def level_sizes(M0: int, C: int, L: int) -> list[int]:
    return [M0 * C ** l for l in range(L)]


def level_offsets(M0: int, C: int, L: int) -> list[int]:
    offs, acc = [], 0
    for n in level_sizes(M0, C, L):
        offs.append(acc)
        acc += n
    return offs


def total_rows(M0: int, C: int, L: int) -> int:
    return sum(level_sizes(M0, C, L))


def _sq_dist_seq(K: np.ndarray, Cw: np.ndarray) -> np.ndarray:
    """||K_n - Cw_{n,j}||^2 with terms added in index order. K [N,d];
    Cw [M,d] (shared) or [N,M,d] (per key). Returns [N,M]."""
    N, d = K.shape
    out = np.zeros((N, Cw.shape[-2]))
    for j in range(d):
        c = Cw[..., j] if Cw.ndim == 3 else Cw[None, :, j]
        t = K[:, j:j + 1] - c
        out += t * t
    return out


def precompute(K: np.ndarray, V: np.ndarray, codebook: np.ndarray, M0: int, C: int, L: int) -> dict:
    """Assignment and full-tree statistics. K, V [B,H,N,d]; codebook
    [H, total_rows(M0,C,L), d]. Returns assign [B,H,N] (row ids), depth
    [B,H,N] (level of the leaf), counts [B,H,Mtot] int64, vsum [B,H,Mtot,d]."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    cb = np.asarray(codebook, dtype=np.float64)
    B, H, N, d = K.shape
    offs = level_offsets(M0, C, L)
    Mtot = total_rows(M0, C, L)
    assert cb.shape == (H, Mtot, d), (cb.shape, (H, Mtot, d))
    assign = np.zeros((B, H, N), dtype=np.int64)
    depth = np.zeros((B, H, N), dtype=np.int64)
    counts = np.zeros((B, H, Mtot), dtype=np.int64)
    vsum = np.zeros((B, H, Mtot, d))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            k, v, c = K[b, h], V[b, h], cb[h]
            D = _sq_dist_seq(k, c[:M0])
            local = np.argmin(D, axis=1)             # first index on ties
            dist = D[rows, local]
            node = local.copy()
            lev = np.zeros(N, dtype=np.int64)
            active = np.ones(N, dtype=bool)
            np.add.at(counts[b, h], node, 1)
            np.add.at(vsum[b, h], node, v)
            for l in range(1, L):
                ch_local = local[:, None] * C + np.arange(C)[None, :]
                ch = offs[l] + ch_local
                Dc = _sq_dist_seq(k, c[ch])
                best = np.argmin(Dc, axis=1)
                dc = Dc[rows, best]
                move = active & (dc < dist)
                local = np.where(move, ch_local[rows, best], local)
                node = np.where(move, ch[rows, best], node)
                dist = np.where(move, dc, dist)
                lev = np.where(move, l, lev)
                active = move
                np.add.at(counts[b, h], node[move], 1)
                np.add.at(vsum[b, h], node[move], v[move])
            assign[b, h] = node
            depth[b, h] = lev
    return {"assign": assign, "depth": depth, "counts": counts, "vsum": vsum}


def _p_levels(P, L: int) -> list[int]:
    if np.isscalar(P):
        return [int(P)] * (L - 1)
    P = [int(x) for x in P]
    assert len(P) == L - 1, "one P per expanded level"
    return P


def attention(Q: np.ndarray, codebook: np.ndarray, counts: np.ndarray, vsum: np.ndarray, M0: int, C: int,
              L: int, P, T: int, scale: float, tile_ids=None) -> dict:
    """Adaptive attention over a depth-L tree for every tile (or the listed
    global tile ids b*H*ntiles + h*ntiles + t). P: one number for every
    level or a sequence of L-1. Returns O [n,T,d] (rows past N are 0), and
    per tile and expanded level l: ``candidates[j][l]`` (row ids),
    ``score[j][l]`` (importance / rows), ``selected[j][l]`` (row ids, by
    descending importance) and ``zbar[j][l]`` (the normaliser the level's
    importance used, per row); for a full run also O_full [B,H,N,d]."""
    Q = np.asarray(Q, dtype=np.float64)
    cb = np.asarray(codebook, dtype=np.float64)
    counts = np.asarray(counts)
    vsum = np.asarray(vsum, dtype=np.float64)
    B, H, N, d = Q.shape
    offs = level_offsets(M0, C, L)
    Ps = _p_levels(P, L)
    ntiles = (N + T - 1) // T
    ids = np.arange(B * H * ntiles) if tile_ids is None else np.asarray(tile_ids)
    O = np.zeros((ids.size, T, d))
    cands_all, score_all, sel_all, z_all = [], [], [], []
    for j, g in enumerate(ids):
        bh, t = divmod(int(g), ntiles)
        b, h = divmod(bh, H)
        i0, i1 = t * T, min(N, (t + 1) * T)
        q = Q[b, h, i0:i1]
        rows = i1 - i0
        n = counts[b, h].astype(np.float64)
        vs = vsum[b, h]
        c = cb[h]
        S0 = scale * (q @ c[:M0].T)
        live = n[:M0] > 0
        m = np.where(live[None, :], S0, -np.inf).max(axis=1)
        A0 = np.where(live[None, :], np.exp(S0 - m[:, None]), 0.0)
        Z = A0 @ n[:M0]
        X = A0 @ vs[:M0]
        cand = np.arange(M0)                          # level-0 row ids
        cA = A0
        lc, ls, lsel, lz = [], [], [], []
        for l in range(L - 1):
            w = ((cA * n[cand][None, :]) / Z[:, None]).sum(axis=0)
            order = np.lexsort((cand, -w))            # descending w, then lower row id
            chosen = order[:min(Ps[l], cand.size)]
            lc.append(cand.copy())
            ls.append(w / rows)
            lsel.append(cand[chosen].copy())
            lz.append(Z.copy())
            new_ids, new_A = [], []
            for k in chosen:
                f = int(cand[k])
                fl = f - offs[l]                      # index within level l
                ch = offs[l + 1] + fl * C + np.arange(C)
                Sc = scale * (q @ c[ch].T)
                live_c = n[ch] > 0
                Ac = np.where(live_c[None, :], np.exp(Sc - m[:, None]), 0.0)
                dA = np.where(live_c[None, :], Ac - cA[:, [k]], 0.0)
                X = X + dA @ vs[ch]
                Z = Z + dA @ n[ch]
                new_ids.append(ch)
                new_A.append(Ac)
            cand = np.concatenate(new_ids) if new_ids else np.zeros(0, dtype=np.int64)
            cA = np.concatenate(new_A, axis=1) if new_A else np.zeros((rows, 0))
        O[j, :rows] = X / Z[:, None]
        cands_all.append(lc)
        score_all.append(ls)
        sel_all.append(lsel)
        z_all.append(lz)
    out = {"O": O, "candidates": cands_all, "score": score_all, "selected": sel_all, "zbar": z_all}
    if tile_ids is None:
        out["O_full"] = O.reshape(B, H, ntiles * T, d)[:, :, :N, :]
    return out
