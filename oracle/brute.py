"""Pure-Python brute force for tiny AVQ-attention problems.

TEST INFRASTRUCTURE ONLY. This is a second, independent statement of the
method, written per key rather than per codeword, so that it shares neither
code nor algebra with the C oracle:

* assignment takes each key's distances to every codeword of the tree, then
  applies the hierarchical rule (nearest parent; a child of that parent wins
  only when strictly closer, lowest index among equals) -- AVQ-Attention §4.2;
* importance sums, over the tile's queries and over every KEY of a parent,
  that key's softmax share under parent-only attention (no counts, no
  aggregated values) -- §4.3 "Codeword importance";
* each query's output is a softmax over the keys in which key k is
  represented by its leaf codeword when its parent is selected for the
  query's tile and by its parent otherwise -- the meaning of "refine the
  selected parents with their children" (§4.3; papernotes summary, the worked
  example's closing paragraph). No DeltaA correction appears here.

Plain Python floats (fp64) and ``math.exp``; meant for N <= 256, d <= 8.
"""
from __future__ import annotations

import math


def _sqd(a, b):
    return sum((x - y) * (x - y) for x, y in zip(a, b))


def assign_keys(keys, cb, M0, C):
    """keys: list of d-lists; cb: list of Mtot d-lists. Returns (parent, leaf) per key."""
    out = []
    for k in keys:
        dist = [_sqd(k, c) for c in cb]                    # every codeword of the tree
        parent = min(range(M0), key=lambda p: (dist[p], p))
        cands = [(dist[parent], 0, parent)]                # parent first on equal distance
        for c in range(C):
            idx = M0 + parent * C + c
            cands.append((dist[idx], 1 + c, idx))
        leaf = min(cands)[2]
        out.append((parent, leaf))
    return out


def brute_force(Q, K, V, cb, M0, C, P, T, scale):
    """One head. Q, K, V: lists of d-lists (N of them); cb: Mtot d-lists.

    Returns dict(parent, leaf, selected (per tile), score (per tile), O).
    """
    N = len(K)
    pl = assign_keys(K, cb, M0, C)
    parent = [x[0] for x in pl]
    leaf = [x[1] for x in pl]

    def logit(i, j):
        return scale * sum(a * b for a, b in zip(Q[i], cb[j]))

    ntiles = (len(Q) + T - 1) // T
    selected, scores, O = [], [], []
    for t in range(ntiles):
        rows = range(t * T, min((t + 1) * T, len(Q)))
        w = [0.0] * M0
        for i in rows:
            sp = [logit(i, p) for p in range(M0)]
            z_terms = [sp[parent[k]] for k in range(N)]
            m = max(z_terms)
            e = [math.exp(s - m) for s in z_terms]
            z = sum(e)
            for k in range(N):
                w[parent[k]] += e[k] / z
        order = sorted(range(M0), key=lambda p: (-w[p], p))
        sel = set(order[:P])
        selected.append(order[:P])
        scores.append([x / len(rows) for x in w])
        for i in rows:
            s = [logit(i, leaf[k] if parent[k] in sel else parent[k]) for k in range(N)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            O.append([sum(e[k] * V[k][j] for k in range(N)) / z for j in range(len(V[0]))])
    return {"parent": parent, "leaf": leaf, "selected": selected, "score": scores, "O": O}


def deep_paths(keys, cb, M0, C, L):
    """Per key, the list of row ids from its level-0 node down to its leaf in a
    depth-L tree (levels stored one after another; node j of level l has the
    children j*C + c of level l+1): nearest level-0 node, then each level's
    nearest child of the current node while it is strictly closer."""
    offs, acc = [], 0
    for l in range(L):
        offs.append(acc)
        acc += M0 * C ** l
    out = []
    for k in keys:
        dist = [_sqd(k, c) for c in cb]                    # every row of the tree
        local = min(range(M0), key=lambda p: (dist[p], p))
        path = [local]
        for l in range(1, L):
            kids = [offs[l] + local * C + c for c in range(C)]
            best = min(kids, key=lambda r: (dist[r], r))
            if not dist[best] < dist[path[-1]]:
                break
            path.append(best)
            local = best - offs[l]
        out.append(path)
    return out


def brute_force_deep(Q, K, V, cb, M0, C, L, Ps, T, scale):
    """One head, a depth-L tree, Ps[l] nodes expanded at level l.

    Per key rather than per codeword: at every stage of a tile each key is
    represented by one node of its path (its level-0 node at first; the next
    node of its path once the representing node is expanded). A candidate's
    importance sums, over the tile's queries and the keys that reached it,
    their softmax share under the current representation; each query's
    output is a softmax over the keys with the logits of their final
    representing nodes. Returns dict(paths, selected (per tile, per level),
    score (per tile, per level: {row id: importance / rows}), O)."""
    N = len(K)
    paths = deep_paths(K, cb, M0, C, L)

    def logit(i, j):
        return scale * sum(a * b for a, b in zip(Q[i], cb[j]))

    ntiles = (len(Q) + T - 1) // T
    selected, scores, O = [], [], []
    for t in range(ntiles):
        rows = list(range(t * T, min((t + 1) * T, len(Q))))
        depth_rep = [0] * N                                # index into each key's path
        cands = list(range(M0))
        tsel, tscore = [], []
        for l in range(L - 1):
            w = {c: 0.0 for c in cands}
            for i in rows:
                s = [logit(i, paths[k][depth_rep[k]]) for k in range(N)]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                for k in range(N):
                    if len(paths[k]) > l and paths[k][l] in w:
                        w[paths[k][l]] += math.exp(logit(i, paths[k][l]) - m) / z
            order = sorted(cands, key=lambda c: (-w[c], c))
            chosen = order[:Ps[l]]
            tsel.append(chosen)
            tscore.append({c: w[c] / len(rows) for c in cands})
            chosen_set = set(chosen)
            for k in range(N):
                if depth_rep[k] == l and len(paths[k]) > l + 1 and paths[k][l] in chosen_set:
                    depth_rep[k] = l + 1
            offs_next = sum(M0 * C ** x for x in range(l + 1))
            offs_cur = offs_next - M0 * C ** l
            cands = [offs_next + (c - offs_cur) * C + j for c in chosen for j in range(C)]
        selected.append(tsel)
        scores.append(tscore)
        for i in rows:
            s = [logit(i, paths[k][depth_rep[k]]) for k in range(N)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            O.append([sum(e[k] * V[k][j] for k in range(N)) / z for j in range(len(V[0]))])
    return {"paths": paths, "selected": selected, "score": scores, "O": O}
