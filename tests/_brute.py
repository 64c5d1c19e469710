"""Brute-force restatements used to pin the oracle (pure Python, tiny inputs).

Each function states the definition in a different form from the oracle's
running scan, so that a slip in one is caught by the other:

* ``nn_by_definition``: the lowest index k whose score equals the row maximum
  (the argmax set first, then its minimum).
* ``mutual_by_quantifiers``: (i, j) is kept iff j beats every k < j strictly
  and ties-or-beats every k > j in row i, and i does the same in column j.
* ``walks``: follows every seed's walk u -> NN21(NN12(u)) on its own, without
  frontiers or sets, and reads the fast scheme's result off the walks.
* ``nn_l2_by_definition``: for pointmaps, the lowest index among the points at
  the minimal squared Euclidean distance (the minimal set first, then its
  minimum index).
"""

from __future__ import annotations


def dot(a, b):
    return sum(int(x) * int(y) for x, y in zip(a, b))


def nn_by_definition(q, db):
    scores = [dot(q, row) for row in db]
    m = max(scores)
    return min(k for k, s in enumerate(scores) if s == m), m


def mutual_by_quantifiers(D1, D2):
    n1, n2 = len(D1), len(D2)
    S = [[dot(D1[i], D2[j]) for j in range(n2)] for i in range(n1)]
    out = []
    for i in range(n1):
        for j in range(n2):
            row_ok = all(S[i][j] > S[i][k] for k in range(j)) and \
                all(S[i][j] >= S[i][k] for k in range(j + 1, n2))
            col_ok = all(S[i][j] > S[k][j] for k in range(i)) and \
                all(S[i][j] >= S[k][j] for k in range(i + 1, n1))
            if row_ok and col_ok:
                out.append((i, j, S[i][j]))
    return out


def nn_l2_by_definition(q, db):
    dist = [sum((float(a) - float(b)) ** 2 for a, b in zip(q, row)) for row in db]
    m = min(dist)
    return min(k for k, s in enumerate(dist) if s == m), m


def walk_step(u, D1, D2, nn=nn_by_definition):
    v, s = nn(D1[u], D2)
    u2, _ = nn(D2[v], D1)
    return v, s, u2


def walks(seeds, D1, D2, max_iter, nn=nn_by_definition):
    """Per-seed walks. Returns (kept set of (u, v, s), list of walks).

    A seed's walk visits u_0 = seed, u_1, ... with u_{t+1} = NN21(NN12(u_t));
    it is kept iff some u_t with t <= max_iter - 1 is a fixed point (it stops
    there). Each walk is returned as (nodes, scores, fixed_or_None).
    """
    kept = set()
    info = []
    for s0 in seeds:
        u = s0
        nodes, scores = [u], []
        fixed = None
        for t in range(max_iter):
            v, s, u2 = walk_step(u, D1, D2, nn)
            scores.append(s)
            if u2 == u:
                fixed = (u, v, s)
                kept.add(fixed)
                break
            u = u2
            nodes.append(u)
        info.append((nodes, scores, fixed))
    return kept, info


def nn_margin_by_definition(q, db, score):
    """Nearest neighbour with its top-2 margin, from the full score list.

    ``score(q, row)`` returns an exact score (higher is better). Returns
    (index, best, margin): the lowest index among the maximal scores, that
    score, and best minus the largest score over every OTHER row (0 on a tie,
    ``inf`` for a one-row database).
    """
    scores = [score(q, row) for row in db]
    m = max(scores)
    k = min(i for i, s in enumerate(scores) if s == m)
    others = [s for i, s in enumerate(scores) if i != k]
    return k, m, (m - max(others)) if others else float("inf")


def walk_gaps(seeds, D1, D2, max_iter, score, backward=True):
    """The walk-gap record of the fast scheme, read off per-seed walks.

    Each seed's walk u_0 = seed, u_{t+1} = NN21(NN12(u_t)) is followed on its
    own for at most ``max_iter`` steps. The gap of a walk is the smallest
    top-2 margin met on it, over the forward step (row u_t against image 2)
    and the backward step (its match against image 1) of every step taken,
    the last (fixed-point) step included (``backward=False`` counts the
    forward steps only, to show which cases the backward margins decide).
    For each pixel u at which some walk stops at a fixed point, the record
    is the LARGEST gap over all walks that stop at u: it is small only when
    every walk to u passes a near-tie. Returns {u: [gap of each walk that
    stops at u]}; the record is the maximum of each list.
    """
    out = {}
    for s0 in seeds:
        u, g = s0, float("inf")
        for _ in range(max_iter):
            v, _, fm = nn_margin_by_definition(D1[u], D2, score)
            u2, _, bm = nn_margin_by_definition(D2[v], D1, score)
            g = min(g, fm, bm) if backward else min(g, fm)
            if u2 == u:
                out.setdefault(u, []).append(g)
                break
            u = u2
    return out
