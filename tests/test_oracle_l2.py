"""Pins for the oracle's pointmap matching (nearest 3D point; no GPU).

What is computed: for float32 points of d <= 3 coordinates, NN(q, DB) =
argmin_k |q - DB_k|^2 with the lowest index on ties, and on top of it the same
dense mutual set and fast reciprocal scheme as for descriptors ("DUSt3R /
MASt3R explained": two pixels match when their predicted 3D points are nearest
neighbours in the shared frame; the fast-matching paragraph).

The pins reach the oracle from outside itself: a k-d tree from SciPy, an exact
identity with the (separately pinned) integer dot-product scan, a hand-worked
fixture, brute force on tiny maps and a noise-free permutation whose answer is
known by construction.
"""

from __future__ import annotations

import itertools
import os

import numpy as np
import pytest

import oracle
import synth
from tests import _brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_pointmap_golden(name="pointmap_line_1x5_1x3.txt"):
    lines = [ln.strip() for ln in open(os.path.join(GOLDEN, name))
             if ln.strip() and not ln.startswith("#")]
    it = iter(lines)
    fx = {"fast": []}
    for ln in it:
        tok = ln.split()
        if tok[0] in ("image1", "image2"):
            H, W, d = map(int, tok[1:])
            rows = [list(map(float, next(it).split())) for _ in range(H * W)]
            fx[tok[0]] = (H, W, np.array(rows, dtype=np.float32).reshape(H, W, d))
        elif tok[0] == "fast":
            sub, mi = int(tok[1]), int(tok[2])
            parts = [p.split() for p in ln.split(None, 3)[3].split("|")]
            vals = parts[0][1:]
            fx["fast"].append(dict(
                sub=sub, max_iter=mi,
                pairs=[(int(vals[k]), int(vals[k + 1]), float(vals[k + 2]))
                       for k in range(0, len(vals), 3)],
                sizes=list(map(int, parts[1][1:])), first=list(map(int, parts[2][1:]))))
        else:
            vals = tok[1:]
            fx[tok[0]] = [(int(vals[k]), int(vals[k + 1]), float(vals[k + 2]))
                          for k in range(0, len(vals), 3)] if tok[0] == "dense" else \
                [(int(vals[k]), float(vals[k + 1])) for k in range(0, len(vals), 2)]
    return fx


def test_golden_pointmap_fixture():
    fx = load_pointmap_golden()
    _, W1, m1 = fx["image1"]
    _, W2, m2 = fx["image2"]
    D1, D2 = m1.reshape(-1, 3), m2.reshape(-1, 3)
    r12 = oracle.nn(D1, D2, "l2")
    r21 = oracle.nn(D2, D1, "l2")
    assert list(zip(r12.idx.tolist(), r12.score.tolist())) == fx["nn12"]
    assert list(zip(r21.idx.tolist(), r21.score.tolist())) == fx["nn21"]
    dm = oracle.dense_mutual(D1, D2, "l2")
    assert [(i, j, s) for (i, j), s in zip(dm.pairs.tolist(), dm.score.tolist())] == fx["dense"]
    for case in fx["fast"]:
        r = oracle.fast_reciprocal(m1, 1, W1, m2, 1, W2, "l2", case["sub"], case["max_iter"])
        got = [(u, v, s) for (u, v), s in zip(r.pairs.tolist(), r.score.tolist())]
        assert got == case["pairs"], case
        assert r.frontier_sizes == case["sizes"] and r.first_seen == case["first"], case


def test_nn_l2_matches_scipy_kdtree():
    """Continuous random points (ties have probability zero): the nearest
    neighbour and its distance agree with SciPy's k-d tree."""
    from scipy.spatial import cKDTree
    rng = np.random.default_rng(11)
    for d in (1, 2, 3):
        q = rng.uniform(-3, 3, size=(700, d)).astype(np.float32)
        db = rng.uniform(-3, 3, size=(1500, d)).astype(np.float32)
        r = oracle.nn(q, db, "l2")
        dist, idx = cKDTree(db.astype(np.float64)).query(q.astype(np.float64), k=2)
        assert np.array_equal(r.idx, idx[:, 0])
        np.testing.assert_allclose(r.score, dist[:, 0] ** 2, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(r.second, dist[:, 1] ** 2, rtol=1e-12, atol=1e-15)


def test_nn_l2_equals_integer_dot_scan_on_augmented_points():
    """For integer points, |a - b|^2 = |a|^2 - (2<a, b> - |b|^2) exactly, so
    the nearest point is the argmax of the int8 dot product of (2a, -1) with
    (b, |b|^2) -- ties included, since both scans keep the lowest index."""
    rng = np.random.default_rng(12)
    for amp, d in [(1, 3), (2, 3), (5, 3), (3, 2), (6, 1)]:
        a = rng.integers(-amp, amp + 1, size=(400, d))
        b = rng.integers(-amp, amp + 1, size=(300, d))
        qa = np.concatenate([2 * a, -np.ones((400, 1), dtype=np.int64)], axis=1).astype(np.int8)
        da = np.concatenate([b, (b * b).sum(1, keepdims=True)], axis=1).astype(np.int8)
        ri = oracle.nn(qa, da, "i8")
        rl = oracle.nn(a.astype(np.float32), b.astype(np.float32), "l2")
        assert np.array_equal(rl.idx, ri.idx), (amp, d)
        assert np.array_equal(rl.score, (a * a).sum(1) - ri.score), (amp, d)


def test_nn_l2_by_definition_on_tie_heavy_points():
    rng = np.random.default_rng(13)
    for d in (1, 2, 3):
        q = rng.integers(-2, 3, size=(60, d)).astype(np.float32) * 0.25
        db = rng.integers(-2, 3, size=(40, d)).astype(np.float32) * 0.25
        r = oracle.nn(q, db, "l2")
        for i in range(len(q)):
            k, s = _brute.nn_l2_by_definition(q[i], db)
            assert (r.idx[i], r.score[i]) == (k, s)


def test_nn_l2_edge_cases():
    db = np.array([[1.0, 2.0, 3.0]], dtype=np.float32)
    r = oracle.nn(np.zeros((0, 3), dtype=np.float32), db, "l2")
    assert r.idx.shape == (0,)
    r = oracle.nn(np.array([[1.0, 2.0, 3.0], [0.0, 0.0, 0.0]], dtype=np.float32), db, "l2")
    assert r.idx.tolist() == [0, 0] and r.score.tolist() == [0.0, 14.0]
    # identical database points: index 0 wins, runner-up equals the best
    r = oracle.nn(np.ones((1, 3), dtype=np.float32), np.zeros((5, 3), dtype=np.float32), "l2")
    assert r.idx.tolist() == [0] and r.score.tolist() == [3.0] and r.second.tolist() == [3.0]
    # float32 extremes of a pointmap's range stay exact in double
    q = np.array([[1e-3, -250.0, 99.5]], dtype=np.float32)
    db = np.array([[1e-3, -250.0, 99.5], [1e-3, -250.0, 99.75]], dtype=np.float32)
    r = oracle.nn(q, db, "l2")
    assert r.idx.tolist() == [0] and r.score.tolist() == [0.0] and r.second.tolist() == [0.0625]


def test_dense_mutual_l2_matches_quantifier_form():
    """(i, j) is mutual iff j is strictly nearer to i than every k < j and at
    least as near as every k > j, and the same for i in column j."""
    rng = np.random.default_rng(14)
    for trial in range(60):
        n1, n2 = (int(x) for x in rng.integers(1, 12, size=2))
        d = int(rng.integers(1, 4))
        D1 = (rng.integers(-2, 3, size=(n1, d)) * 0.5).astype(np.float32)
        D2 = (rng.integers(-2, 3, size=(n2, d)) * 0.5).astype(np.float32)
        Dm = [[sum((float(a) - float(b)) ** 2 for a, b in zip(D1[i], D2[j])) for j in range(n2)]
              for i in range(n1)]
        exp = []
        for i in range(n1):
            for j in range(n2):
                row = all(Dm[i][j] < Dm[i][k] for k in range(j)) and \
                    all(Dm[i][j] <= Dm[i][k] for k in range(j + 1, n2))
                col = all(Dm[i][j] < Dm[k][j] for k in range(i)) and \
                    all(Dm[i][j] <= Dm[k][j] for k in range(i + 1, n1))
                if row and col:
                    exp.append((i, j, Dm[i][j]))
        dm = oracle.dense_mutual(D1, D2, "l2", nthreads=1)
        got = [(i, j, s) for (i, j), s in zip(dm.pairs.tolist(), dm.score.tolist())]
        assert got == exp, trial


def test_fast_l2_matches_per_seed_walks_and_walks_are_monotone():
    rng = np.random.default_rng(15)
    shapes = [(2, 3), (3, 3), (4, 5), (6, 5)]
    for (H1, W1), (H2, W2) in itertools.product(shapes, shapes[::2]):
        d = int(rng.integers(1, 4))
        m1 = (rng.integers(-2, 3, size=(H1, W1, d)) * 0.5).astype(np.float32)
        m2 = (rng.integers(-2, 3, size=(H2, W2, d)) * 0.5).astype(np.float32)
        D1, D2 = m1.reshape(-1, d), m2.reshape(-1, d)
        for sub in (1, 2, 3):
            for mi in (1, 2, 64):
                r = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "l2", sub, mi, nthreads=1)
                got = {(u, v, s) for (u, v), s in zip(r.pairs.tolist(), r.score.tolist())}
                seeds = [y * W1 + x for y in range(0, H1, sub) for x in range(0, W1, sub)]
                exp, info = _brute.walks(seeds, D1, D2, mi, nn=_brute.nn_l2_by_definition)
                assert got == exp, (H1, W1, H2, W2, d, sub, mi)
        # with unbounded rounds every walk ends, at non-increasing distances
        _, info = _brute.walks(range(H1 * W1), D1, D2, H1 * W1 + 1,
                               nn=_brute.nn_l2_by_definition)
        for nodes, dists, fixed in info:
            assert fixed is not None and len(set(nodes)) == len(nodes)
            assert all(a >= b for a, b in zip(dists, dists[1:]))


def test_fast_l2_noise_free_permutation_is_exact():
    """View 2 = a permutation of view 1's (distinct) points: every pixel's
    nearest point is its own copy at distance 0, so every seed is kept at
    once with its planted partner."""
    rng = np.random.default_rng(16)
    H, W = 24, 32
    p1 = rng.uniform(-2, 2, size=(H * W, 3)).astype(np.float32)
    perm = rng.permutation(H * W)
    p2 = np.empty_like(p1)
    p2[perm] = p1
    r = oracle.fast_reciprocal(p1.reshape(H, W, 3), H, W, p2.reshape(H, W, 3), H, W, "l2", 4, 10)
    seeds = oracle.grid_seeds(H, W, 4)
    assert r.pairs[:, 0].tolist() == sorted(seeds.tolist())
    assert np.array_equal(r.pairs[:, 1], perm[r.pairs[:, 0]])
    assert np.all(r.score == 0.0) and r.frontier_sizes == [len(seeds)]


def test_fast_l2_subset_of_dense_on_the_synthetic_pointmaps():
    p = synth.pointmap_pair(synth.BASE_SEED + 7, H=48, W=64)
    D1, D2 = p.desc1.reshape(-1, 3), p.desc2.reshape(-1, 3)
    r = oracle.fast_reciprocal(p.desc1, 48, 64, p.desc2, 48, 64, "l2", 8, 10, track_gaps=True)
    dm = oracle.dense_mutual(D1, D2, "l2")
    assert set(map(tuple, r.pairs.tolist())) <= set(map(tuple, dm.pairs.tolist()))
    np.testing.assert_array_equal(r.score, oracle.score_of(D1, r.pairs[:, 0], D2, r.pairs[:, 1], "l2"))
    # the margins tracked along the walks are distances: non-negative
    assert all(g >= 0 for g in r.min_gap.values())
    # most kept pairs follow the generator's warp to within a few pixels
    gt = p.gt_src[r.pairs[:, 1]]
    ok = gt >= 0
    near = (np.abs(gt[ok] % 64 - r.pairs[ok, 0] % 64) + np.abs(gt[ok] // 64 - r.pairs[ok, 0] // 64)) <= 4
    assert near.mean() > 0.9


def test_pointmap_generator_is_seeded_and_float32():
    a = synth.pointmap_pair(5, H=8, W=12)
    b = synth.pointmap_pair(5, H=8, W=12)
    assert a.desc1.dtype == np.float32 and a.desc1.shape == (8, 12, 3)
    assert np.array_equal(a.desc1, b.desc1) and np.array_equal(a.desc2, b.desc2)
    assert np.all(a.desc1[..., 2] > 2.0)  # in front of the camera
