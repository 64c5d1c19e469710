"""Pins for the oracle's confidence-masked matching (no GPU).

What is computed: the matching of the other oracle functions restricted to
the pixels whose confidence is at least the threshold -- they alone are
seeds and database candidates ("MASt3R dissection", section 5: mask the
pixels or reject low-confidence matches; "DUSt3R / MASt3R explained": the
per-pixel confidence beside each output).

Pinned against: brute force by definition (nearest neighbour over the kept
rows, walks per seed, the quantifier form of the mutual set), the unmasked
oracle when every pixel is kept, the unmasked oracle run on the compacted
maps with explicit seeds, and the invariants the definition implies.
"""

from __future__ import annotations

import itertools

import numpy as np

import oracle
import synth
from tests import _brute


def _nn_kept_by_definition(keep, l2=False):
    def nn(q, db):
        rows = [(k, row) for k, row in enumerate(db) if keep[k]]
        if l2:
            vals = [(sum((float(a) - float(b)) ** 2 for a, b in zip(q, row)), k) for k, row in rows]
            m = min(v for v, _ in vals)
        else:
            vals = [(-_brute.dot(q, row), k) for k, row in rows]
            m = min(v for v, _ in vals)
        k = min(k for v, k in vals if v == m)
        return k, (m if l2 else -m)
    return nn


def test_confident_threshold_is_inclusive():
    conf = np.array([1.0, 1.9999, 2.0, 5.0], dtype=np.float32)
    assert oracle.confident(conf, 4, 2.0).tolist() == [False, False, True, True]
    assert oracle.confident(None, 3, 2.0).tolist() == [True] * 3


def test_nn_masked_by_definition():
    rng = np.random.default_rng(21)
    for trial in range(40):
        nq, ndb, d = (int(x) for x in rng.integers(1, 30, size=3))
        q = rng.integers(-3, 4, size=(nq, d)).astype(np.int8)
        db = rng.integers(-3, 4, size=(ndb, d)).astype(np.int8)
        keep = rng.uniform(size=ndb) < 0.6
        keep[rng.integers(ndb)] = True
        r = oracle.nn_masked(q, db, keep, "i8")
        f = _nn_kept_by_definition(keep)
        for i in range(nq):
            assert (r.idx[i], r.score[i]) == f(q[i], db), trial
        assert np.all(keep[r.idx])


def test_masked_with_everything_kept_equals_unmasked():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    n1, n2 = p.H1 * p.W1, p.H2 * p.W2
    k1, k2 = np.ones(n1, bool), np.ones(n2, bool)
    a = oracle.fast_reciprocal_masked(p.desc1, p.H1, p.W1, k1, p.desc2, p.H2, p.W2, k2, "i8", 4, 10)
    b = oracle.fast_reciprocal(p.desc1, p.H1, p.W1, p.desc2, p.H2, p.W2, "i8", 4, 10)
    assert np.array_equal(a.pairs, b.pairs) and np.array_equal(a.score, b.score)
    assert a.frontier_sizes == b.frontier_sizes and a.first_seen == b.first_seen
    D1, D2 = p.desc1.reshape(n1, -1), p.desc2.reshape(n2, -1)
    dm = oracle.dense_mutual_masked(D1, k1, D2, k2, "i8")
    du = oracle.dense_mutual(D1, D2, "i8")
    assert np.array_equal(dm.pairs, du.pairs) and np.array_equal(dm.score, du.score)


def test_masked_fast_matches_per_seed_walks_exhaustively():
    rng = np.random.default_rng(22)
    shapes = [(2, 3), (3, 3), (4, 5), (6, 5)]
    n_cases = 0
    for (H1, W1), (H2, W2) in itertools.product(shapes, shapes[::2]):
        for l2 in (False, True):
            d = int(rng.integers(1, 4))
            if l2:
                m1 = (rng.integers(-2, 3, size=(H1, W1, d)) * 0.5).astype(np.float32)
                m2 = (rng.integers(-2, 3, size=(H2, W2, d)) * 0.5).astype(np.float32)
            else:
                m1 = rng.integers(-2, 3, size=(H1, W1, d)).astype(np.int8)
                m2 = rng.integers(-2, 3, size=(H2, W2, d)).astype(np.int8)
            D1, D2 = m1.reshape(-1, d), m2.reshape(-1, d)
            for p_keep in (0.3, 0.7, 1.0):
                k1 = rng.uniform(size=H1 * W1) < p_keep
                k2 = rng.uniform(size=H2 * W2) < p_keep
                k2[rng.integers(H2 * W2)] = True
                for sub, mi in [(1, 64), (2, 2), (3, 1)]:
                    r = oracle.fast_reciprocal_masked(m1, H1, W1, k1, m2, H2, W2, k2,
                                                      "l2" if l2 else "i8", sub, mi, nthreads=1)
                    got = {(u, v, s) for (u, v), s in zip(r.pairs.tolist(), r.score.tolist())}
                    seeds = [y * W1 + x for y in range(0, H1, sub) for x in range(0, W1, sub)
                             if k1[y * W1 + x]]
                    # a walk step searches the other image's kept pixels only
                    nn12 = _nn_kept_by_definition(k2, l2)
                    nn21 = _nn_kept_by_definition(k1, l2)
                    exp = set()
                    for s0 in seeds:
                        u = s0
                        for _ in range(mi):
                            v, sc = nn12(D1[u], D2)
                            u2, _ = nn21(D2[v], D1)
                            if u2 == u:
                                exp.add((u, v, sc))
                                break
                            u = u2
                    assert got == exp, (H1, W1, H2, W2, l2, p_keep, sub, mi)
                    assert all(k1[u] and k2[v] for u, v, _ in got)
                    n_cases += 1
    assert n_cases == 4 * 2 * 2 * 3 * 3


def test_masked_dense_matches_quantifier_form_over_kept_pixels():
    rng = np.random.default_rng(23)
    for trial in range(80):
        n1, n2 = (int(x) for x in rng.integers(1, 14, size=2))
        d = int(rng.integers(1, 4))
        D1 = rng.integers(-2, 3, size=(n1, d)).astype(np.int8)
        D2 = rng.integers(-2, 3, size=(n2, d)).astype(np.int8)
        k1 = rng.uniform(size=n1) < 0.6
        k2 = rng.uniform(size=n2) < 0.6
        dm = oracle.dense_mutual_masked(D1, k1, D2, k2, "i8")
        got = [(i, j, int(s)) for (i, j), s in zip(dm.pairs.tolist(), dm.score.tolist())]
        i_k, j_k = np.nonzero(k1)[0], np.nonzero(k2)[0]
        if i_k.size == 0 or j_k.size == 0:
            assert got == []
            continue
        sub = _brute.mutual_by_quantifiers(D1[i_k], D2[j_k])
        exp = [(int(i_k[i]), int(j_k[j]), s) for i, j, s in sub]
        assert got == exp, trial


def test_masked_fast_equals_unmasked_fast_on_compacted_maps():
    """Masking is the same as matching the compacted maps (kept pixels in
    order) from the kept grid pixels, with indices mapped back."""
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    c1, c2 = synth.confidence_maps(77, p.H1, p.W1, p.gt_src)
    n1, n2 = p.H1 * p.W1, p.H2 * p.W2
    k1, k2 = oracle.confident(c1, n1, 1.8), oracle.confident(c2, n2, 1.8)
    assert 0.3 < k1.mean() < 0.95 and 0.3 < k2.mean() < 0.95
    r = oracle.fast_reciprocal_masked(p.desc1, p.H1, p.W1, k1, p.desc2, p.H2, p.W2, k2, "i8", 4, 10)
    D1, D2 = p.desc1.reshape(n1, -1), p.desc2.reshape(n2, -1)
    i_k, j_k = np.nonzero(k1)[0], np.nonzero(k2)[0]
    pos1 = -np.ones(n1, dtype=np.int64)
    pos1[i_k] = np.arange(i_k.size)
    seeds = [int(pos1[u]) for u in oracle.grid_seeds(p.H1, p.W1, 4) if k1[u]]
    c = oracle.fast_reciprocal(D1[i_k], 1, i_k.size, D2[j_k], 1, j_k.size, "i8", 1, 10,
                               seeds=np.array(seeds, dtype=np.int64))
    mapped = {(int(i_k[u]), int(j_k[v]), int(s)) for (u, v), s in zip(c.pairs.tolist(), c.score)}
    assert mapped == {(u, v, int(s)) for (u, v), s in zip(r.pairs.tolist(), r.score)}
    assert c.frontier_sizes == r.frontier_sizes


def test_masked_fast_is_subset_of_masked_dense_and_avoids_masked_pixels():
    p = synth.warped_pair_int8(31, H=48, W=64)
    c1, c2 = synth.confidence_maps(31, 48, 64, p.gt_src)
    k1 = oracle.confident(c1, 48 * 64, 2.0)
    k2 = oracle.confident(c2, 48 * 64, 2.0)
    r = oracle.fast_reciprocal_masked(p.desc1, 48, 64, k1, p.desc2, 48, 64, k2, "i8", 4, 10)
    D1, D2 = p.desc1.reshape(-1, 24), p.desc2.reshape(-1, 24)
    dm = oracle.dense_mutual_masked(D1, k1, D2, k2, "i8")
    assert set(map(tuple, r.pairs.tolist())) <= set(map(tuple, dm.pairs.tolist()))
    assert np.all(k1[r.pairs[:, 0]]) and np.all(k2[r.pairs[:, 1]])
    assert np.all(k1[dm.pairs[:, 0]]) and np.all(k2[dm.pairs[:, 1]])
    assert len(r.pairs) > 20


def test_everything_masked_gives_nothing():
    p = synth.warped_pair_int8(32, H=16, W=16)
    n = 256
    none, all_ = np.zeros(n, bool), np.ones(n, bool)
    r = oracle.fast_reciprocal_masked(p.desc1, 16, 16, all_, p.desc2, 16, 16, none, "i8", 4, 10)
    assert len(r.pairs) == 0 and r.frontier_sizes == [16]
    r = oracle.fast_reciprocal_masked(p.desc1, 16, 16, none, p.desc2, 16, 16, all_, "i8", 4, 10)
    assert len(r.pairs) == 0 and r.frontier_sizes == []
    D1, D2 = p.desc1.reshape(n, -1), p.desc2.reshape(n, -1)
    assert len(oracle.dense_mutual_masked(D1, all_, D2, none, "i8").pairs) == 0


def test_confidence_generator_is_seeded():
    a = synth.confidence_maps(4, 12, 16)
    b = synth.confidence_maps(4, 12, 16)
    assert a[0].dtype == np.float32 and a[0].shape == (12, 16)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.all(a[0] >= 1.0) and np.all(a[0][:1] <= 1.3)  # sky band
