"""GPU parity of the pointmap path (nearest 3D point; FASTNN_F32_L2).

What the GPU returns, by construction: the nearest point by the fp64
squared distance (dx^2 + dy^2) + dz^2 (the oracle's own expression and
order) rounded to fp32, the lowest index among points whose fp32 values tie;
the score is that fp32 value. (The fp32 scan only preselects; every point its
rounding error could place first is re-ranked this way.) So against the
oracle, which ranks by the fp64 value itself:

* scores equal float32(oracle squared distance) bit for bit;
* an index differs only when two fp64 distances round to the same fp32
  value, and then the GPU's index is the lower one.

Integer-valued points make all arithmetic exact, so there every result must
match the oracle exactly, ties included.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import (fastnn_mutual_dense, fastnn_nn, fastnn_reciprocal,
                                                fastnn_reciprocal_masked)
from tests._dev import gpu_pairs, require_cuda
from tests.test_gpu_reciprocal import expected_rounds
from tests.test_oracle_l2 import load_pointmap_golden

pytestmark = pytest.mark.gpu

# An oracle walk whose top-2 margin is this small may pass an fp32 collision.
COLLISION_GAP = 1e-9


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def check_nn_l2(idx_g, score_g, q, db):
    """Scores are float32 of the fp64 distance of the chosen point; the chosen
    point ties the oracle's in fp32 and is never a higher index."""
    ref = oracle.nn(q, db, "l2")
    idx = idx_g.cpu().numpy().astype(np.int64)
    sc = score_g.cpu().numpy()
    assert np.all((idx >= 0) & (idx < len(db)))
    exact = oracle.score_of(q, np.arange(len(q)), db, idx, "l2")
    assert np.array_equal(sc, f32(exact))
    assert np.array_equal(f32(exact), f32(ref.score))
    diff = idx != ref.idx
    assert np.all(idx[diff] < ref.idx[diff])
    return int(diff.sum())


NN_CASES = [
    # nq, ndb, d
    (1, 1, 3), (5, 3, 3), (300, 1000, 3), (129, 1023, 3), (128, 1024, 3), (200, 1025, 3),
    (1000, 5000, 3), (333, 4099, 2), (700, 2048, 1), (4000, 300, 3),
]


@pytest.mark.parametrize("nq,ndb,d", NN_CASES)
def test_nn_l2_random_points_within_tolerance(nq, ndb, d):
    rng = np.random.default_rng(nq * 7 + ndb + d)
    q = rng.uniform(-3, 3, size=(nq, d)).astype(np.float32)
    db = rng.uniform(-3, 3, size=(ndb, d)).astype(np.float32)
    idx, score = fastnn_nn(dev(q), dev(db))
    torch.cuda.synchronize()
    check_nn_l2(idx, score, q, db)


@pytest.mark.parametrize("nq,ndb,d,amp", [(300, 1000, 3, 2), (700, 2049, 3, 8), (129, 300, 1, 3),
                                          (1000, 1024, 2, 1), (257, 5000, 3, 5)])
def test_nn_l2_integer_points_bit_exact(nq, ndb, d, amp):
    """Small integer coordinates: every fp32 step is exact, ties are massive,
    and the lowest index must win exactly as in the oracle."""
    rng = np.random.default_rng(nq + ndb * 3 + amp)
    q = rng.integers(-amp, amp + 1, size=(nq, d)).astype(np.float32)
    db = rng.integers(-amp, amp + 1, size=(ndb, d)).astype(np.float32)
    idx, score = fastnn_nn(dev(q), dev(db))
    ref = oracle.nn(q, db, "l2")
    assert np.array_equal(idx.cpu().numpy(), ref.idx)
    assert np.array_equal(score.cpu().numpy().astype(np.float64), ref.score)


# Two points whose squared distances from the origin differ in fp64 yet round
# to the same fp32 value (1.0): |p_near|^2 = 0.99999999627..., |p_far|^2 = 1.
P_NEAR = (0.609195351600647, 0.7930201888084412, 0.0)
P_FAR = (1.0, 0.0, 0.0)


@pytest.mark.parametrize("near_first", [False, True])
def test_nn_l2_fp32_collision_ranks_by_the_exact_distance(near_first):
    """The oracle ranks by the fp64 squared distance; two points that collide
    in fp32 must still be told apart by it, whichever index is lower."""
    near, far = np.array(P_NEAR, np.float32), np.array(P_FAR, np.float32)
    d_near = float(np.sum(near.astype(np.float64) ** 2))
    assert d_near < 1.0 and np.float32(d_near) == np.float32(1.0)
    rng = np.random.default_rng(5)
    others = rng.uniform(2.0, 4.0, size=(40, 3)).astype(np.float32)  # all farther away
    db = np.concatenate([[near, far] if near_first else [far, near], others]).astype(np.float32)
    q = np.zeros((3, 3), dtype=np.float32)
    ref = oracle.nn(q, db, "l2")
    expect = 0 if near_first else 1
    assert np.all(ref.idx == expect)
    idx, score = fastnn_nn(dev(q), dev(db))
    assert np.all(idx.cpu().numpy() == expect)
    assert np.all(score.cpu().numpy() == np.float32(1.0))
    # the dense mutual set and the fast scheme take the same (exact) partner
    pairs, _, count = fastnn_mutual_dense(dev(q[:1]), dev(db))
    assert int(count[0]) == 1 and pairs[0].tolist() == [0, expect]
    m1 = q[:1].reshape(1, 1, 3)
    m2 = db.reshape(1, -1, 3)
    fp, fs, fc, _ = fastnn_reciprocal(dev(m1), dev(m2), 1, 10)
    assert int(fc[0]) == 1 and fp[0, 0].tolist() == [0, expect]


def test_nn_l2_identical_database_points_pick_index_zero():
    q = np.full((300, 3), 0.5, dtype=np.float32)
    db = np.ones((3000, 3), dtype=np.float32)
    idx, score = fastnn_nn(dev(q), dev(db))
    assert torch.all(idx == 0) and torch.all(score == 0.75)


def test_nn_l2_full_size_pointmap_sampled_queries():
    p = synth.make_workload("pair_512x384_pts3_f32").pairs[0]
    D1, D2 = p.desc1.reshape(-1, 3), p.desc2.reshape(-1, 3)
    rng = np.random.default_rng(3)
    qi = np.sort(rng.choice(D1.shape[0], size=512, replace=False))
    idx, score = fastnn_nn(dev(D1[qi]), dev(D2))
    assert check_nn_l2(idx, score, D1[qi], D2) == 0


# ---------------------------------------------------------------- fast matching

def run_fast(m1, m2, sub, max_iter):
    pairs, score, count, iters = fastnn_reciprocal(dev(m1), dev(m2), sub, max_iter)
    torch.cuda.synchronize()
    return pairs, score, count, iters


def check_fast_exact(m1, m2, sub, max_iter, b=0, gpu=None):
    H1, W1, _ = m1.shape
    H2, W2, _ = m2.shape
    pairs, score, count, iters = gpu if gpu is not None else run_fast(m1, m2, sub, max_iter)
    p, s = gpu_pairs(pairs, score, count, b)
    ref = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "l2", sub, max_iter)
    got = {(int(u), int(v), float(x)) for (u, v), x in zip(p.tolist(), s.tolist())}
    exp = {(int(u), int(v), float(x)) for (u, v), x in zip(ref.pairs.tolist(), ref.score.tolist())}
    assert len(got) == len(p)
    assert got == exp, (sorted(got - exp)[:5], sorted(exp - got)[:5])
    assert int(iters[b]) == expected_rounds(ref)
    return p


def test_golden_pointmap_fixture():
    fx = load_pointmap_golden()
    _, _, m1 = fx["image1"]
    _, _, m2 = fx["image2"]
    for case in fx["fast"]:
        pairs, score, count, iters = run_fast(m1, m2, case["sub"], case["max_iter"])
        p, s = gpu_pairs(pairs, score, count)
        assert {(u, v, x) for (u, v), x in zip(p.tolist(), s.tolist())} == set(case["pairs"])
        rounds = next((i for i, f in enumerate(case["first"]) if f == 0), len(case["first"]))
        assert int(iters[0]) == rounds
    D1, D2 = m1.reshape(-1, 3), m2.reshape(-1, 3)
    pairs, score, count = fastnn_mutual_dense(dev(D1), dev(D2))
    p, s = gpu_pairs(pairs, score, count)
    assert [(u, v, x) for (u, v), x in zip(p.tolist(), s.tolist())] == fx["dense"]


@pytest.mark.parametrize("seed", range(16))
def test_fast_l2_integer_maps_exact(seed):
    rng = np.random.default_rng(500 + seed)
    H1, W1, H2, W2 = (int(x) for x in rng.integers(1, 48, size=4))
    d = int(rng.integers(1, 4))
    amp = int(rng.choice([1, 2, 4]))
    m1 = rng.integers(-amp, amp + 1, size=(H1, W1, d)).astype(np.float32)
    m2 = rng.integers(-amp, amp + 1, size=(H2, W2, d)).astype(np.float32)
    check_fast_exact(m1, m2, int(rng.integers(1, 5)), int(rng.choice([1, 2, 10, 255])))


def test_fast_l2_noise_free_permutation():
    rng = np.random.default_rng(17)
    H, W = 96, 128
    p1 = rng.uniform(-2, 2, size=(H * W, 3)).astype(np.float32)
    perm = rng.permutation(H * W)
    p2 = np.empty_like(p1)
    p2[perm] = p1
    pairs, score, count, iters = run_fast(p1.reshape(H, W, 3), p2.reshape(H, W, 3), 4, 10)
    p, s = gpu_pairs(pairs, score, count)
    seeds = oracle.grid_seeds(H, W, 4)
    assert sorted(p[:, 0].tolist()) == sorted(seeds.tolist())
    assert np.array_equal(p[:, 1], perm[p[:, 0]]) and np.all(s == 0.0)
    assert int(iters[0]) == 1


def check_fast_l2_certificate(m1, m2, sub, max_iter, gpu=None):
    """Kept pairs and their scores equal the oracle's, except pairs reached
    only through walks that pass an fp32 collision (oracle margin below
    COLLISION_GAP); the GPU round count matches unless such a walk exists."""
    H1, W1, _ = m1.shape
    H2, W2, _ = m2.shape
    pairs, score, count, iters = gpu if gpu is not None else run_fast(m1, m2, sub, max_iter)
    p, s = gpu_pairs(pairs, score, count)
    D1, D2 = m1.reshape(-1, 3), m2.reshape(-1, 3)
    assert np.array_equal(s, f32(oracle.score_of(D1, p[:, 0], D2, p[:, 1], "l2")))
    ref = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "l2", sub, max_iter, track_gaps=True)
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    for u, v in exp - got:
        assert ref.min_gap[u] < COLLISION_GAP, (u, v, ref.min_gap[u])
    for u, v in got - exp:
        # a walk that left the oracle's path at a collision still ends at a
        # pair of mutually nearest points (in fp32)
        d2 = f32(oracle.score_of(D1, np.array([u]), D2, np.array([v]), "l2"))[0]
        assert d2 == f32(oracle.nn(D1[[u]], D2, "l2").score)[0], (u, v)
        assert d2 == f32(oracle.nn(D2[[v]], D1, "l2").score)[0], (u, v)
    if got == exp:
        assert int(iters[0]) == expected_rounds(ref)
    return len(got ^ exp), len(exp)


def test_fast_l2_small_pointmaps_certificate():
    for seed in range(4):
        m = synth.pointmap_pair(600 + seed, H=48, W=64)
        check_fast_l2_certificate(m.desc1, m.desc2, 4, 10)


def test_fast_l2_pair_512x384_full_size():
    w = synth.make_workload("pair_512x384_pts3_f32")
    p = w.pairs[0]
    symdiff, n = check_fast_l2_certificate(p.desc1, p.desc2, w.subsample, w.max_iter)
    assert n > 1000 and symdiff == 0


def test_fast_l2_outlier_free_surfaces_exact():
    """Smooth surfaces without outliers in either view: both passes skip most
    database chunks (their boxes are far from the queries' box by more than
    every bound); the result must still equal the oracle's."""
    for seed in range(3):
        m = synth.pointmap_pair(650 + seed, H=96, W=256, outlier_frac=0.0)
        symdiff, n = check_fast_l2_certificate(m.desc1, m.desc2, 4, 10)
        assert n > 200 and symdiff == 0


@pytest.mark.parametrize("scale,offset", [(1e4, 1e5), (1e-4, 0.0), (3.0, -2e3)])
def test_fast_l2_extreme_scales_exact(scale, offset):
    """Coordinates far from unit scale or far from the origin: the window
    floor and the chunk-skip test keep their margins relative to the
    magnitudes involved, so the result still follows the oracle's."""
    m = synth.pointmap_pair(670, H=64, W=192, outlier_frac=0.1)
    m1 = (m.desc1.astype(np.float64) * scale + offset).astype(np.float32)
    m2 = (m.desc2.astype(np.float64) * scale + offset).astype(np.float32)
    # Any difference from the oracle must sit on an fp32 collision (checked
    # inside); a margin too narrow would show up as a difference elsewhere.
    _, n = check_fast_l2_certificate(m1, m2, 4, 10)
    assert n > 100


def test_fast_l2_outlier_free_surfaces_masked_exact():
    m = synth.pointmap_pair(660, H=96, W=256, outlier_frac=0.0)
    c1, c2 = synth.confidence_maps(661, 96, 256, m.gt_src)
    k1, k2 = oracle.confident(c1, 96 * 256, 2.0), oracle.confident(c2, 96 * 256, 2.0)
    pairs, score, count, iters = fastnn_reciprocal_masked(
        dev(m.desc1), dev(m.desc2), 4, 10, conf1=dev(c1), conf2=dev(c2), threshold=2.0)
    p, s = gpu_pairs(pairs, score, count)
    ref = oracle.fast_reciprocal_masked(m.desc1, 96, 256, k1, m.desc2, 96, 256, k2, "l2", 4, 10)
    assert set(map(tuple, p.tolist())) == set(map(tuple, ref.pairs.tolist()))
    assert len(p) > 100


def test_fast_l2_batch_pairs_independent():
    maps = [synth.pointmap_pair(700 + b, H=72, W=128) for b in range(3)]
    d1 = np.stack([m.desc1 for m in maps])
    d2 = np.stack([m.desc2 for m in maps])
    g = run_fast(d1, d2, 4, 10)
    for b in range(3):
        gb = run_fast(maps[b].desc1, maps[b].desc2, 4, 10)
        n = int(g[2][b])
        assert n == int(gb[2][0]) and n > 100
        assert torch.equal(g[0][b, :n], gb[0][0, :n])
        assert torch.equal(g[1][b, :n], gb[1][0, :n])


# ---------------------------------------------------------------- dense mutual

@pytest.mark.parametrize("n1,n2,d,amp", [(1000, 777, 3, 3), (1, 1, 3, 1), (2049, 3000, 2, 6),
                                         (513, 129, 1, 4)])
def test_dense_l2_integer_points_exact(n1, n2, d, amp):
    rng = np.random.default_rng(n1 * 5 + n2 + d)
    D1 = rng.integers(-amp, amp + 1, size=(n1, d)).astype(np.float32)
    D2 = rng.integers(-amp, amp + 1, size=(n2, d)).astype(np.float32)
    pairs, score, count = fastnn_mutual_dense(dev(D1), dev(D2))
    p, s = gpu_pairs(pairs, score, count)
    ref = oracle.dense_mutual(D1, D2, "l2")
    assert np.array_equal(p, ref.pairs)
    assert np.array_equal(s.astype(np.float64), ref.score)


def test_dense_l2_pointmaps_match_oracle():
    m = synth.pointmap_pair(800, H=48, W=64)
    D1, D2 = m.desc1.reshape(-1, 3), m.desc2.reshape(-1, 3)
    pairs, score, count = fastnn_mutual_dense(dev(D1), dev(D2))
    p, s = gpu_pairs(pairs, score, count)
    assert np.array_equal(s, f32(oracle.score_of(D1, p[:, 0], D2, p[:, 1], "l2")))
    ref = oracle.dense_mutual(D1, D2, "l2")
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    m12 = oracle.margin(ref.nn12, "l2")
    m21 = oracle.margin(ref.nn21, "l2")
    for i, j in got ^ exp:
        jj = ref.nn12.idx[i]
        assert min(m12[i], m21[jj], m21[j]) < COLLISION_GAP
    assert got == exp


def test_dense_l2_full_size_sampled():
    """All 196,608 x 196,608 distances of the full pointmap pair: output
    structure, scores, and the oracle's verdict on sampled pixels."""
    m = synth.make_workload("dense_512x384_pts3_f32").pairs[0]
    D1, D2 = m.desc1.reshape(-1, 3), m.desc2.reshape(-1, 3)
    pairs, score, count = fastnn_mutual_dense(dev(D1), dev(D2))
    p, s = gpu_pairs(pairs, score, count)
    assert len(p) > 10000
    assert np.all(np.diff(p[:, 0]) > 0) and len(np.unique(p[:, 1])) == len(p)
    assert np.array_equal(s, f32(oracle.score_of(D1, p[:, 0], D2, p[:, 1], "l2")))
    rng = np.random.default_rng(6)
    sel = p[rng.choice(len(p), size=300, replace=False)]
    assert np.array_equal(oracle.nn(D1[sel[:, 0]], D2, "l2").idx, sel[:, 1])
    assert np.array_equal(oracle.nn(D2[sel[:, 1]], D1, "l2").idx, sel[:, 0])
    probe = np.sort(rng.choice(D1.shape[0], size=300, replace=False))
    v = oracle.nn(D1[probe], D2, "l2").idx
    back = oracle.nn(D2[v], D1, "l2").idx
    kept = set(p[:, 0].tolist())
    assert all((int(u) in kept) == (int(b) == int(u)) for u, b in zip(probe, back))
