"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself: a library argmax over
a matrix product (torch and NumPy both document that ties return the first
maximal index), the hand-worked fixture in tests/golden, brute-force
restatements on tiny maps (tests/_brute.py), a planted-permutation case whose
answer is exact by construction, and invariants that the reciprocal-set
definition implies.
"""

from __future__ import annotations

import itertools
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# golden fixture
# ---------------------------------------------------------------------------

def _load_golden(name):
    lines = [ln.strip() for ln in open(os.path.join(GOLDEN, name))
             if ln.strip() and not ln.startswith("#")]
    it = iter(lines)
    fx = {"fast": []}
    for ln in it:
        tok = ln.split()
        if tok[0] in ("image1", "image2"):
            H, W, d = map(int, tok[1:])
            rows = [list(map(int, next(it).split())) for _ in range(H * W)]
            fx[tok[0]] = (H, W, np.array(rows, dtype=np.int8).reshape(H, W, d))
        elif tok[0] == "fast":
            body = ln.split(None, 3)
            sub, mi = int(body[1]), int(body[2])
            parts = [p.split() for p in body[3].split("|")]
            pairs = list(map(int, parts[0][1:]))
            fx["fast"].append(dict(sub=sub, max_iter=mi,
                                   pairs=[tuple(pairs[k:k + 3]) for k in range(0, len(pairs), 3)],
                                   sizes=list(map(int, parts[1][1:])),
                                   first=list(map(int, parts[2][1:]))))
        else:
            fx[tok[0]] = list(map(int, tok[1:]))
    return fx


def test_golden_chain_fixture():
    fx = _load_golden("chain_2x2_1x3_d2.txt")
    H1, W1, m1 = fx["image1"]
    H2, W2, m2 = fx["image2"]
    D1 = m1.reshape(H1 * W1, -1)
    D2 = m2.reshape(H2 * W2, -1)
    r12 = oracle.nn(D1, D2, "i8")
    r21 = oracle.nn(D2, D1, "i8")
    assert r12.idx.tolist() == fx["nn12_idx"]
    assert r12.score.tolist() == fx["nn12_score"]
    assert r21.idx.tolist() == fx["nn21_idx"]
    assert r21.score.tolist() == fx["nn21_score"]
    dm = oracle.dense_mutual(D1, D2, "i8")
    exp = fx["dense"]
    assert [tuple(p) + (int(s),) for p, s in zip(dm.pairs.tolist(), dm.score)] == \
        [tuple(exp[k:k + 3]) for k in range(0, len(exp), 3)]
    for case in fx["fast"]:
        r = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "i8", case["sub"], case["max_iter"])
        got = [(int(u), int(v), int(s)) for (u, v), s in zip(r.pairs.tolist(), r.score)]
        assert got == case["pairs"], case
        assert r.frontier_sizes == case["sizes"], case
        assert r.first_seen == case["first"], case


# ---------------------------------------------------------------------------
# nearest neighbour
# ---------------------------------------------------------------------------

def test_nn_i8_matches_torch_argmax_tiny_config():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    r = oracle.nn(D1, D2, "i8")
    S = torch.matmul(torch.from_numpy(D1).long(), torch.from_numpy(D2).long().T)
    # torch.argmax documents that the first maximal index is returned on ties
    ref = torch.argmax(S, dim=1).numpy()
    assert np.array_equal(r.idx, ref)
    assert np.array_equal(r.score, S.max(dim=1).values.numpy())
    # ties really occur in this workload, so the tie rule is exercised
    assert int((S == S.max(dim=1, keepdim=True).values).sum(dim=1).gt(1).sum()) > 0


def test_nn_i8_matches_numpy_argmax_on_full_size_database():
    p = synth.warped_pair_int8(synth.BASE_SEED + 2)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    rng = np.random.default_rng(7)
    qi = rng.choice(D1.shape[0], size=48, replace=False)
    r = oracle.nn(D1[qi], D2, "i8")
    S = D1[qi].astype(np.float64) @ D2.astype(np.float64).T  # exact: |s| < 2^53
    ref = np.argmax(S, axis=1)  # NumPy: first occurrence on ties
    assert np.array_equal(r.idx, ref)
    assert np.array_equal(r.score, S.max(axis=1).astype(np.int64))


@pytest.mark.parametrize("d,lo,hi", [(1, -1, 1), (2, -1, 1), (3, -2, 2), (24, -1, 1)])
def test_nn_i8_heavy_ties_by_definition(d, lo, hi):
    rng = np.random.default_rng(d * 100 + hi)
    q = rng.integers(lo, hi + 1, size=(40, d)).astype(np.int8)
    db = rng.integers(lo, hi + 1, size=(30, d)).astype(np.int8)
    r = oracle.nn(q, db, "i8", nthreads=2)
    for i in range(q.shape[0]):
        k, s = _brute.nn_by_definition(q[i], db)
        assert (r.idx[i], r.score[i]) == (k, s)


def test_nn_edge_sizes():
    db = np.array([[3, -4]], dtype=np.int8)
    r = oracle.nn(np.zeros((0, 2), dtype=np.int8), db, "i8")
    assert r.idx.shape == (0,)
    r = oracle.nn(np.array([[1, 1], [-1, 0]], dtype=np.int8), db, "i8")
    assert r.idx.tolist() == [0, 0] and r.score.tolist() == [-1, -3]
    # all-zero scores: every candidate ties, index 0 wins
    r = oracle.nn(np.zeros((1, 4), dtype=np.int8), np.ones((9, 4), dtype=np.int8), "i8")
    assert r.idx.tolist() == [0] and r.score.tolist() == [0]
    # extreme int8 values: exact in int64
    q = np.full((1, 64), -128, dtype=np.int8)
    db = np.stack([np.full(64, -128), np.full(64, 127)]).astype(np.int8)
    r = oracle.nn(q, db, "i8")
    assert r.idx.tolist() == [0] and r.score.tolist() == [64 * 128 * 128]


def test_nn_bf16_matches_float64_argmax_and_runner_up():
    p = synth.warped_pair_bf16(synth.BASE_SEED + 4, H=48, W=64)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    r = oracle.nn(D1[:500], D2, "bf16")
    A = synth.bf16_bits_to_f64(D1[:500])
    B = synth.bf16_bits_to_f64(D2)
    S = A @ B.T
    srt = np.sort(S, axis=1)
    assert np.allclose(r.score, srt[:, -1], atol=1e-12, rtol=0)
    assert np.allclose(r.second, srt[:, -2], atol=1e-12, rtol=0)
    gap = srt[:, -1] - srt[:, -2]
    sure = gap > 1e-9
    assert np.array_equal(r.idx[sure], np.argmax(S, axis=1)[sure])
    assert sure.mean() > 0.99


def test_nn_bf16_ties_and_runner_up_on_duplicates():
    one = synth.f64_to_bf16_bits(np.array([1.0, 0.5]))
    db = np.stack([synth.f64_to_bf16_bits(np.array([0.25, 0.0])), one, one])
    r = oracle.nn(one[None, :], db, "bf16")
    assert r.idx.tolist() == [1]
    assert r.score[0] == 1.25 and r.second[0] == 1.25  # tied best: gap 0


def test_bf16_rounding_helper_is_round_to_nearest_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even (1)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.1])
    b = synth.f64_to_bf16_bits(x)
    back = synth.bf16_bits_to_f64(b)
    assert back[0] == 1.0 and back[1] == 1.0 + 2.0 ** -6 and back[2] == -2.5
    assert abs(back[3] - 0.1) <= 2.0 ** -11


# ---------------------------------------------------------------------------
# dense mutual nearest neighbours
# ---------------------------------------------------------------------------

def _tiny_maps(rng, n1, n2, d, lo, hi):
    return (rng.integers(lo, hi + 1, size=(n1, d)).astype(np.int8),
            rng.integers(lo, hi + 1, size=(n2, d)).astype(np.int8))


def test_dense_mutual_matches_quantifier_form_exhaustively():
    rng = np.random.default_rng(11)
    for trial in range(150):
        n1, n2 = int(rng.integers(1, 13)), int(rng.integers(1, 13))
        d = int(rng.integers(1, 4))
        D1, D2 = _tiny_maps(rng, n1, n2, d, -2, 2)
        r = oracle.dense_mutual(D1, D2, "i8", nthreads=1)
        got = [(i, j, int(s)) for (i, j), s in zip(r.pairs.tolist(), r.score)]
        assert got == _brute.mutual_by_quantifiers(D1, D2), trial


def test_dense_mutual_is_symmetric_under_swapping_images():
    p = synth.tiny_permuted_pair(synth.BASE_SEED + 1)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    a = oracle.dense_mutual(D1, D2, "i8")
    b = oracle.dense_mutual(D2, D1, "i8")
    assert sorted(map(tuple, a.pairs.tolist())) == sorted((j, i) for i, j in b.pairs.tolist())
    # at most one partner per pixel on either side
    assert len(set(a.pairs[:, 0])) == len(a.pairs) == len(set(a.pairs[:, 1]))


def test_dense_mutual_recovers_planted_permutation_exactly():
    p = synth.planted_sign_pair(123, H=12, W=16, d=20, c=8)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    r = oracle.dense_mutual(D1, D2, "i8")
    got = set(map(tuple, r.pairs.tolist()))
    planted = {(int(i), int(j)) for j, i in enumerate(p.gt_src) if i >= 0}
    assert planted <= got
    # a planted pair scores the common squared norm c^2 d; nothing else can
    assert all(int(s) == 64 * 20 for (i, j), s in zip(r.pairs.tolist(), r.score) if (i, j) in planted)


# ---------------------------------------------------------------------------
# fast reciprocal matching
# ---------------------------------------------------------------------------

def _fast_vs_walks(m1, m2, sub, max_iter):
    H1, W1, _ = m1.shape
    H2, W2, _ = m2.shape
    D1 = m1.reshape(H1 * W1, -1)
    D2 = m2.reshape(H2 * W2, -1)
    r = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "i8", sub, max_iter, nthreads=1)
    got = {(u, v, int(s)) for (u, v), s in zip(r.pairs.tolist(), r.score)}
    seeds = [y * W1 + x for y in range(0, H1, sub) for x in range(0, W1, sub)]
    exp, info = _brute.walks(seeds, D1, D2, max_iter)
    return r, got, exp, info, D1, D2


def test_fast_matches_per_seed_walks_exhaustively():
    rng = np.random.default_rng(5)
    shapes = [(2, 2), (2, 3), (3, 3), (4, 3), (5, 4), (6, 5)]
    n_cases = 0
    for (H1, W1), (H2, W2) in itertools.product(shapes, shapes[::2]):
        for d in (1, 2, 3):
            m1 = rng.integers(-2, 3, size=(H1, W1, d)).astype(np.int8)
            m2 = rng.integers(-2, 3, size=(H2, W2, d)).astype(np.int8)
            for sub in (1, 2, 3):
                for mi in (1, 2, 64):
                    r, got, exp, info, D1, D2 = _fast_vs_walks(m1, m2, sub, mi)
                    assert got == exp, (H1, W1, H2, W2, d, sub, mi)
                    n_cases += 1
    assert n_cases == 6 * 3 * 3 * 3 * 3


def test_fast_is_subset_of_dense_and_contains_mutual_seeds():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    r = oracle.fast_reciprocal(p.desc1, p.H1, p.W1, p.desc2, p.H2, p.W2, "i8",
                               w.subsample, w.max_iter)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    dm = oracle.dense_mutual(D1, D2, "i8")
    dense = set(map(tuple, dm.pairs.tolist()))
    fast = set(map(tuple, r.pairs.tolist()))
    assert fast <= dense
    seeds = set(oracle.grid_seeds(p.H1, p.W1, w.subsample).tolist())
    assert {(i, j) for i, j in dense if i in seeds} <= fast
    assert len(seeds) == 48
    # scores reported are the exact dot products of the kept pairs
    assert np.array_equal(r.score, oracle.score_of(D1, r.pairs[:, 0], D2, r.pairs[:, 1], "i8"))


def test_walks_terminate_with_monotone_scores():
    rng = np.random.default_rng(3)
    for trial in range(60):
        m1 = rng.integers(-2, 3, size=(5, 6, 2)).astype(np.int8)
        m2 = rng.integers(-2, 3, size=(4, 5, 2)).astype(np.int8)
        D1, D2 = m1.reshape(30, 2), m2.reshape(20, 2)
        big = 30 + 1  # more rounds than pixels: every walk must end
        kept, info = _brute.walks(range(30), D1, D2, big)
        for nodes, scores, fixed in info:
            assert fixed is not None
            assert len(set(nodes)) == len(nodes)  # no cycle
            assert all(a <= b for a, b in zip(scores, scores[1:]))
        r = oracle.fast_reciprocal(m1, 5, 6, m2, 4, 5, "i8", 1, big, nthreads=1)
        dense = oracle.dense_mutual(D1, D2, "i8", nthreads=1)
        # from every pixel, with unbounded rounds, the fast set is the whole mutual set
        assert set(map(tuple, r.pairs.tolist())) == set(map(tuple, dense.pairs.tolist()))


def test_fast_planted_permutation_converges_in_one_round():
    p = synth.planted_sign_pair(99, H=16, W=24, d=20, c=8)
    sub = 4
    r = oracle.fast_reciprocal(p.desc1, 16, 24, p.desc2, 16, 24, "i8", sub, 10)
    seeds = oracle.grid_seeds(16, 24, sub)
    inv = {int(i): j for j, i in enumerate(p.gt_src) if i >= 0}
    got = dict(map(tuple, r.pairs.tolist()))
    for u in seeds.tolist():
        if u in inv:
            assert got[u] == inv[u]
    assert r.frontier_sizes[0] == len(seeds)


def test_fast_first_seen_counts():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    r = oracle.fast_reciprocal(p.desc1, p.H1, p.W1, p.desc2, p.H2, p.W2, "i8", 2, 10)
    assert r.first_seen[0] == r.frontier_sizes[0] == (48 // 2) * (64 // 2)
    assert all(0 <= f <= s for f, s in zip(r.first_seen, r.frontier_sizes))
    assert len(r.frontier_sizes) <= 10


def test_bf16_fast_gap_tracking_on_tiny_pair():
    p = synth.warped_pair_bf16(77, H=24, W=32)
    r = oracle.fast_reciprocal(p.desc1, 24, 32, p.desc2, 24, 32, "bf16", 4, 10, track_gaps=True)
    assert set(r.min_gap) == set(r.pairs[:, 0].tolist())
    assert all(g >= 0 for g in r.min_gap.values())


# ---------------------------------------------------------------------------
# the walk-gap record behind the float tolerance rule
# ---------------------------------------------------------------------------

def _dyadic_pair(rng, H1, W1, H2, W2, d):
    """Integer maps k1, k2 (values in -9..9, read as k/8 by the float types):
    a third of image 2's rows are copies of image-1 rows nudged by one step in
    one coordinate, and some rows repeat, so near-ties and exact ties are
    frequent and walks merge."""
    k1 = rng.integers(-8, 9, size=(H1 * W1, d))
    k2 = rng.integers(-8, 9, size=(H2 * W2, d))
    for j in rng.choice(H2 * W2, size=max(1, (H2 * W2) // 3), replace=False):
        k2[j] = k1[rng.integers(H1 * W1)]
        k2[j, rng.integers(d)] += rng.choice([-1, 1])
    if H1 * W1 > 2:
        k1[rng.integers(H1 * W1)] = k1[rng.integers(H1 * W1)]
    return k1, k2


def _as_bf16(k):
    """Bit patterns of the bfloat16 values k / 8 (exact for |k| <= 9)."""
    return (np.asarray(k, dtype=np.float32) / np.float32(8)).view(np.uint32).__rshift__(16) \
        .astype(np.uint16)


@pytest.mark.parametrize("dtype", ["bf16", "l2"])
def test_walk_gap_record_equals_per_seed_walks(dtype):
    """min_gap[u] = max over the walks that stop at u of the smallest top-2
    margin met on the walk, forward and backward steps included; computed by
    following each seed's walk on its own with exact scores."""
    rng = np.random.default_rng(2024 if dtype == "bf16" else 2025)
    if dtype == "bf16":
        # 64 <q, p> is an integer: exact in the brute force and in the oracle's doubles
        score = _brute.dot
        scale = 64.0
    else:
        # -64 |q - p|^2, exact likewise (float32 coordinates k / 8)
        def score(a, b):
            return -sum((int(x) - int(y)) ** 2 for x, y in zip(a, b))
        scale = 64.0
    merges = backward_decides = finite = 0
    for _ in range(120):
        H1, W1, H2, W2 = (int(x) for x in rng.integers(1, 6, size=4))
        if H1 * W1 < 2 or H2 * W2 < 2:
            continue
        d = int(rng.integers(1, 4))
        k1, k2 = _dyadic_pair(rng, H1, W1, H2, W2, d)
        sub = int(rng.integers(1, 3))
        max_iter = int(rng.choice([1, 2, 3, 10]))
        if dtype == "bf16":
            m1, m2 = _as_bf16(k1), _as_bf16(k2)
        else:
            m1 = (k1.astype(np.float32) / np.float32(8))
            m2 = (k2.astype(np.float32) / np.float32(8))
        r = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, dtype, sub, max_iter,
                                   nthreads=1, track_gaps=True)
        seeds = oracle.grid_seeds(H1, W1, sub).tolist()
        walks = _brute.walk_gaps(seeds, k1.tolist(), k2.tolist(), max_iter, score)
        fwd_only = _brute.walk_gaps(seeds, k1.tolist(), k2.tolist(), max_iter, score,
                                    backward=False)
        assert set(r.min_gap) == set(walks) == set(r.pairs[:, 0].tolist())
        for u, gaps in walks.items():
            want = max(gaps)
            got = r.min_gap[u] * scale
            if want == float("inf"):
                assert got > 1e290
            else:
                assert got == want, (u, got, want, gaps)
                finite += want > 0
            merges += len(set(gaps)) > 1
            backward_decides += max(fwd_only[u]) != want
    # the cases exercise every part of the record: positive finite gaps,
    # walks to one pixel with different gaps (the maximum over walks), and
    # walks whose smallest margin is a backward step's
    assert finite > 20 and merges > 5 and backward_decides > 5, (finite, merges, backward_decides)


# ---------------------------------------------------------------------------
# IEEE half descriptors
# ---------------------------------------------------------------------------

def test_half_widening_is_exact_on_every_finite_pattern():
    lib = oracle._load()
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    got = np.array([lib.oracle_half_to_double(int(b)) for b in bits[finite]])
    assert np.array_equal(got, ref[finite])


def test_nn_f16_matches_float64_argmax_and_runner_up():
    p = synth.warped_pair_bf16(synth.BASE_SEED + 4, H=48, W=64, storage="f16")
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    r = oracle.nn(D1[:400], D2, "f16")
    S = D1[:400].view(np.float16).astype(np.float64) @ D2.view(np.float16).astype(np.float64).T
    srt = np.sort(S, axis=1)
    assert np.allclose(r.score, srt[:, -1], atol=1e-12, rtol=0)
    assert np.allclose(r.second, srt[:, -2], atol=1e-12, rtol=0)
    sure = srt[:, -1] - srt[:, -2] > 1e-9
    assert np.array_equal(r.idx[sure], np.argmax(S, axis=1)[sure])
    assert np.array_equal(oracle.score_of(D1, np.arange(400), D2, r.idx, "f16"), r.score)


def test_nn_long_descriptors_d64_by_definition():
    rng = np.random.default_rng(64)
    q = rng.integers(-2, 3, size=(30, 64)).astype(np.int8)
    db = rng.integers(-2, 3, size=(50, 64)).astype(np.int8)
    r = oracle.nn(q, db, "i8", nthreads=1)
    for i in range(30):
        assert (r.idx[i], r.score[i]) == _brute.nn_by_definition(q[i], db)
