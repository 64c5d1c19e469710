"""GPU parity of fastnn_reciprocal (fast reciprocal matching) against the oracle.

int8: the GPU's set of kept pairs and their int32 scores must equal the
oracle's exactly, and its round count must equal the number of rounds whose
frontier holds a pixel never seen before (the oracle's ``first_seen``), since
the GPU drops pixels already visited. bfloat16: the certificate rule in
``check_fast_bf16``.
"""

from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import FastNNError, fastnn_reciprocal
from tests._dev import BF16_TOL, gpu_pairs, require_cuda, to_dev
from tests.test_oracle import _load_golden

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def run_gpu(m1, m2, sub, max_iter, capacity=None, half="bf16"):
    d1 = to_dev(m1, half)
    d2 = to_dev(m2, half)
    pairs, score, count, iters = fastnn_reciprocal(d1, d2, sub, max_iter, capacity=capacity)
    torch.cuda.synchronize()
    return pairs, score, count, iters


def as_set(p, s):
    return {(int(u), int(v), int(x)) for (u, v), x in zip(p.tolist(), s.tolist())}


def expected_rounds(ref: oracle.FastResult) -> int:
    n = 0
    for f in ref.first_seen:
        if f == 0:
            break
        n += 1
    return n


def check_fast_int8(m1, m2, sub, max_iter, b=0, gpu=None):
    H1, W1, _ = m1.shape
    H2, W2, _ = m2.shape
    pairs, score, count, iters = gpu if gpu is not None else run_gpu(m1, m2, sub, max_iter)
    p, s = gpu_pairs(pairs, score, count, b)
    ref = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, "i8", sub, max_iter)
    got = as_set(p, s)
    exp = as_set(ref.pairs, ref.score)
    assert len(got) == len(p), "duplicate pairs in GPU output"
    assert got == exp, (f"gpu-only {sorted(got - exp)[:5]}, oracle-only {sorted(exp - got)[:5]}")
    assert int(iters[b]) == expected_rounds(ref)
    return p, ref


def test_golden_fixture_all_cases():
    fx = _load_golden("chain_2x2_1x3_d2.txt")
    _, _, m1 = fx["image1"]
    _, _, m2 = fx["image2"]
    for case in fx["fast"]:
        pairs, score, count, iters = run_gpu(m1, m2, case["sub"], case["max_iter"])
        p, s = gpu_pairs(pairs, score, count)
        assert as_set(p, s) == set(case["pairs"]), case
        rounds = next((i for i, f in enumerate(case["first"]) if f == 0), len(case["first"]))
        assert int(iters[0]) == rounds, case


def test_tiny_config_exact_and_deterministic():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    g1 = run_gpu(p.desc1, p.desc2, w.subsample, w.max_iter)
    check_fast_int8(p.desc1, p.desc2, w.subsample, w.max_iter, gpu=g1)
    g2 = run_gpu(p.desc1, p.desc2, w.subsample, w.max_iter)
    n = int(g1[2][0])
    assert torch.equal(g1[0][0, :n], g2[0][0, :n])  # same order, not just the same set


@pytest.mark.parametrize("seed", range(24))
def test_random_small_maps(seed):
    rng = np.random.default_rng(seed)
    H1, W1, H2, W2 = (int(x) for x in rng.integers(1, 40, size=4))
    d = int(rng.choice([1, 2, 3, 24, 32]))
    amp = int(rng.choice([1, 2, 8]))
    m1 = rng.integers(-amp, amp + 1, size=(H1, W1, d)).astype(np.int8)
    m2 = rng.integers(-amp, amp + 1, size=(H2, W2, d)).astype(np.int8)
    sub = int(rng.integers(1, 5))
    max_iter = int(rng.choice([1, 2, 3, 10, 255]))
    check_fast_int8(m1, m2, sub, max_iter)


def test_subset_of_dense_and_seed_completeness_tiny():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    gp, _ = check_fast_int8(p.desc1, p.desc2, 2, 10)
    dense = oracle.dense_mutual(p.desc1.reshape(-1, 24), p.desc2.reshape(-1, 24), "i8")
    dset = set(map(tuple, dense.pairs.tolist()))
    assert set(map(tuple, gp.tolist())) <= dset


def test_planted_permutation_recovered():
    m = synth.planted_sign_pair(5, H=32, W=48, d=24, c=8)
    sub = 4
    pairs, score, count, iters = run_gpu(m.desc1, m.desc2, sub, 10)
    p, s = gpu_pairs(pairs, score, count)
    got = dict(map(tuple, p.tolist()))
    inv = {int(i): j for j, i in enumerate(m.gt_src) if i >= 0}
    seeds = oracle.grid_seeds(32, 48, sub).tolist()
    hit = [u for u in seeds if u in inv]
    assert all(got.get(u) == inv[u] for u in hit)
    assert np.all(s[np.isin(p[:, 0], hit)] == 64 * 24)


def test_capacity_below_seed_count_is_rejected():
    m = np.zeros((16, 16, 24), dtype=np.int8)
    with pytest.raises(FastNNError):
        run_gpu(m, m, 4, 10, capacity=15)


def test_pair_512x384_int8_full_size():
    w = synth.make_workload("pair_512x384_d24_i8")
    p = w.pairs[0]
    gp, ref = check_fast_int8(p.desc1, p.desc2, w.subsample, w.max_iter)
    assert len(gp) > 1000
    inl = np.mean([p.gt_src[v] == u for u, v in gp.tolist()])
    assert inl > 0.5  # reported, loosely bounded: most kept pairs follow the warp


def test_batch_pairs_are_independent_and_exact():
    """A reduced batch of 512x288-shaped warped pairs (d = 32, 4-px grid)."""
    pairs_in = [synth.warped_pair_int8(synth.BASE_SEED + 5 + 1000 * b, H=72, W=128, d=32)
                for b in range(3)]
    d1 = np.stack([q.desc1 for q in pairs_in])
    d2 = np.stack([q.desc2 for q in pairs_in])
    g = run_gpu(d1, d2, 4, 15)
    for b in range(3):
        check_fast_int8(pairs_in[b].desc1, pairs_in[b].desc2, 4, 15, b=b, gpu=g)
        gb = run_gpu(pairs_in[b].desc1, pairs_in[b].desc2, 4, 15)
        n = int(g[2][b])
        assert n == int(gb[2][0])
        assert torch.equal(g[0][b, :n], gb[0][0, :n])


@pytest.mark.slow
def test_batch16_512x288_full_size_exact():
    """The 16-pair workload in one call, every pair compared with the oracle
    in full (kept set, scores and round count)."""
    w = synth.make_workload("batch16_512x288_d32_i8")
    d1, d2 = w.stacked()
    assert len(oracle.grid_seeds(288, 512, w.subsample)) == 9216
    g = run_gpu(d1, d2, w.subsample, w.max_iter)
    for b in range(16):
        gp, ref = check_fast_int8(w.pairs[b].desc1, w.pairs[b].desc2, w.subsample, w.max_iter,
                                  b=b, gpu=g)
        assert len(gp) > 1000


def check_fast_bf16(m1, m2, sub, max_iter, gpu=None, tol=BF16_TOL, dtype="bf16"):
    """Certificate rule for float descriptors.

    Each GPU pair (u, v) is approximately reciprocal: the exact best score of
    u's row and of v's column exceed s(u, v) by at most tol, and the reported
    score is within tol of the exact one. Each oracle pair the GPU lacks must
    sit at the end of walks that all pass a near-tie (top-2 gap < tol).
    """
    H1, W1, d = m1.shape
    H2, W2, _ = m2.shape
    pairs, score, count, iters = (gpu if gpu is not None
                                  else run_gpu(m1, m2, sub, max_iter, half=dtype))
    p, s = gpu_pairs(pairs, score, count)
    D1 = m1.reshape(-1, d)
    D2 = m2.reshape(-1, d)
    exact = oracle.score_of(D1, p[:, 0], D2, p[:, 1], dtype)
    assert np.all(np.abs(s - exact) <= tol)
    r12 = oracle.nn(D1[p[:, 0]], D2, dtype)
    r21 = oracle.nn(D2[p[:, 1]], D1, dtype)
    assert np.all(r12.score - exact <= tol) and np.all(r21.score - exact <= tol)
    ref = oracle.fast_reciprocal(m1, H1, W1, m2, H2, W2, dtype, sub, max_iter, track_gaps=True)
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    for u, v in exp - got:
        assert ref.min_gap[u] < tol, (u, v, ref.min_gap[u])
    return len(got ^ exp), len(exp)


def test_bf16_small_maps_certificate():
    for seed in range(4):
        m = synth.warped_pair_bf16(100 + seed, H=48, W=64)
        check_fast_bf16(m.desc1, m.desc2, 4, 10)


def test_pair_512x384_bf16_full_size():
    w = synth.make_workload("pair_512x384_d24_bf16")
    p = w.pairs[0]
    symdiff, n = check_fast_bf16(p.desc1, p.desc2, w.subsample, w.max_iter)
    assert n > 500 and symdiff <= 0.05 * n
