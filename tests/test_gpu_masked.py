"""GPU parity of confidence-masked matching against the oracle.

A pixel takes part iff its confidence is at least the threshold ("MASt3R
dissection", section 5: mask pixels or reject low-confidence matches). The
GPU compacts the kept pixels of each map in pixel order, runs the usual
kernels with per-pair database counts, and maps indices back; int8 and
integer-valued pointmaps must match the oracle exactly (pairs, scores, round
counts), float descriptors follow the tolerance rule of tests/_dev.py.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import (fastnn_mutual_dense, fastnn_mutual_dense_masked,
                                                fastnn_reciprocal, fastnn_reciprocal_masked)
from tests._dev import BF16_TOL, gpu_pairs, require_cuda, to_dev
from tests.test_gpu_reciprocal import expected_rounds

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return torch.from_numpy(a).cuda()
    return to_dev(a)


def run_masked(m1, m2, c1, c2, thr, sub, max_iter):
    pairs, score, count, iters = fastnn_reciprocal_masked(
        dev(m1), dev(m2), sub, max_iter,
        conf1=None if c1 is None else dev(c1.astype(np.float32)),
        conf2=None if c2 is None else dev(c2.astype(np.float32)), threshold=thr)
    torch.cuda.synchronize()
    return pairs, score, count, iters


def check_masked_exact(m1, m2, c1, c2, thr, sub, max_iter, dtype, b=0, gpu=None):
    H1, W1, _ = m1.shape
    H2, W2, _ = m2.shape
    pairs, score, count, iters = gpu if gpu is not None else run_masked(m1, m2, c1, c2, thr, sub,
                                                                      max_iter)
    p, s = gpu_pairs(pairs, score, count, b)
    k1 = oracle.confident(c1, H1 * W1, thr)
    k2 = oracle.confident(c2, H2 * W2, thr)
    ref = oracle.fast_reciprocal_masked(m1, H1, W1, k1, m2, H2, W2, k2, dtype, sub, max_iter)
    got = {(int(u), int(v), float(x)) for (u, v), x in zip(p.tolist(), s.tolist())}
    exp = {(int(u), int(v), float(x)) for (u, v), x in zip(ref.pairs.tolist(), ref.score.tolist())}
    assert len(got) == len(p)
    assert got == exp, (sorted(got - exp)[:5], sorted(exp - got)[:5])
    assert int(iters[b]) == expected_rounds(ref)
    return p, ref


@pytest.mark.parametrize("seed", range(20))
def test_masked_fast_random_small_maps_exact(seed):
    rng = np.random.default_rng(900 + seed)
    H1, W1, H2, W2 = (int(x) for x in rng.integers(1, 40, size=4))
    l2 = seed % 4 == 3
    d = int(rng.integers(1, 4)) if l2 else int(rng.choice([1, 3, 24, 32, 48]))
    amp = int(rng.choice([1, 2, 8]))
    dt = np.float32 if l2 else np.int8
    m1 = rng.integers(-amp, amp + 1, size=(H1, W1, d)).astype(dt)
    m2 = rng.integers(-amp, amp + 1, size=(H2, W2, d)).astype(dt)
    c1 = rng.uniform(0, 1, size=(H1, W1)).astype(np.float32)
    c2 = rng.uniform(0, 1, size=(H2, W2)).astype(np.float32)
    thr = float(rng.choice([0.0, 0.3, 0.7]))
    check_masked_exact(m1, m2, c1, c2, thr, int(rng.integers(1, 5)),
                       int(rng.choice([1, 2, 10, 255])), "l2" if l2 else "i8")


def test_masked_with_no_maps_equals_unmasked():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    a = run_masked(p.desc1, p.desc2, None, None, 0.0, 4, 10)
    b = fastnn_reciprocal(dev(p.desc1), dev(p.desc2), 4, 10)
    n = int(a[2][0])
    assert n == int(b[2][0]) and int(a[3][0]) == int(b[3][0])
    assert torch.equal(a[0][0, :n], b[0][0, :n]) and torch.equal(a[1][0, :n], b[1][0, :n])


def test_masked_all_of_one_image_dropped():
    p = synth.warped_pair_int8(41, H=32, W=48)
    ones = np.ones((32, 48), np.float32)
    zeros = np.zeros((32, 48), np.float32)
    pairs, score, count, iters = run_masked(p.desc1, p.desc2, ones, zeros, 0.5, 4, 10)
    assert int(count[0]) == 0 and int(iters[0]) == 1  # one round from the kept seeds, no match
    pairs, score, count, iters = run_masked(p.desc1, p.desc2, zeros, ones, 0.5, 4, 10)
    assert int(count[0]) == 0 and int(iters[0]) == 0  # no seed
    pairs, score, count = fastnn_mutual_dense_masked(dev(p.desc1.reshape(-1, 24)),
                                                     dev(p.desc2.reshape(-1, 24)),
                                                     conf1=dev(ones), conf2=dev(zeros),
                                                     threshold=0.5)
    assert int(count[0]) == 0


def test_masked_pair_512x384_conf_full_size_exact():
    w = synth.make_workload("pair_512x384_d24_i8_conf")
    p = w.pairs[0]
    c1, c2 = w.extra["conf1"][0], w.extra["conf2"][0]
    thr = w.extra["threshold"]
    gp, ref = check_masked_exact(p.desc1, p.desc2, c1, c2, thr, w.subsample, w.max_iter, "i8")
    assert len(gp) > 1000
    k1 = oracle.confident(c1, p.H1 * p.W1, thr)
    k2 = oracle.confident(c2, p.H2 * p.W2, thr)
    assert np.all(k1[gp[:, 0]]) and np.all(k2[gp[:, 1]])


def test_masked_batch_pairs_independent():
    maps = [synth.warped_pair_int8(950 + b, H=72, W=128, d=32) for b in range(3)]
    confs = [synth.confidence_maps(960 + b, 72, 128, maps[b].gt_src) for b in range(3)]
    d1 = np.stack([m.desc1 for m in maps])
    d2 = np.stack([m.desc2 for m in maps])
    c1 = np.stack([c[0] for c in confs])
    c2 = np.stack([c[1] for c in confs])
    g = run_masked(d1, d2, c1, c2, 2.0, 4, 15)
    for b in range(3):
        check_masked_exact(maps[b].desc1, maps[b].desc2, confs[b][0], confs[b][1], 2.0, 4, 15,
                           "i8", b=b, gpu=g)


def test_masked_pointmaps_exact_on_integer_points():
    rng = np.random.default_rng(970)
    m1 = rng.integers(-3, 4, size=(40, 56, 3)).astype(np.float32)
    m2 = rng.integers(-3, 4, size=(36, 60, 3)).astype(np.float32)
    c1 = rng.uniform(size=(40, 56)).astype(np.float32)
    c2 = rng.uniform(size=(36, 60)).astype(np.float32)
    check_masked_exact(m1, m2, c1, c2, 0.4, 4, 10, "l2")


# ---------------------------------------------------------------- dense

@pytest.mark.parametrize("n1,n2,d,amp,l2", [(1000, 777, 24, 8, False), (2049, 3000, 3, 3, True),
                                            (513, 129, 1, 2, False), (300, 5000, 32, 4, False)])
def test_masked_dense_exact(n1, n2, d, amp, l2):
    rng = np.random.default_rng(n1 + n2 + d)
    dt = np.float32 if l2 else np.int8
    D1 = rng.integers(-amp, amp + 1, size=(n1, d)).astype(dt)
    D2 = rng.integers(-amp, amp + 1, size=(n2, d)).astype(dt)
    c1 = rng.uniform(size=n1).astype(np.float32)
    c2 = rng.uniform(size=n2).astype(np.float32)
    pairs, score, count = fastnn_mutual_dense_masked(dev(D1), dev(D2), conf1=dev(c1),
                                                     conf2=dev(c2), threshold=0.35)
    p, s = gpu_pairs(pairs, score, count)
    ref = oracle.dense_mutual_masked(D1, oracle.confident(c1, n1, 0.35), D2,
                                     oracle.confident(c2, n2, 0.35), "l2" if l2 else "i8")
    assert np.array_equal(p, ref.pairs)
    assert np.array_equal(s.astype(np.float64), ref.score.astype(np.float64))


def test_masked_dense_without_maps_equals_unmasked():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    D1, D2 = dev(p.desc1.reshape(-1, 24)), dev(p.desc2.reshape(-1, 24))
    a = fastnn_mutual_dense_masked(D1, D2)
    b = fastnn_mutual_dense(D1, D2)
    n = int(a[2][0])
    assert n == int(b[2][0]) and torch.equal(a[0][:n], b[0][:n]) and torch.equal(a[1][:n], b[1][:n])


def test_masked_dense_bf16_within_tolerance():
    m = synth.warped_pair_bf16(33, H=48, W=64)
    c1, c2 = synth.confidence_maps(34, 48, 64, m.gt_src)
    D1, D2 = m.desc1.reshape(-1, 24), m.desc2.reshape(-1, 24)
    pairs, score, count = fastnn_mutual_dense_masked(dev(D1), dev(D2), conf1=dev(c1.ravel()),
                                                     conf2=dev(c2.ravel()), threshold=2.0)
    p, s = gpu_pairs(pairs, score, count)
    k1 = oracle.confident(c1, 48 * 64, 2.0)
    k2 = oracle.confident(c2, 48 * 64, 2.0)
    assert np.all(k1[p[:, 0]]) and np.all(k2[p[:, 1]])
    exact = oracle.score_of(D1, p[:, 0], D2, p[:, 1], "bf16")
    assert np.all(np.abs(s - exact) <= BF16_TOL)
    ref = oracle.dense_mutual_masked(D1, k1, D2, k2, "bf16")
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    assert len(got ^ exp) <= 0.05 * max(1, len(exp))


@pytest.mark.parametrize("keep1,keep2", [(False, True), (True, False), (False, False)])
def test_masked_dense_with_an_empty_side(keep1, keep2):
    """No kept pixel on one side: the forward pass has no query or no database
    row, the image of NN12 is empty, and no pair comes out."""
    rng = np.random.default_rng(79)
    D1 = rng.integers(-4, 5, size=(1500, 24)).astype(np.int8)
    D2 = rng.integers(-4, 5, size=(1300, 24)).astype(np.int8)
    c1 = np.full(1500, 1.0 if keep1 else 0.0, np.float32)
    c2 = np.full(1300, 1.0 if keep2 else 0.0, np.float32)
    pairs, score, count = fastnn_mutual_dense_masked(dev(D1), dev(D2), conf1=dev(c1),
                                                     conf2=dev(c2), threshold=0.5)
    assert int(count[0]) == 0
