"""GPU parity of fastnn_mutual_dense (all mutual nearest-neighbour pairs)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import fastnn_mutual_dense, fastnn_reciprocal
from tests._dev import BF16_TOL, gpu_pairs, require_cuda, to_dev
from tests.test_oracle import _load_golden

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def run_dense(D1, D2):
    pairs, score, count = fastnn_mutual_dense(to_dev(D1), to_dev(D2))
    torch.cuda.synchronize()
    return gpu_pairs(pairs, score, count)


def check_dense_int8(D1, D2):
    p, s = run_dense(D1, D2)
    ref = oracle.dense_mutual(D1, D2, "i8")
    assert np.array_equal(p, ref.pairs)  # same pairs, same (ascending) order
    assert np.array_equal(s.astype(np.int64), ref.score)
    return p


def test_golden_fixture():
    fx = _load_golden("chain_2x2_1x3_d2.txt")
    _, _, m1 = fx["image1"]
    _, _, m2 = fx["image2"]
    p, s = run_dense(m1.reshape(-1, 2), m2.reshape(-1, 2))
    exp = fx["dense"]
    assert [(int(a), int(b), int(c)) for (a, b), c in zip(p.tolist(), s.tolist())] == \
        [tuple(exp[k:k + 3]) for k in range(0, len(exp), 3)]


def test_tiny_config_exact():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    got = check_dense_int8(p.desc1.reshape(-1, 24), p.desc2.reshape(-1, 24))
    # the tiny pair's planted correspondences are largely mutual
    assert len(got) > 1000


@pytest.mark.parametrize("n1,n2,d,amp", [(1000, 777, 24, 8), (1, 1, 3, 2), (300, 5000, 7, 1),
                                         (2049, 4095, 32, 16), (513, 129, 1, 3)])
def test_random_ragged_sizes(n1, n2, d, amp):
    rng = np.random.default_rng(n1 + n2 + d)
    D1 = rng.integers(-amp, amp + 1, size=(n1, d)).astype(np.int8)
    D2 = rng.integers(-amp, amp + 1, size=(n2, d)).astype(np.int8)
    check_dense_int8(D1, D2)


def test_bf16_small_within_tolerance():
    m = synth.warped_pair_bf16(31, H=48, W=64)
    D1 = m.desc1.reshape(-1, 24)
    D2 = m.desc2.reshape(-1, 24)
    p, s = run_dense(D1, D2)
    exact = oracle.score_of(D1, p[:, 0], D2, p[:, 1], "bf16")
    assert np.all(np.abs(s - exact) <= BF16_TOL)
    ref = oracle.dense_mutual(D1, D2, "bf16")
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    for i, j in got ^ exp:
        # a disagreement needs a near-tie in row i or in the column of its partner
        g12 = ref.nn12.score[i] - ref.nn12.second[i]
        jj = ref.nn12.idx[i]
        g21 = ref.nn21.score[jj] - ref.nn21.second[jj]
        g21b = ref.nn21.score[j] - ref.nn21.second[j]
        assert min(g12, g21, g21b) < BF16_TOL


@pytest.mark.slow
def test_dense_512x384_full_size_exact():
    """The 196,608 x 196,608 workload compared with the oracle in full: the
    same mutual pairs in the same (ascending) order with the same int32
    scores. The oracle runs its two plain scans on every host core."""
    m = synth.make_workload("dense_512x384_d24_i8").pairs[0]
    D1 = m.desc1.reshape(-1, 24)
    D2 = m.desc2.reshape(-1, 24)
    p, s = run_dense(D1, D2)
    ref = oracle.dense_mutual(D1, D2, "i8")
    assert len(ref.pairs) > 10000
    assert np.array_equal(p, ref.pairs)
    assert np.array_equal(s.astype(np.int64), ref.score)
    # the fast scheme on the same maps keeps a subset of the dense set
    fp, fs, fc, _ = fastnn_reciprocal(to_dev(m.desc1), to_dev(m.desc2), 8, 10)
    fast, _ = gpu_pairs(fp, fs, fc)
    assert set(map(tuple, fast.tolist())) <= set(map(tuple, p.tolist()))


def test_backward_pass_on_a_one_row_image():
    """Every forward match is the same dominant row j*: the backward pass runs
    on a one-row list, and the only mutual pair is (NN21(j*), j*)."""
    rng = np.random.default_rng(77)
    D1 = rng.integers(1, 9, size=(3000, 24)).astype(np.int8)
    D2 = rng.integers(-8, 9, size=(2000, 24)).astype(np.int8)
    D2[1234] = 127
    p = check_dense_int8(D1, D2)
    assert len(p) == 1 and int(p[0, 1]) == 1234


def test_backward_pass_on_a_two_row_image_with_ties():
    """Two equal dominant rows: every forward match is the lower one (lowest
    index wins), so the image is that row alone; ties in the backward pass
    keep the lowest image-1 index."""
    rng = np.random.default_rng(78)
    D1 = rng.integers(1, 3, size=(700, 8)).astype(np.int8)
    D1[5] = 2
    D1[9] = 2
    D2 = rng.integers(-2, 3, size=(900, 8)).astype(np.int8)
    D2[300] = 100
    D2[600] = 100
    p = check_dense_int8(D1, D2)
    assert p.tolist() == [[5, 300]]
