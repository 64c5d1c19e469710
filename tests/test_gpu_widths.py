"""GPU parity for IEEE-half descriptors and descriptor widths up to d = 64.

Half descriptors (the mixed-precision inference of "Speedy MASt3R", section
HybridCast) run the 16-bit tensor-core path with half operands; their scores
follow the same float tolerance rule as bfloat16 (tests/_dev.py). Widths
33 <= d <= 64 double the repacked row to K = 64 elements (two or four 32-byte
MMA steps per tile, 64- or 128-byte swizzled rows). int8 results stay
bit-exact at every width.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import fastnn_mutual_dense, fastnn_nn
from tests._dev import BF16_TOL, check_nn_bf16, check_nn_exact, gpu_pairs, require_cuda, to_dev
from tests.test_gpu_reciprocal import check_fast_bf16, check_fast_int8, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


WIDE_I8 = [
    # nq, ndb, d, lo, hi
    (300, 1000, 33, -8, 8),
    (129, 2049, 48, -128, 127),
    (1000, 3072, 64, -16, 16),
    (700, 300, 64, -1, 1),       # dense ties: lowest index must win
    (257, 513, 64, -128, 127),   # 64 * 128 * 128: 32-bit epilogue
    (300, 1024, 64, -22, 22),    # 64 * 22 * 22 < 2^15: 16-bit packed epilogue
    (500, 700, 16, -16, 16),
]


@pytest.mark.parametrize("nq,ndb,d,lo,hi", WIDE_I8)
def test_nn_int8_wide_bit_exact(nq, ndb, d, lo, hi):
    rng = np.random.default_rng(nq * 131 + ndb * 7 + d)
    q = rng.integers(lo, hi + 1, size=(nq, d)).astype(np.int8)
    db = rng.integers(lo, hi + 1, size=(ndb, d)).astype(np.int8)
    idx, score = fastnn_nn(to_dev(q), to_dev(db))
    torch.cuda.synchronize()
    check_nn_exact(idx, score, oracle.nn(q, db, "i8"))


FLOAT_CASES = [
    # dtype, nq, ndb, d
    ("f16", 500, 3000, 24), ("f16", 300, 700, 32), ("f16", 100, 257, 5), ("f16", 1, 1, 24),
    ("f16", 129, 1000, 16), ("f16", 300, 2000, 48), ("f16", 257, 1500, 64),
    ("bf16", 300, 2000, 48), ("bf16", 257, 1500, 64), ("bf16", 128, 256, 33),
]


@pytest.mark.parametrize("dtype,nq,ndb,d", FLOAT_CASES)
def test_nn_float_within_tolerance(dtype, nq, ndb, d):
    rng = np.random.default_rng(nq + 3 * ndb + d)
    cvt = synth.f64_to_f16_bits if dtype == "f16" else synth.f64_to_bf16_bits
    q = cvt(_unit(rng, nq, d))
    db = cvt(_unit(rng, ndb, d))
    idx, score = fastnn_nn(to_dev(q, dtype), to_dev(db, dtype))
    ref = oracle.nn(q, db, dtype)
    check_nn_bf16(idx, score, q, db, ref, dtype=dtype)
    sep = (ref.score - ref.second) > 1e-3
    assert np.array_equal(idx.cpu().numpy()[sep], ref.idx[sep])


def test_nn_f16_exact_products_beyond_bf16_precision():
    """Half significands (11 bits) that bfloat16 (8 bits) cannot hold: scores
    of 0.5 * (1 + k / 1024) differ in bits a bf16 path would round away, and
    the fp32 sum of exact half products must still rank them exactly."""
    d = 24
    db = np.zeros((1024, d))
    db[:, 0] = 0.5 * (1.0 + np.arange(1024)[::-1] / 1024.0)  # strictly decreasing
    q = np.zeros((3, d))
    q[:, 0] = 1.0
    qb, dbb = synth.f64_to_f16_bits(q), synth.f64_to_f16_bits(db)
    idx, score = fastnn_nn(to_dev(qb, "f16"), to_dev(dbb, "f16"))
    assert torch.all(idx == 0)
    assert torch.all(score == float(db[0, 0]))
    # the best row removed: the next one wins, by a gap of 2^-11
    idx, score = fastnn_nn(to_dev(qb, "f16"), to_dev(dbb[1:], "f16"))
    assert torch.all(idx == 0) and torch.all(score == float(db[1, 0]))


def test_nn_f16_subnormal_queries():
    """Queries scaled into the half subnormal range (below 2^-14): the
    products stay exact in fp32, so the ranking is that of the exact scores."""
    rng = np.random.default_rng(77)
    d = 32
    qf = _unit(rng, 200, d) * 2.0 ** -16
    q = synth.f64_to_f16_bits(qf)
    db = synth.f64_to_f16_bits(_unit(rng, 1000, d))
    assert np.mean((q & 0x7C00) == 0) > 0.9  # mostly subnormal patterns
    idx, score = fastnn_nn(to_dev(q, "f16"), to_dev(db, "f16"))
    ref = oracle.nn(q, db, "f16")
    check_nn_bf16(idx, score, q, db, ref, tol=BF16_TOL * 2.0 ** -16, dtype="f16")


def test_nn_f16_full_size_database_sampled_queries():
    p = synth.warped_pair_bf16(synth.BASE_SEED + 4, storage="f16")
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    rng = np.random.default_rng(5)
    qi = np.sort(rng.choice(D1.shape[0], size=256, replace=False))
    idx, score = fastnn_nn(to_dev(D1[qi], "f16"), to_dev(D2, "f16"))
    check_nn_bf16(idx, score, D1[qi], D2, oracle.nn(D1[qi], D2, "f16"), dtype="f16")


# ---------------------------------------------------------------- fast matching

@pytest.mark.parametrize("seed", range(8))
def test_fast_int8_wide_random_small_maps(seed):
    rng = np.random.default_rng(1000 + seed)
    H1, W1, H2, W2 = (int(x) for x in rng.integers(1, 40, size=4))
    d = int(rng.choice([16, 33, 48, 64]))
    amp = int(rng.choice([1, 2, 8, 127]))
    m1 = rng.integers(-amp, amp + 1, size=(H1, W1, d)).astype(np.int8)
    m2 = rng.integers(-amp, amp + 1, size=(H2, W2, d)).astype(np.int8)
    check_fast_int8(m1, m2, int(rng.integers(1, 5)), int(rng.choice([1, 3, 10, 255])))


@pytest.mark.parametrize("d", [16, 64])
def test_fast_int8_warped_pair_wide(d):
    p = synth.warped_pair_int8(synth.BASE_SEED + 11 + d, H=96, W=128, d=d)
    gp, _ = check_fast_int8(p.desc1, p.desc2, 4, 10)
    assert len(gp) > 100


def test_fast_f16_small_maps_certificate():
    for seed in range(3):
        m = synth.warped_pair_bf16(200 + seed, H=48, W=64, storage="f16")
        check_fast_bf16(m.desc1, m.desc2, 4, 10, dtype="f16")


def test_fast_bf16_d64_certificate():
    m = synth.warped_pair_bf16(300, H=64, W=96, d=64)
    check_fast_bf16(m.desc1, m.desc2, 4, 10)


def test_fast_f16_pair_512x384_full_size():
    p = synth.warped_pair_bf16(synth.BASE_SEED + 4, storage="f16")
    symdiff, n = check_fast_bf16(p.desc1, p.desc2, 8, 10, dtype="f16")
    assert n > 500 and symdiff <= 0.05 * n


def test_fast_f16_and_bf16_agree_where_separated():
    """The same float maps stored as half and as bfloat16: pairs whose walks
    stay clear of near-ties are kept by both formats."""
    m16 = synth.warped_pair_bf16(400, H=48, W=64, storage="f16")
    mbf = synth.warped_pair_bf16(400, H=48, W=64, storage="bf16")
    a = gpu_pairs(*run_gpu(m16.desc1, m16.desc2, 4, 10, half="f16")[:3])[0]
    b = gpu_pairs(*run_gpu(mbf.desc1, mbf.desc2, 4, 10, half="bf16")[:3])[0]
    sa, sb = set(map(tuple, a.tolist())), set(map(tuple, b.tolist()))
    assert len(sa & sb) >= 0.8 * max(len(sa), len(sb))


# ---------------------------------------------------------------- dense mutual

@pytest.mark.parametrize("n1,n2,d,amp", [(1000, 777, 64, 8), (513, 2049, 48, 127), (300, 300, 33, 1)])
def test_dense_int8_wide_exact(n1, n2, d, amp):
    rng = np.random.default_rng(n1 + n2 * 3 + d)
    D1 = rng.integers(-amp, amp + 1, size=(n1, d)).astype(np.int8)
    D2 = rng.integers(-amp, amp + 1, size=(n2, d)).astype(np.int8)
    pairs, score, count = fastnn_mutual_dense(to_dev(D1), to_dev(D2))
    p, s = gpu_pairs(pairs, score, count)
    ref = oracle.dense_mutual(D1, D2, "i8")
    assert np.array_equal(p, ref.pairs)
    assert np.array_equal(s.astype(np.int64), ref.score)


def test_dense_f16_small_within_tolerance():
    m = synth.warped_pair_bf16(31, H=48, W=64, storage="f16")
    D1 = m.desc1.reshape(-1, 24)
    D2 = m.desc2.reshape(-1, 24)
    pairs, score, count = fastnn_mutual_dense(to_dev(D1, "f16"), to_dev(D2, "f16"))
    p, s = gpu_pairs(pairs, score, count)
    exact = oracle.score_of(D1, p[:, 0], D2, p[:, 1], "f16")
    assert np.all(np.abs(s - exact) <= BF16_TOL)
    ref = oracle.dense_mutual(D1, D2, "f16")
    got = set(map(tuple, p.tolist()))
    exp = set(map(tuple, ref.pairs.tolist()))
    for i, j in got ^ exp:
        g12 = ref.nn12.score[i] - ref.nn12.second[i]
        jj = ref.nn12.idx[i]
        g21 = ref.nn21.score[jj] - ref.nn21.second[jj]
        g21b = ref.nn21.score[j] - ref.nn21.second[j]
        assert min(g12, g21, g21b) < BF16_TOL
