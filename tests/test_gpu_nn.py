"""GPU parity of fastnn_nn (the tensor-core argmax kernel) against the oracle.

int8 descriptors must match bit for bit (index and int32 score); bfloat16
descriptors follow the tolerance rule in tests/_dev.py. Sizes span several
128-query and 256-row tiles with ragged tails, databases shorter than one
tile, d from 1 to 32, tie-heavy value ranges and extreme int8 values.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import fastnn_nn, fastnn_device_status
from tests._dev import check_nn_bf16, check_nn_exact, require_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


I8_CASES = [
    # nq, ndb, d, lo, hi
    (1, 1, 24, -8, 8),
    (5, 3, 2, -2, 2),
    (300, 1000, 24, -8, 8),
    (129, 257, 7, -3, 3),
    (128, 256, 24, -16, 16),
    (1000, 3072, 32, -16, 16),
    (700, 300, 24, -1, 1),     # dense ties: lowest index must win
    (200, 513, 24, -128, 127),  # extreme int8 values
    (4000, 2000, 1, -5, 5),    # d = 1: massive ties
    (333, 4099, 17, -16, 16),
    (300, 1024, 32, -31, 31),   # 32 * 31 * 31 < 2^15: 16-bit packed epilogue, near its limit
    (300, 1024, 32, -32, 31),   # 32 * 32 * 32 = 2^15: 32-bit epilogue
    (256, 8192, 24, 0, 1),      # non-negative 0/1 values: long runs of equal maxima
]


@pytest.mark.parametrize("nq,ndb,d,lo,hi", I8_CASES)
def test_nn_int8_bit_exact(nq, ndb, d, lo, hi):
    rng = np.random.default_rng(nq * 7919 + ndb * 31 + d)
    q = rng.integers(lo, hi + 1, size=(nq, d)).astype(np.int8)
    db = rng.integers(lo, hi + 1, size=(ndb, d)).astype(np.int8)
    idx, score = fastnn_nn(to_dev(q), to_dev(db))
    torch.cuda.synchronize()
    check_nn_exact(idx, score, oracle.nn(q, db, "i8"))


def test_nn_int8_all_equal_database_picks_index_zero():
    q = np.ones((300, 24), dtype=np.int8)
    db = np.ones((1000, 24), dtype=np.int8)
    idx, score = fastnn_nn(to_dev(q), to_dev(db))
    assert torch.all(idx == 0) and torch.all(score == 24)


def test_nn_int8_full_size_database_sampled_queries():
    p = synth.warped_pair_int8(synth.BASE_SEED + 2)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    rng = np.random.default_rng(1)
    qi = np.sort(rng.choice(D1.shape[0], size=1000, replace=False))
    idx, score = fastnn_nn(to_dev(D1[qi]), to_dev(D2))
    check_nn_exact(idx, score, oracle.nn(D1[qi], D2, "i8"))


def test_nn_int8_deterministic_and_workspace_reuse():
    rng = np.random.default_rng(3)
    q = to_dev(rng.integers(-2, 3, size=(2000, 24)).astype(np.int8))
    db = to_dev(rng.integers(-2, 3, size=(5000, 24)).astype(np.int8))
    i1, s1 = fastnn_nn(q, db)
    ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    i2, s2 = fastnn_nn(q, db, workspace=ws)
    i3, s3 = fastnn_nn(q, db, workspace=ws)
    assert torch.equal(i1, i2) and torch.equal(i2, i3) and torch.equal(s1, s3)
    assert fastnn_device_status(ws) == 0


BF16_CASES = [(500, 3000, 24), (300, 700, 32), (100, 257, 5), (1, 1, 24), (129, 1000, 24)]


@pytest.mark.parametrize("nq,ndb,d", BF16_CASES)
def test_nn_bf16_within_tolerance(nq, ndb, d):
    rng = np.random.default_rng(nq + ndb + d)
    qf = rng.standard_normal((nq, d))
    dbf = rng.standard_normal((ndb, d))
    qf /= np.linalg.norm(qf, axis=1, keepdims=True)
    dbf /= np.linalg.norm(dbf, axis=1, keepdims=True)
    q = synth.f64_to_bf16_bits(qf)
    db = synth.f64_to_bf16_bits(dbf)
    idx, score = fastnn_nn(to_dev(q), to_dev(db))
    ref = oracle.nn(q, db, "bf16")
    check_nn_bf16(idx, score, q, db, ref)
    # with well separated maxima the index must agree exactly
    sep = (ref.score - ref.second) > 1e-3
    assert np.array_equal(idx.cpu().numpy()[sep], ref.idx[sep])


def test_nn_bf16_full_size_database_sampled_queries():
    p = synth.warped_pair_bf16(synth.BASE_SEED + 4)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    rng = np.random.default_rng(2)
    qi = np.sort(rng.choice(D1.shape[0], size=256, replace=False))
    idx, score = fastnn_nn(to_dev(D1[qi]), to_dev(D2))
    check_nn_bf16(idx, score, D1[qi], D2, oracle.nn(D1[qi], D2, "bf16"))


@pytest.mark.parametrize("half", ["bf16", "f16"])
def test_float_dot_products_do_not_depend_on_operand_roles(half):
    """The score of a mutual pair is the same fp32 number whichever map holds
    the queries. The fast scheme's passes start each query at the score it is
    known to reach from the previous pass (computed with the roles swapped),
    lowered by a safety margin; equality here means the margin is never used."""
    p = synth.warped_pair_bf16(synth.BASE_SEED + 9, H=96, W=128)
    D1 = p.desc1.reshape(-1, p.d)
    D2 = p.desc2.reshape(-1, p.d)
    if half == "f16":
        D1 = synth.f64_to_f16_bits(synth.bf16_bits_to_f64(D1))
        D2 = synth.f64_to_f16_bits(synth.bf16_bits_to_f64(D2))
    i12, s12 = fastnn_nn(to_dev(D1, half), to_dev(D2, half))
    i21, s21 = fastnn_nn(to_dev(D2, half), to_dev(D1, half))
    i12, s12 = i12.cpu().numpy(), s12.cpu().numpy()
    i21, s21 = i21.cpu().numpy(), s21.cpu().numpy()
    mutual = np.nonzero(i21[i12] == np.arange(len(i12)))[0]
    assert len(mutual) > 1000
    assert np.array_equal(s12[mutual].view(np.uint32), s21[i12[mutual]].view(np.uint32))
