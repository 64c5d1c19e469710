"""Failure path of the kernels' bounded waits, exercised without a GPU fault.

With the wait limit set far below a call's duration (fastnn_set_wait_timeout_ns),
the kernels' own waits -- pipeline stages, accumulators, grid barriers -- run
out: the kernel stops issuing work, drains what is in flight, frees its
tensor memory and returns, and the workspace status reads FASTNN_ERR_TIMEOUT.
The next call, with the default limit, must succeed and match the oracle on
the same device: the context stays usable.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import reciprocal_nearest_neighbours_b200 as fnn
from tests._dev import gpu_pairs, require_cuda, to_dev

pytestmark = pytest.mark.gpu

FASTNN_ERR_TIMEOUT = -5
SHORT_NS = 200


@pytest.fixture(autouse=True)
def _cuda_and_reset():
    require_cuda()
    yield
    fnn.fastnn_set_wait_timeout_ns(0)


def _ws(nbytes=1 << 26):
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda")


def _run_twice(call, check):
    ws = _ws()
    fnn.fastnn_set_wait_timeout_ns(SHORT_NS)
    call(ws)
    torch.cuda.synchronize()
    assert fnn.fastnn_device_status(ws) == FASTNN_ERR_TIMEOUT
    fnn.fastnn_set_wait_timeout_ns(0)
    out = call(ws)
    torch.cuda.synchronize()
    assert fnn.fastnn_device_status(ws) == 0
    check(out)


def test_fast_int8_times_out_then_recovers():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    d1, d2 = to_dev(p.desc1), to_dev(p.desc2)
    ref = oracle.fast_reciprocal(p.desc1, p.H1, p.W1, p.desc2, p.H2, p.W2, "i8", 4, 10)

    def check(out):
        pr, sc = gpu_pairs(out[0], out[1], out[2])
        assert set(map(tuple, pr.tolist())) == set(map(tuple, ref.pairs.tolist()))
    _run_twice(lambda ws: fnn.fastnn_reciprocal(d1, d2, 4, 10, workspace=ws), check)


def test_dense_int8_times_out_then_recovers():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    D1, D2 = p.desc1.reshape(-1, 24), p.desc2.reshape(-1, 24)
    ref = oracle.dense_mutual(D1, D2, "i8")

    def check(out):
        pr, _ = gpu_pairs(out[0], out[1], out[2])
        assert np.array_equal(pr, ref.pairs)
    _run_twice(lambda ws: fnn.fastnn_mutual_dense(to_dev(D1), to_dev(D2), workspace=ws), check)


def test_pointmap_fast_times_out_then_recovers():
    rng = np.random.default_rng(81)
    m1 = rng.integers(-3, 4, size=(40, 48, 3)).astype(np.float32)
    m2 = rng.integers(-3, 4, size=(36, 52, 3)).astype(np.float32)
    d1, d2 = torch.from_numpy(m1).cuda(), torch.from_numpy(m2).cuda()
    ref = oracle.fast_reciprocal(m1, 40, 48, m2, 36, 52, "l2", 4, 10)

    def check(out):
        pr, _ = gpu_pairs(out[0], out[1], out[2])
        assert set(map(tuple, pr.tolist())) == set(map(tuple, ref.pairs.tolist()))
    _run_twice(lambda ws: fnn.fastnn_reciprocal(d1, d2, 4, 10, workspace=ws), check)


def test_pointmap_dense_short_limit_then_exact():
    """A standalone pass may finish before any of its waits runs out (a wait
    suspends until a short copy lands): either status is acceptable for the
    short-limit call, and the next call must be exact."""
    rng = np.random.default_rng(82)
    D1 = rng.integers(-3, 4, size=(1920, 3)).astype(np.float32)
    D2 = rng.integers(-3, 4, size=(1872, 3)).astype(np.float32)
    t1, t2 = torch.from_numpy(D1).cuda(), torch.from_numpy(D2).cuda()
    ws = _ws()
    fnn.fastnn_set_wait_timeout_ns(SHORT_NS)
    fnn.fastnn_mutual_dense(t1, t2, workspace=ws)
    torch.cuda.synchronize()
    assert fnn.fastnn_device_status(ws) in (0, FASTNN_ERR_TIMEOUT)
    fnn.fastnn_set_wait_timeout_ns(0)
    pairs, score, count = fnn.fastnn_mutual_dense(t1, t2, workspace=ws)
    torch.cuda.synchronize()
    assert fnn.fastnn_device_status(ws) == 0
    pr, _ = gpu_pairs(pairs, score, count)
    assert np.array_equal(pr, oracle.dense_mutual(D1, D2, "l2").pairs)


def test_masked_fast_times_out_then_recovers():
    p = synth.warped_pair_int8(83, H=48, W=64)
    c1, c2 = synth.confidence_maps(84, 48, 64, p.gt_src)
    d1, d2 = to_dev(p.desc1), to_dev(p.desc2)
    k1, k2 = oracle.confident(c1, 48 * 64, 2.0), oracle.confident(c2, 48 * 64, 2.0)
    ref = oracle.fast_reciprocal_masked(p.desc1, 48, 64, k1, p.desc2, 48, 64, k2, "i8", 4, 10)
    t1, t2 = torch.from_numpy(c1).cuda(), torch.from_numpy(c2).cuda()

    def check(out):
        pr, _ = gpu_pairs(out[0], out[1], out[2])
        assert set(map(tuple, pr.tolist())) == set(map(tuple, ref.pairs.tolist()))
    _run_twice(lambda ws: fnn.fastnn_reciprocal_masked(d1, d2, 4, 10, conf1=t1, conf2=t2,
                                                       threshold=2.0, workspace=ws), check)
