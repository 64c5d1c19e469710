"""The allocation-free entry point against the workspace entry point (GPU).

fastnn_reciprocal_noalloc serves callers that cannot allocate device memory:
it keeps its scratch in the library's fixed device array instead of a
caller workspace. Its results must be the very same as fastnn_reciprocal's on
the same inputs, call after call, since the array keeps the previous call's
contents. Its status word (a bounded wait that ran out) is read with
fastnn_noalloc_device_status. This file is collected last on purpose.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
import reciprocal_nearest_neighbours_b200 as fnn
from tests._dev import require_cuda, to_dev

pytestmark = pytest.mark.gpu


def _outputs(B, S, dtype, dev):
    return (torch.full((B, S, 2), -7, dtype=torch.int32, device=dev),
            torch.zeros((B, S), dtype=dtype, device=dev),
            torch.full((B,), -7, dtype=torch.int32, device=dev),
            torch.full((B,), -7, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("name", ["tiny_64x48_d24_i8", "pair_512x384_d24_i8",
                                  "pair_512x384_d24_bf16"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    require_cuda()
    w = synth.make_workload(name)
    p = w.pairs[0]
    d1, d2 = to_dev(p.desc1), to_dev(p.desc2)
    S = fnn.seed_count(p.H1, p.W1, w.subsample)
    sdt = torch.int32 if p.dtype == "i8" else torch.float32
    ref_pairs, ref_score, ref_count, ref_iters = fnn.fastnn_reciprocal(d1, d2, w.subsample,
                                                                       w.max_iter)
    torch.cuda.synchronize()
    n = int(ref_count[0])
    assert n > 0
    for _ in range(2):  # the second call starts from the first call's leftovers
        pairs, score, count, iters = _outputs(1, S, sdt, d1.device)
        fnn.fastnn_reciprocal_noalloc(d1, d2, w.subsample, w.max_iter, pairs, score, count, iters)
        torch.cuda.synchronize()
        assert int(count[0]) == n
        assert int(iters[0]) == int(ref_iters[0])
        assert torch.equal(pairs[0, :n], ref_pairs[0, :n])
        assert torch.equal(score[0, :n], ref_score[0, :n])


def test_noalloc_rejects_workloads_beyond_its_scratch():
    require_cuda()
    lib = fnn.library()
    # 16 pairs of 512 x 288 need far more than the fixed scratch array
    need = fnn.fastnn_workspace_size(fnn.FASTNN_OP_RECIPROCAL, 147456, 147456, 32, fnn.FASTNN_I8,
                                     16, 9216)
    assert need > (32 << 20)
    d = torch.zeros((16, 288, 512, 32), dtype=torch.int8, device="cuda")
    pairs, score, count, iters = _outputs(16, 9216, torch.int32, d.device)
    rc = lib.fastnn_reciprocal_noalloc(d.data_ptr(), 288, 512, d.data_ptr(), 288, 512, 32,
                                       fnn.FASTNN_I8, 4, 15, 16, pairs.data_ptr(),
                                       score.data_ptr(), 9216, count.data_ptr(), iters.data_ptr(),
                                       None, None)
    assert rc == -3  # FASTNN_ERR_CAPACITY, nothing enqueued
    assert int(count[0]) == -7


def _reference(w, half):
    p = w.pairs[0]
    d1, d2 = to_dev(p.desc1, half), to_dev(p.desc2, half)
    ws = torch.empty(fnn.fastnn_workspace_size(
        fnn.FASTNN_OP_RECIPROCAL, p.H1 * p.W1, p.H2 * p.W2, p.d,
        fnn.FASTNN_I8 if p.dtype == "i8" else fnn.FASTNN_BF16, 1,
        fnn.seed_count(p.H1, p.W1, w.subsample)), dtype=torch.uint8, device=d1.device)
    ref = fnn.fastnn_reciprocal(d1, d2, w.subsample, w.max_iter, workspace=ws)
    torch.cuda.synchronize()
    return d1, d2, ref


def test_noalloc_after_calls_of_other_shapes_and_types():
    """Each call leaves the shared array holding its own state (repacked maps,
    keys, claims of a different size and layout); the next call, of another
    shape or descriptor type, must still equal fastnn_reciprocal with a
    workspace of its own."""
    require_cuda()
    for name in ["pair_512x384_d24_bf16", "tiny_64x48_d24_i8", "pair_512x384_d24_i8",
                 "tiny_64x48_d24_i8", "pair_512x384_d24_bf16"]:
        w = synth.make_workload(name)
        p = w.pairs[0]
        d1, d2, (rp, rs, rc, ri) = _reference(w, "bf16")
        S = fnn.seed_count(p.H1, p.W1, w.subsample)
        sdt = torch.int32 if p.dtype == "i8" else torch.float32
        pairs, score, count, iters = _outputs(1, S, sdt, d1.device)
        fnn.fastnn_reciprocal_noalloc(d1, d2, w.subsample, w.max_iter, pairs, score, count, iters)
        assert fnn.fastnn_noalloc_device_status() == 0
        n = int(rc[0])
        assert n > 0 and int(count[0]) == n and int(iters[0]) == int(ri[0]), name
        assert torch.equal(pairs[0, :n], rp[0, :n]) and torch.equal(score[0, :n], rs[0, :n]), name


def test_noalloc_timeout_is_readable_then_exact():
    """A wait limit far below the call's duration makes the kernel's bounded
    waits run out: the allocation-free call's status reads
    FASTNN_ERR_TIMEOUT, and the next call (default limit) is exact again."""
    require_cuda()
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    d1, d2, (rp, rs, rc, ri) = _reference(w, "bf16")
    S = fnn.seed_count(p.H1, p.W1, w.subsample)
    try:
        fnn.fastnn_set_wait_timeout_ns(200)
        out = _outputs(1, S, torch.int32, d1.device)
        fnn.fastnn_reciprocal_noalloc(d1, d2, w.subsample, w.max_iter, *out)
        assert fnn.fastnn_noalloc_device_status() == -5  # FASTNN_ERR_TIMEOUT
    finally:
        fnn.fastnn_set_wait_timeout_ns(0)
    pairs, score, count, iters = _outputs(1, S, torch.int32, d1.device)
    fnn.fastnn_reciprocal_noalloc(d1, d2, w.subsample, w.max_iter, pairs, score, count, iters)
    assert fnn.fastnn_noalloc_device_status() == 0
    n = int(rc[0])
    assert int(count[0]) == n and torch.equal(pairs[0, :n], rp[0, :n])
    assert torch.equal(score[0, :n], rs[0, :n])
