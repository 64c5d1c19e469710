"""The sharded dense path's GPU steps (one process, one GPU)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from reciprocal_nearest_neighbours_b200 import (fastnn_image_rows, fastnn_mutual_dense,
                                                fastnn_mutual_from_nn, fastnn_nn, parallel)
from tests._dev import require_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def test_mutual_from_nn_matches_definition_with_row_offset():
    rng = np.random.default_rng(0)
    n1_total, n2, i0, n1 = 5000, 3000, 1234, 1700
    nn12 = rng.integers(0, n2, size=n1).astype(np.int32)
    nn21 = rng.integers(0, n1_total, size=n2).astype(np.int32)
    # plant mutual pairs
    for i in rng.choice(n1, size=300, replace=False):
        nn21[nn12[i]] = i0 + i
    score = rng.integers(-1000, 1000, size=n1).astype(np.int32)
    pairs, sc, cnt = fastnn_mutual_from_nn(torch.from_numpy(nn12).cuda(),
                                           torch.from_numpy(score).cuda(), i0,
                                           torch.from_numpy(nn21).cuda(), n1_total)
    n = int(cnt[0])
    i = np.arange(n1)
    keep = nn21[nn12] == i0 + i
    exp = np.stack([i0 + i[keep], nn12[keep]], axis=1)
    assert np.array_equal(pairs[:n].cpu().numpy(), exp)
    assert np.array_equal(sc[:n].cpu().numpy(), score[keep])
    # an empty shard reports zero pairs
    _, _, c0 = fastnn_mutual_from_nn(torch.zeros(0, dtype=torch.int32, device="cuda"), None, 0,
                                     torch.from_numpy(nn21).cuda(), n1_total)
    assert int(c0[0]) == 0


def test_sharded_path_single_rank_equals_dense_kernel():
    w = synth.make_workload("tiny_64x48_d24_i8")
    p = w.pairs[0]
    d1 = to_dev(p.desc1.reshape(-1, 24))
    d2 = to_dev(p.desc2.reshape(-1, 24))
    pairs, scores = parallel.sharded_mutual_dense(d1, d2)
    ref_p, ref_s, ref_c = fastnn_mutual_dense(d1, d2)
    n = int(ref_c[0])
    assert torch.equal(pairs, ref_p[:n]) and torch.equal(scores, ref_s[:n])
    dm = oracle.dense_mutual(p.desc1.reshape(-1, 24), p.desc2.reshape(-1, 24), "i8")
    assert np.array_equal(pairs.cpu().numpy().astype(np.int64), dm.pairs)


def test_image_rows_are_the_sorted_distinct_partners():
    rng = np.random.default_rng(3)
    # The last size exceeds the flag pass's capped grid (each thread takes
    # several groups of four rows) and spans ~2,000 blocks of the list passes.
    for n1, n2 in [(1, 1), (5000, 3000), (3000, 50000), (4097, 4097), (10, 8191),
                   (10_000_003, 8_000_000)]:
        nn12 = rng.integers(-3, n2 + 3, size=n1).astype(np.int32)  # a few out of range
        rows, count = fastnn_image_rows(torch.from_numpy(nn12).cuda(), n2)
        exp = np.unique(nn12[(nn12 >= 0) & (nn12 < n2)])
        assert int(count[0]) == len(exp)
        assert np.array_equal(rows[: len(exp)].cpu().numpy(), exp)
    rows, count = fastnn_image_rows(torch.zeros(0, dtype=torch.int32, device="cuda"), 100)
    assert int(count[0]) == 0


def test_sharded_path_rank_blocks_compose_on_one_gpu():
    """Emulate two ranks' row blocks on one GPU (the collectives become
    concatenations) and check that the concatenated per-rank outputs form the
    dense set, with the backward passes restricted to the image of NN12."""
    m = synth.warped_pair_int8(99, H=48, W=64, d=24)
    D1 = to_dev(m.desc1.reshape(-1, 24))
    D2 = to_dev(m.desc2.reshape(-1, 24))
    n1, n2 = D1.shape[0], D2.shape[0]
    blocks1 = [parallel.shard_bounds(n1, r, 2) for r in range(2)]
    fwd = [fastnn_nn(D1[lo:hi].contiguous(), D2) for lo, hi in blocks1]
    nn12_all = torch.cat([f[0] for f in fwd])
    rows, count = fastnn_image_rows(nn12_all, n2)
    rows = rows[: int(count[0])]
    assert rows.numel() < n2
    blocks2 = [parallel.shard_bounds(rows.numel(), r, 2) for r in range(2)]
    idx21_rows = torch.cat([fastnn_nn(D2.index_select(0, rows[lo:hi].long()).contiguous(), D1)[0]
                            for lo, hi in blocks2])
    nn21 = torch.full((n2,), -1, dtype=torch.int32, device="cuda")
    nn21[rows.long()] = idx21_rows
    out = []
    for (lo, hi), (i12, s12) in zip(blocks1, fwd):
        pr, sc, c = fastnn_mutual_from_nn(i12, s12, lo, nn21, n1)
        out.append(pr[: int(c[0])])
    ref_p, _, ref_c = fastnn_mutual_dense(D1, D2)
    assert torch.equal(torch.cat(out), ref_p[: int(ref_c[0])])
