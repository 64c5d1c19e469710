"""The mutual test and its ordered emit over many blocks of rows.

A block of the count and emit passes covers 4,096 image-1 rows; the emit
places the block's kept pairs at the scanned count of the blocks before it.
These cases span one block, a few with a ragged tail, and almost ten
thousand (more than one 8,192-count tile of the scan), with 16-byte-aligned and unaligned index
and score arrays, integer, float and no scores. The expected output is the
mutual test written out with numpy: row i0 + i is kept with partner
j = nn12[i] iff nn21[j] == i0 + i ("MASt3R dissection", sections 1 and 3), in
ascending i.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from reciprocal_nearest_neighbours_b200 import fastnn_mutual_from_nn
from tests._dev import require_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()


def _smooth_case(seed, n1, n2, i0, n1_total, keep_frac=0.7):
    """A smooth correspondence: row i's partner lies near i (scaled to n2),
    and about keep_frac of the partners point back."""
    rng = np.random.default_rng(seed)
    i = np.arange(n1, dtype=np.int64)
    base = (i * n2) // max(n1, 1)
    nn12 = np.clip(base + rng.integers(-3, 4, size=n1), 0, n2 - 1).astype(np.int32)
    nn21 = rng.integers(0, n1_total, size=n2).astype(np.int32)
    back = rng.random(n1) < keep_frac
    nn21[nn12[back]] = (i0 + i[back]).astype(np.int32)
    return nn12, nn21


def _expected(nn12, nn21, i0, score):
    i = np.arange(nn12.size, dtype=np.int64)
    keep = nn21[nn12] == i0 + i
    pairs = np.stack([i0 + i[keep], nn12[keep].astype(np.int64)], axis=1)
    return pairs, (score[keep] if score is not None else None)


@pytest.mark.parametrize("n1,n2", [(4096, 4096), (3 * 4096 + 517, 9000),
                                   (200_003, 150_001), (40_000_000, 36_000_000)])
def test_many_blocks_match_definition(n1, n2):
    i0 = 1_000 if n1 < 1_000_000 else 0
    n1_total = i0 + n1 + 7
    nn12, nn21 = _smooth_case(n1 % 997, n1, n2, i0, n1_total)
    score = np.random.default_rng(5).integers(-30000, 30000, size=n1).astype(np.int32)
    pairs, sc, cnt = fastnn_mutual_from_nn(torch.from_numpy(nn12).cuda(),
                                           torch.from_numpy(score).cuda(), i0,
                                           torch.from_numpy(nn21).cuda(), n1_total)
    exp_p, exp_s = _expected(nn12, nn21, i0, score)
    n = int(cnt[0])
    assert n == len(exp_p) and n > 0
    assert np.array_equal(pairs[:n].cpu().numpy().astype(np.int64), exp_p)
    assert np.array_equal(sc[:n].cpu().numpy(), exp_s)


@pytest.mark.parametrize("score_kind", ["int", "float", "none"])
def test_unaligned_arrays_and_score_kinds(score_kind):
    """Arrays that start 4 bytes past a 16-byte boundary take the kernel's
    element-wise loads; the output is the same."""
    n1, n2, i0 = 70_001, 66_000, 12
    n1_total = i0 + n1
    nn12, nn21 = _smooth_case(17, n1, n2, i0, n1_total, keep_frac=0.4)
    t12 = torch.empty(n1 + 1, dtype=torch.int32, device="cuda")
    t12[1:] = torch.from_numpy(nn12).cuda()
    nn12_dev = t12[1:]
    assert nn12_dev.data_ptr() % 16 != 0
    if score_kind == "int":
        score = np.arange(n1, dtype=np.int32) * 3 - 5
        ts = torch.empty(n1 + 1, dtype=torch.int32, device="cuda")
    elif score_kind == "float":
        score = (np.arange(n1, dtype=np.float32) * 0.25 - 7.0).astype(np.float32)
        ts = torch.empty(n1 + 1, dtype=torch.float32, device="cuda")
    else:
        score, ts = None, None
    s_dev = None
    if ts is not None:
        ts[1:] = torch.from_numpy(score).cuda()
        s_dev = ts[1:]
    pairs, sc, cnt = fastnn_mutual_from_nn(nn12_dev, s_dev, i0,
                                           torch.from_numpy(nn21).cuda(), n1_total)
    exp_p, exp_s = _expected(nn12, nn21, i0, score)
    n = int(cnt[0])
    assert n == len(exp_p)
    assert np.array_equal(pairs[:n].cpu().numpy().astype(np.int64), exp_p)
    if exp_s is not None:
        assert np.array_equal(sc[:n].cpu().numpy(), exp_s)


def test_no_kept_rows_and_all_kept_rows():
    n = 3 * 4096 + 1
    nn12 = np.arange(n, dtype=np.int32)
    none_back = np.roll(np.arange(n, dtype=np.int32), 1)  # nn21[j] = j - 1: nothing returns
    for nn21, exp_n in [(none_back, 0), (np.arange(n, dtype=np.int32), n)]:
        pairs, _, cnt = fastnn_mutual_from_nn(torch.from_numpy(nn12).cuda(), None, 0,
                                              torch.from_numpy(nn21).cuda(), n)
        assert int(cnt[0]) == exp_n
        if exp_n:
            got = pairs[:exp_n].cpu().numpy()
            assert np.array_equal(got[:, 0], np.arange(n)) and np.array_equal(got[:, 1], np.arange(n))
