"""Multi-rank host logic over gloo on the CPU (world sizes 2 and 3).

The compute callables are the CPU oracle (test infrastructure) so that the
sharding, the padded collectives, the index offsets and the output order of
reciprocal_nearest_neighbours_b200.parallel can be checked without GPUs.
"""

from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

from reciprocal_nearest_neighbours_b200.parallel import shard_bounds  # noqa: E402


def test_shard_bounds_cover_every_item_once():
    for n in [0, 1, 5, 7, 100, 3072]:
        for world in [1, 2, 3, 8]:
            seen = []
            for r in range(world):
                lo, hi = shard_bounds(n, r, world)
                assert 0 <= lo <= hi <= n
                seen.extend(range(lo, hi))
                assert hi - lo in (n // world, n // world + 1)
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_nn(q, db):
    import oracle
    r = oracle.nn(q.numpy(), db.numpy(), "i8", nthreads=1)
    return torch.from_numpy(r.idx.copy()), torch.from_numpy(r.score.astype(np.int32))


def _cpu_image(nn12_all, n2):
    v = nn12_all.numpy()
    return torch.from_numpy(np.unique(v[(v >= 0) & (v < n2)]).astype(np.int32))


def _cpu_emit(nn12, score12, i0, nn21, n1_total):
    i = torch.arange(nn12.numel(), dtype=torch.int64) + i0
    keep = nn21[nn12.long()].long() == i
    pairs = torch.stack([i[keep], nn12.long()[keep]], dim=1).to(torch.int32)
    return pairs, score12[keep]


def _worker(rank, world, port, task, out_dir):
    sys.path.insert(0, ROOT)
    import synth
    from reciprocal_nearest_neighbours_b200 import parallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        if task == "dense":
            p = synth.warped_pair_int8(4242, H=24, W=40, d=24)
            d1 = torch.from_numpy(p.desc1.reshape(-1, 24))
            d2 = torch.from_numpy(p.desc2.reshape(-1, 24)[:777])  # n2 != n1, uneven shards
            backward_rows = []

            def nn(q, db):
                if db.shape[0] == d1.shape[0]:  # the backward pass: queries are image-2 rows
                    backward_rows.append(q.shape[0])
                return _oracle_nn(q, db)
            pairs, scores = parallel.sharded_mutual_dense(d1, d2, nn=nn, emit=_cpu_emit,
                                                          image=_cpu_image)
            torch.save((pairs, scores, sum(backward_rows)),
                       os.path.join(out_dir, f"dense_{rank}.pt"))
        else:
            pairs_in = [synth.warped_pair_int8(77 + b, H=16, W=24, d=24) for b in range(5)]
            d1 = torch.from_numpy(np.stack([q.desc1 for q in pairs_in]))
            d2 = torch.from_numpy(np.stack([q.desc2 for q in pairs_in]))

            def match(a, b, sub, mi):
                import oracle
                res = []
                for k in range(a.shape[0]):
                    H1, W1, _ = a[k].shape
                    H2, W2, _ = b[k].shape
                    r = oracle.fast_reciprocal(a[k].numpy(), H1, W1, b[k].numpy(), H2, W2, "i8",
                                               sub, mi, nthreads=1)
                    res.append(r.pairs)
                return res

            lo, hi, res = parallel.pair_parallel_reciprocal(d1, d2, 4, 10, match=match)
            # rank-ordered gather of per-pair counts and the concatenated pairs
            counts = torch.tensor([len(x) for x in (res or [])], dtype=torch.int64)
            flat = torch.from_numpy(np.concatenate(res) if res else np.zeros((0, 2), np.int64))
            all_counts = parallel.gather_varlen(counts)
            all_pairs = parallel.gather_varlen(flat)
            torch.save((lo, hi, all_counts, all_pairs), os.path.join(out_dir, f"pairs_{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_dense_mutual_over_gloo_equals_single_process(world, tmp_path):
    import oracle
    import synth
    mp.start_processes(_worker, args=(world, _free_port(), "dense", str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    p = synth.warped_pair_int8(4242, H=24, W=40, d=24)
    D1 = p.desc1.reshape(-1, 24)
    D2 = p.desc2.reshape(-1, 24)[:777]
    ref = oracle.dense_mutual(D1, D2, "i8")
    backward = 0
    for r in range(world):
        pairs, scores, rows = torch.load(tmp_path / f"dense_{r}.pt")
        assert np.array_equal(pairs.numpy().astype(np.int64), ref.pairs)
        assert np.array_equal(scores.numpy().astype(np.int64), ref.score)
        backward += rows
    assert len(ref.pairs) > 50
    # the backward passes together ran exactly the image of NN12, not all of image 2
    image = np.unique(ref.nn12.idx)
    assert backward == len(image) < D2.shape[0]


def test_pair_parallel_fast_matching_over_gloo(tmp_path):
    import oracle
    import synth
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), "pairs", str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    pairs_in = [synth.warped_pair_int8(77 + b, H=16, W=24, d=24) for b in range(5)]
    refs = [oracle.fast_reciprocal(q.desc1, 16, 24, q.desc2, 16, 24, "i8", 4, 10).pairs
            for q in pairs_in]
    bounds = []
    for r in range(world):
        lo, hi, counts, flat = torch.load(tmp_path / f"pairs_{r}.pt")
        bounds.append((lo, hi))
        assert counts.tolist() == [len(x) for x in refs]
        assert np.array_equal(flat.numpy(), np.concatenate(refs))
    assert bounds == [(0, 2), (2, 5)]
