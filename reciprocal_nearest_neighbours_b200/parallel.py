"""Matching across several GPUs: one process per GPU, torch.distributed plumbing.

Two ways the path shards:

* Pair-parallel fast matching (``pair_parallel_reciprocal``). Image pairs are
  independent, so rank r matches a contiguous block of the batch on its own
  GPU; nothing crosses between GPUs on the data path. A round of the fast
  scheme on one pair is tens of microseconds, so one pair is never split:
  replicas only.
* Sharded dense mutual nearest neighbours of one pair
  (``sharded_mutual_dense``). Rank r finds the nearest neighbours of its block
  of image-1 rows against all of image 2 with the tensor-core kernel. A pair
  (i, j) of the reciprocal set has j = NN12(i), so only the image-2 rows that
  some image-1 row matches (the image of NN12) need their own nearest
  neighbour: the forward results are all-gathered (4 bytes per image-1
  pixel), every rank lists that image with the library (ascending, so the
  same list everywhere), and rank r runs the backward pass on its block of
  the list alone -- about half of image 2 on the synthetic pairs, as on one
  GPU. The backward results are all-gathered too (4 bytes per listed row);
  each rank then tests mutuality for its own image-1 rows on its GPU and
  emits them in ascending order, so the concatenation over ranks is the
  dense set.

The compute steps are passed in as callables (defaulting to the CUDA library)
so that the host-side logic -- shard bounds, padding for the collective,
index offsets, ordering -- can be exercised by CPU processes over ``gloo``.
"""

from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def shard_bounds(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous block [lo, hi) of n items owned by ``rank`` of ``world``."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    return n * rank // world, n * (rank + 1) // world


def _rank_world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def all_gather_blocks(local: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """Concatenate the ranks' contiguous blocks (sizes from ``shard_bounds``) of a length-n vector.

    Blocks are padded to the largest block for the collective and trimmed
    after it, so every rank returns the same full vector.
    """
    rank, world = _rank_world(group)
    if world == 1:
        return local
    sizes = [shard_bounds(n, r, world)[1] - shard_bounds(n, r, world)[0] for r in range(world)]
    if local.numel() != sizes[rank]:
        raise ValueError("local block has the wrong size")
    width = max(sizes)
    padded = torch.zeros(width, dtype=local.dtype, device=local.device)
    padded[: local.numel()] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([parts[r][: sizes[r]] for r in range(world)])


def gather_varlen(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather tensors whose first dimension differs between ranks (rank order)."""
    rank, world = _rank_world(group)
    if world == 1:
        return local
    cnt = torch.tensor([local.shape[0]], dtype=torch.int64, device=local.device)
    cnts = [torch.empty_like(cnt) for _ in range(world)]
    dist.all_gather(cnts, cnt, group=group)
    sizes = [int(c.item()) for c in cnts]
    width = max(sizes) if sizes else 0
    shape = (max(width, 1),) + tuple(local.shape[1:])
    padded = torch.zeros(shape, dtype=local.dtype, device=local.device)
    padded[: local.shape[0]] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([parts[r][: sizes[r]] for r in range(world)])


def _default_nn(q, db):
    from . import fastnn_nn
    return fastnn_nn(q, db)


def _default_image(nn12_all, n2):
    from . import fastnn_image_rows
    rows, count = fastnn_image_rows(nn12_all, n2)
    return rows[: int(count[0])]


def _default_emit(nn12, score12, i0, nn21, n1_total):
    from . import fastnn_mutual_from_nn
    pairs, score, count = fastnn_mutual_from_nn(nn12, score12, i0, nn21, n1_total)
    n = int(count[0])
    return pairs[:n], score[:n]


def sharded_mutual_dense(desc1: torch.Tensor, desc2: torch.Tensor, group=None,
                         nn: Callable | None = None, emit: Callable | None = None,
                         image: Callable | None = None, gather: bool = True):
    """Dense mutual nearest-neighbour pairs of one pair, rows split across ranks.

    ``desc1`` [n1, d] and ``desc2`` [n2, d] are the full maps on every rank.
    ``nn(q, db) -> (idx int32, score)``,
    ``image(nn12_all, n2) -> rows`` (ascending image-2 rows named by NN12) and
    ``emit(nn12, score12, i0, nn21, n1_total) -> (pairs, scores)`` default to
    the CUDA library. Returns this rank's pairs (global indices, ascending
    image-1 index), or, with ``gather``, every rank's pairs in rank order --
    which is the whole dense set in ascending image-1 index.
    """
    nn = nn or _default_nn
    emit = emit or _default_emit
    image = image or _default_image
    rank, world = _rank_world(group)
    n1, n2 = desc1.shape[0], desc2.shape[0]
    lo1, hi1 = shard_bounds(n1, rank, world)
    idx12, s12 = nn(desc1[lo1:hi1].contiguous(), desc2)
    idx12_all = all_gather_blocks(idx12, n1, group)  # exchange 1: 4 B per image-1 pixel
    rows = image(idx12_all, n2)  # the same ascending list on every rank
    lo2, hi2 = shard_bounds(rows.numel(), rank, world)
    mine = rows[lo2:hi2]
    if mine.numel() > 0:
        idx21_mine, _ = nn(desc2.index_select(0, mine.long()).contiguous(), desc1)
    else:
        idx21_mine = torch.zeros(0, dtype=torch.int32, device=desc1.device)
    idx21_rows = all_gather_blocks(idx21_mine, rows.numel(), group)  # exchange 2: 4 B per row
    # NN21 of every image-2 row that can be in a pair; -1 (no partner) elsewhere.
    nn21 = torch.full((n2,), -1, dtype=torch.int32, device=desc1.device)
    nn21[rows.long()] = idx21_rows
    pairs, scores = emit(idx12, s12, lo1, nn21, n1)
    if gather:
        pairs = gather_varlen(pairs, group)
        scores = gather_varlen(scores, group)
    return pairs, scores


def _default_match(d1, d2, subsample, max_iter):
    from . import fastnn_reciprocal
    return fastnn_reciprocal(d1, d2, subsample, max_iter)


def pair_parallel_reciprocal(desc1: torch.Tensor, desc2: torch.Tensor, subsample: int,
                             max_iter: int, group=None, match: Callable | None = None):
    """Fast reciprocal matching of a batch of pairs, split by pairs across ranks.

    ``desc1`` [B, H1, W1, d], ``desc2`` [B, H2, W2, d]. Rank r matches pairs
    [lo, hi) with ``match(d1, d2, subsample, max_iter) -> (pairs, score, count,
    iters)`` (default: the CUDA library). No data crosses between ranks.
    Returns (lo, hi, result of match on this rank's block).
    """
    match = match or _default_match
    rank, world = _rank_world(group)
    lo, hi = shard_bounds(desc1.shape[0], rank, world)
    if hi == lo:
        return lo, hi, None
    return lo, hi, match(desc1[lo:hi].contiguous(), desc2[lo:hi].contiguous(), subsample,
                         max_iter)
