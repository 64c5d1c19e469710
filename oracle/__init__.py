"""CPU oracle for reciprocal nearest-neighbour matching (MASt3R).

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product path
(``reciprocal_nearest_neighbours_b200``) never imports it, and this package
imports nothing from the product path. The two share no code: only the seeded
input generators in ``synth`` serve both.

What the oracle computes, step by step, in the pages' order:

* ``nn`` -- the nearest neighbour of each query descriptor in a database by
  dot product, argmax_k <q, DB_k>, lowest index on ties ("MASt3R dissection",
  section 3 Napkin Formula, the inference-time reciprocal matching set). The
  scan itself is the plain C loop in ``oracle.c``. For pointmaps
  (``dtype="l2"``) it is the nearest 3D point, argmin_k |q - DB_k|^2, lowest
  index on ties ("DUSt3R / MASt3R explained": pixels match when their
  predicted 3D points are nearest neighbours in the shared frame).
* ``dense_mutual`` -- the reciprocal (mutual nearest-neighbour) set
  M = {(i, j) : NN(D1[i], D2) = j and NN(D2[j], D1) = i}
  ("MASt3R dissection", section 1 architecture diagram and section 3; "DUSt3R
  / MASt3R explained", the paragraph on fast reciprocal matching, which names
  this the naive all-pixels computation).
* ``fast_reciprocal`` -- MASt3R's fast reciprocal matching ("DUSt3R / MASt3R
  explained", fast-matching paragraph): seeds on a sparse pixel grid of image
  1; each is mapped to its best match in image 2 and that match is mapped back
  to image 1; pixels that return to themselves are kept; the others continue
  from where they landed, for at most ``max_iter`` rounds.

* ``confident`` / ``nn_masked`` / ``dense_mutual_masked`` /
  ``fast_reciprocal_masked`` -- the same matching restricted to confident
  pixels: the network predicts a per-pixel confidence alongside its outputs
  ("DUSt3R / MASt3R explained", the pointmap paragraph), and the remedy for
  pixels whose geometry is not trustworthy is to mask them or reject their
  low-confidence matches ("MASt3R dissection", section 5, hidden
  assumptions). A pixel takes part iff its confidence is at least the
  threshold: it is then a candidate in its image's database and, if on the
  grid, a seed; other pixels are neither.

Readings taken where the pages are silent (each listed in the design notes):
dot-product similarity for unnormalised integer descriptors; lowest index on
ties; grid origin (0, 0) with step ``subsample`` in x and y; convergence means
u' == u; non-converged walks are dropped after ``max_iter`` rounds; the output
is a set, unique by the image-1 pixel.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against things other than itself (a library argmax over a matrix product,
hand-worked fixtures in ``tests/golden``, closed-form special cases, brute
force on tiny maps, and invariants the definition implies).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", "-Wall", "-o", _LIB, _SRC, "-lm"]
        # Portable x86-64 code: the built library travels to other hosts.
        subprocess.run(cmd, check=True, capture_output=True, text=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_nn_i8.argtypes = [P, I64, P, I64, ctypes.c_int, P, P, ctypes.c_int]
        lib.oracle_nn_i8.restype = ctypes.c_int
        lib.oracle_nn_bf16.argtypes = [P, I64, P, I64, ctypes.c_int, P, P, P, ctypes.c_int]
        lib.oracle_nn_bf16.restype = ctypes.c_int
        lib.oracle_nn_f16.argtypes = [P, I64, P, I64, ctypes.c_int, P, P, P, ctypes.c_int]
        lib.oracle_nn_f16.restype = ctypes.c_int
        lib.oracle_nn_l2.argtypes = [P, I64, P, I64, ctypes.c_int, P, P, P, ctypes.c_int]
        lib.oracle_nn_l2.restype = ctypes.c_int
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


@dataclass
class NNResult:
    idx: np.ndarray  # int32 [nq]
    score: np.ndarray  # int64 (int8), float64 (bf16, f16), float64 squared distance (l2) [nq]
    second: np.ndarray | None = None  # float64 runner-up (float types; for l2 the 2nd smallest)


def nn(q: np.ndarray, db: np.ndarray, dtype: str, nthreads: int | None = None) -> NNResult:
    """Nearest neighbour of every row of ``q`` among the rows of ``db``.

    ``q`` is [nq, d], ``db`` is [ndb, d]; int8 arrays for ``dtype == "i8"``,
    uint16 bit patterns of bfloat16 (``"bf16"``) or IEEE half (``"f16"``),
    float32 points with d <= 3 for ``"l2"`` (nearest by Euclidean distance;
    ``score`` is then the squared distance, lower is better).
    """
    lib = _load()
    nthreads = default_threads() if nthreads is None else nthreads
    q = np.ascontiguousarray(q)
    db = np.ascontiguousarray(db)
    nq, d = q.shape
    ndb = db.shape[0]
    assert db.shape[1] == d and ndb > 0
    idx = np.empty(nq, dtype=np.int32)
    if dtype == "i8":
        assert q.dtype == np.int8 and db.dtype == np.int8
        score = np.empty(nq, dtype=np.int64)
        rc = lib.oracle_nn_i8(_ptr(q), nq, _ptr(db), ndb, d, _ptr(idx), _ptr(score), nthreads)
        assert rc == 0
        return NNResult(idx, score)
    if dtype in ("bf16", "f16"):
        assert q.dtype == np.uint16 and db.dtype == np.uint16
        score = np.empty(nq, dtype=np.float64)
        second = np.empty(nq, dtype=np.float64)
        fn = lib.oracle_nn_bf16 if dtype == "bf16" else lib.oracle_nn_f16
        rc = fn(_ptr(q), nq, _ptr(db), ndb, d, _ptr(idx), _ptr(score), _ptr(second), nthreads)
        assert rc == 0
        return NNResult(idx, score, second)
    if dtype == "l2":
        assert q.dtype == np.float32 and db.dtype == np.float32 and d <= 3
        d2 = np.empty(nq, dtype=np.float64)
        second = np.empty(nq, dtype=np.float64)
        rc = lib.oracle_nn_l2(_ptr(q), nq, _ptr(db), ndb, d, _ptr(idx), _ptr(d2), _ptr(second),
                              nthreads)
        assert rc == 0
        return NNResult(idx, d2, second)
    raise ValueError(dtype)


def margin(r: NNResult, dtype: str) -> np.ndarray:
    """How far each query's winner is ahead of its runner-up (>= 0; 0 on a tie).

    Scores are maximised for the descriptor types and squared distances are
    minimised for ``"l2"``.
    """
    return r.second - r.score if dtype == "l2" else r.score - r.second


def score_of(D1: np.ndarray, i: np.ndarray, D2: np.ndarray, j: np.ndarray, dtype: str) -> np.ndarray:
    """Exact scores <D1[i], D2[j]> for paired index arrays (int64 or float64);
    for ``"l2"`` the squared distances |D1[i] - D2[j]|^2 in float64."""
    if dtype == "l2":
        diff = D1[i].astype(np.float64) - D2[j].astype(np.float64)
        return (diff * diff).sum(axis=1)
    if dtype == "i8":
        return (D1[i].astype(np.int64) * D2[j].astype(np.int64)).sum(axis=1)
    if dtype == "f16":
        a = D1[i].view(np.float16).astype(np.float64)
        b = D2[j].view(np.float16).astype(np.float64)
        return (a * b).sum(axis=1)
    a = (D1[i].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (D2[j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return (a * b).sum(axis=1)


def grid_seeds(H: int, W: int, step: int) -> np.ndarray:
    """Seed pixels y*W + x for x in {0, step, 2 step, ...} < W, y likewise < H."""
    ys = np.arange(0, H, step, dtype=np.int64)
    xs = np.arange(0, W, step, dtype=np.int64)
    return (ys[:, None] * W + xs[None, :]).ravel()


@dataclass
class DenseResult:
    pairs: np.ndarray  # int64 [m, 2] (i, j), ascending i
    score: np.ndarray  # [m]
    nn12: NNResult = None
    nn21: NNResult = None


def dense_mutual(D1: np.ndarray, D2: np.ndarray, dtype: str, nthreads: int | None = None) -> DenseResult:
    """All mutual nearest-neighbour pairs between flattened maps D1 [N1,d], D2 [N2,d]."""
    r12 = nn(D1, D2, dtype, nthreads)
    r21 = nn(D2, D1, dtype, nthreads)
    i = np.arange(D1.shape[0])
    keep = r21.idx[r12.idx] == i
    pairs = np.stack([i[keep], r12.idx[keep].astype(np.int64)], axis=1)
    return DenseResult(pairs, r12.score[keep], r12, r21)


@dataclass
class FastResult:
    pairs: np.ndarray  # int64 [m, 2] (u, v), sorted by u
    score: np.ndarray  # [m]
    frontier_sizes: list = field(default_factory=list)  # |F_t| per round run
    first_seen: list = field(default_factory=list)  # new pixels per round run
    min_gap: dict = field(default_factory=dict)  # bf16: kept pixel -> best walk's min top-2 gap


def fast_reciprocal(D1: np.ndarray, H1: int, W1: int, D2: np.ndarray, H2: int, W2: int,
                    dtype: str, subsample: int, max_iter: int,
                    nthreads: int | None = None, track_gaps: bool = False,
                    seeds: np.ndarray | None = None) -> FastResult:
    """MASt3R fast reciprocal matching from a sparse seed grid.

    F_1 = grid seeds of image 1. Round t (t = 1 .. max_iter, while F_t is not
    empty): for each u in F_t, v = NN(D1[u], D2) and u' = NN(D2[v], D1). If
    u' == u the pair (u, v) is kept; otherwise u' joins F_{t+1}, which is
    taken as a set. Walks still open after ``max_iter`` rounds are dropped.

    ``first_seen[t-1]`` counts the members of F_t that appear in no earlier
    frontier. With ``track_gaps`` (float types), ``min_gap[u]`` for a kept
    pixel u is, over all walks that end at u, the largest value of the
    smallest top-2 margin (``margin``) met on that walk (forward and backward
    steps, u's own included): when it is below a tolerance, every walk to u
    passes a near-tie. For ``"l2"`` the scores kept are squared distances.
    """
    D1 = D1.reshape(H1 * W1, -1)
    D2 = D2.reshape(H2 * W2, -1)
    if seeds is None:
        seeds = grid_seeds(H1, W1, subsample)
    F = [int(u) for u in seeds]
    chain_gap = {u: np.inf for u in F}
    kept = {}
    kept_gap = {}
    sizes, first = [], []
    seen: set = set()
    for _ in range(max_iter):
        if not F:
            break
        sizes.append(len(F))
        first.append(sum(1 for u in F if u not in seen))
        seen.update(F)
        fwd = nn(D1[np.array(F)], D2, dtype, nthreads)
        bwd = nn(D2[fwd.idx], D1, dtype, nthreads)
        if track_gaps:
            fm, bm = margin(fwd, dtype), margin(bwd, dtype)
        nxt_gap = {}
        for k, u in enumerate(F):
            v = int(fwd.idx[k])
            u2 = int(bwd.idx[k])
            g = np.inf
            if track_gaps:
                g = min(chain_gap[u], fm[k], bm[k])
            if u2 == u:
                kept[u] = (v, fwd.score[k])
                kept_gap[u] = max(kept_gap.get(u, -np.inf), g)
            else:
                nxt_gap[u2] = max(nxt_gap.get(u2, -np.inf), g)
        F = sorted(nxt_gap)
        chain_gap = nxt_gap
    us = sorted(kept)
    pairs = np.array([[u, kept[u][0]] for u in us], dtype=np.int64).reshape(-1, 2)
    sc = np.array([kept[u][1] for u in us], dtype=np.int64 if dtype == "i8" else np.float64)
    return FastResult(pairs, sc, sizes, first, kept_gap if track_gaps else {})


# ---------------------------------------------------------------------------
# confidence masks
# ---------------------------------------------------------------------------

def confident(conf: np.ndarray | None, n: int, threshold: float) -> np.ndarray:
    """Boolean [n]: pixel takes part iff conf >= threshold (all, without a map)."""
    if conf is None:
        return np.ones(n, dtype=bool)
    return np.asarray(conf, dtype=np.float32).reshape(-1) >= np.float32(threshold)


def nn_masked(q: np.ndarray, db: np.ndarray, keep_db: np.ndarray, dtype: str,
              nthreads: int | None = None) -> NNResult:
    """NN of every query among the database rows with keep_db set: the lowest
    kept index with the best score. The scan runs over the kept rows in
    increasing index order, so it is the plain scan of the definition with the
    excluded rows skipped. idx = -1 when no row is kept."""
    sub = np.nonzero(keep_db)[0]
    if sub.size == 0:
        nq = q.shape[0]
        z = np.zeros(nq, dtype=np.int64 if dtype == "i8" else np.float64)
        return NNResult(np.full(nq, -1, dtype=np.int64), z, z.copy())
    r = nn(q, db[sub], dtype, nthreads)
    return NNResult(sub[r.idx], r.score, r.second)


def dense_mutual_masked(D1: np.ndarray, keep1: np.ndarray, D2: np.ndarray, keep2: np.ndarray,
                        dtype: str, nthreads: int | None = None) -> DenseResult:
    """Mutual nearest-neighbour pairs among the kept pixels of both maps
    (pixel indices of the full maps, ascending i)."""
    i_all = np.nonzero(keep1)[0]
    r12 = nn_masked(D1[i_all], D2, keep2, dtype, nthreads)
    if i_all.size == 0 or r12.idx[0] < 0:
        return DenseResult(np.zeros((0, 2), dtype=np.int64), r12.score[:0], r12, None)
    j_all = np.nonzero(keep2)[0]
    r21 = nn_masked(D2[j_all], D1, keep1, dtype, nthreads)
    back = dict(zip(j_all.tolist(), r21.idx.tolist()))
    keep = np.array([back[int(j)] == int(i) for i, j in zip(i_all, r12.idx)], dtype=bool)
    pairs = np.stack([i_all[keep], r12.idx[keep].astype(np.int64)], axis=1)
    return DenseResult(pairs, r12.score[keep], r12, r21)


def fast_reciprocal_masked(D1: np.ndarray, H1: int, W1: int, keep1: np.ndarray,
                           D2: np.ndarray, H2: int, W2: int, keep2: np.ndarray,
                           dtype: str, subsample: int, max_iter: int,
                           nthreads: int | None = None,
                           max_seeds: int | None = None) -> FastResult:
    """The fast scheme among confident pixels: the seeds are the kept grid
    pixels (grid order); every nearest-neighbour step searches the kept
    pixels of the other image only; everything else is ``fast_reciprocal``.
    A walk whose step finds no kept pixel ends. ``max_seeds`` keeps only the
    first kept seeds (a bounded sample for timing)."""
    D1 = D1.reshape(H1 * W1, -1)
    D2 = D2.reshape(H2 * W2, -1)
    F = [int(u) for u in grid_seeds(H1, W1, subsample) if keep1[u]][:max_seeds]
    kept = {}
    sizes, first = [], []
    seen: set = set()
    for _ in range(max_iter):
        if not F:
            break
        sizes.append(len(F))
        first.append(sum(1 for u in F if u not in seen))
        seen.update(F)
        fwd = nn_masked(D1[np.array(F)], D2, keep2, dtype, nthreads)
        if fwd.idx[0] < 0:
            break
        bwd = nn_masked(D2[fwd.idx], D1, keep1, dtype, nthreads)
        nxt = set()
        for k, u in enumerate(F):
            v, u2 = int(fwd.idx[k]), int(bwd.idx[k])
            if u2 == u:
                kept[u] = (v, fwd.score[k])
            else:
                nxt.add(u2)
        F = sorted(nxt)
    us = sorted(kept)
    pairs = np.array([[u, kept[u][0]] for u in us], dtype=np.int64).reshape(-1, 2)
    sc = np.array([kept[u][1] for u in us], dtype=np.int64 if dtype == "i8" else np.float64)
    return FastResult(pairs, sc, sizes, first, {})
