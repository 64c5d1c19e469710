"""Seeded synthetic descriptor maps for reciprocal nearest-neighbour matching.

These stand in for the dense local-descriptor maps that MASt3R's matching head
emits (one d-vector per pixel, d = 24, L2-normalised; "MASt3R dissection",
section 1 architecture diagram and section 3 Napkin Formula; "DUSt3R / MASt3R
explained", the paragraph on the dense local feature map). No trained network
or dataset is available, so every input is drawn here from a seed.

This module holds input generation only: random draws, a geometric warp that
builds a second view from the first, outlier replacement and rounding to the
storage type. It contains none of the matching arithmetic (no dot products,
no nearest-neighbour search, no reciprocal test). Both the CPU oracle's tests
and the GPU path's tests and benchmark draw their inputs from here.

Random numbers come from NumPy's PCG64 bit generator (O'Neill, "PCG: A Family
of Simple Fast Space-Efficient Statistically Good Algorithms for Random Number
Generation", 2014), seeded with the integers listed in ``CONFIGS``.

Layout of every map: row-major ``[H, W, d]`` (pixel index p = y * W + x),
``int8`` for integer descriptors, ``uint16`` bit patterns of bfloat16 or IEEE
half for float descriptors, ``float32`` for pointmaps (d = 3).

Pointmaps stand in for DUSt3R's per-pixel 3D points: both views' points in the
first camera's frame ("DUSt3R / MASt3R explained", the pointmap and
coordinate-frame paragraphs), so matched pixels of the two views carry nearly
the same point.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "CONFIGS",
    "PairMaps",
    "Workload",
    "make_workload",
    "tiny_permuted_pair",
    "warped_pair_int8",
    "warped_pair_bf16",
    "pointmap_pair",
    "confidence_maps",
    "planted_sign_pair",
    "random_int8_pair",
    "f64_to_bf16_bits",
    "f64_to_f16_bits",
    "bf16_bits_to_f64",
]

BASE_SEED = 0x5EED0000


@dataclass
class PairMaps:
    """One image pair of descriptor maps plus the generator's ground truth.

    ``gt_src[p]`` is the map-1 pixel that map-2 pixel ``p`` was drawn from, or
    -1 where ``p`` is an outlier (re-drawn at random). It is kept only to
    report inlier rates; matching never reads it.
    """

    desc1: np.ndarray  # [H1, W1, d]
    desc2: np.ndarray  # [H2, W2, d]
    gt_src: np.ndarray  # [H2 * W2] int64
    dtype: str  # "i8", "bf16", "f16" or "l2" (float32 pointmaps)

    @property
    def H1(self) -> int:
        return int(self.desc1.shape[0])

    @property
    def W1(self) -> int:
        return int(self.desc1.shape[1])

    @property
    def H2(self) -> int:
        return int(self.desc2.shape[0])

    @property
    def W2(self) -> int:
        return int(self.desc2.shape[1])

    @property
    def d(self) -> int:
        return int(self.desc1.shape[2])


@dataclass
class Workload:
    """A named matching workload: one or more pairs plus the matching settings."""

    name: str
    pairs: list
    subsample: int
    max_iter: int
    dense: bool = False
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.pairs)

    def stacked(self):
        """Return (desc1 [B,H1,W1,d], desc2 [B,H2,W2,d]) as contiguous arrays."""
        d1 = np.ascontiguousarray(np.stack([p.desc1 for p in self.pairs]))
        d2 = np.ascontiguousarray(np.stack([p.desc2 for p in self.pairs]))
        return d1, d2


# ---------------------------------------------------------------------------
# storage-type helpers (input preparation, not matching arithmetic)
# ---------------------------------------------------------------------------


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (via float32, round-to-nearest-even).

    Returns the raw 16-bit patterns as ``uint16``. Inputs must be finite.
    """
    f32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f32.view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to IEEE half (round-to-nearest-even); raw uint16 bits."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------


def random_int8_pair(seed: int, H1: int, W1: int, H2: int, W2: int, d: int,
                     lo: int, hi: int) -> PairMaps:
    """Two independent maps with entries uniform in the integers [lo, hi]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    d1 = rng.integers(lo, hi + 1, size=(H1, W1, d), dtype=np.int64).astype(np.int8)
    d2 = rng.integers(lo, hi + 1, size=(H2, W2, d), dtype=np.int64).astype(np.int8)
    return PairMaps(d1, d2, np.full(H2 * W2, -1, dtype=np.int64), "i8")


def tiny_permuted_pair(seed: int, H: int = 48, W: int = 64, d: int = 24,
                       amp: int = 8, redraw_frac: float = 0.2) -> PairMaps:
    """Map 1 uniform in [-amp, amp]; map 2 a seeded pixel permutation of map 1.

    map2[pi(i)] = map1[i] for a Fisher-Yates permutation pi, then
    round(redraw_frac * H * W) map-2 pixels (a seeded choice) are re-drawn
    uniformly from the same range.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n = H * W
    m1 = rng.integers(-amp, amp + 1, size=(n, d), dtype=np.int64)
    perm = rng.permutation(n)  # pi
    m2 = np.empty_like(m1)
    m2[perm] = m1
    gt = np.empty(n, dtype=np.int64)
    gt[perm] = np.arange(n)
    k = int(round(redraw_frac * n))
    out = rng.choice(n, size=k, replace=False)
    m2[out] = rng.integers(-amp, amp + 1, size=(k, d), dtype=np.int64)
    gt[out] = -1
    return PairMaps(m1.astype(np.int8).reshape(H, W, d),
                    m2.astype(np.int8).reshape(H, W, d), gt, "i8")


def _warp_sources(rng: np.random.Generator, H: int, W: int, jitter: int = 4,
                  max_rot_deg: float = 10.0, scale_range=(0.9, 1.1),
                  max_shift: float = 16.0) -> np.ndarray:
    """Source pixel in view 1 for every view-2 pixel under a random smooth warp.

    src = round(A (p - c) + c + t + j_p) with A = R(theta) diag(s, s),
    theta ~ U[-10, 10] degrees, s ~ U[0.9, 1.1], t ~ U[-16, 16]^2 px and an
    integer per-pixel jitter j_p ~ U{-4..4}^2; c is the image centre.
    Returns int64 [H*W] source indices, -1 where the source falls outside.
    """
    theta = np.deg2rad(rng.uniform(-max_rot_deg, max_rot_deg))
    s = rng.uniform(*scale_range)
    t = rng.uniform(-max_shift, max_shift, size=2)
    A = s * np.array([[np.cos(theta), -np.sin(theta)],
                      [np.sin(theta), np.cos(theta)]])
    ys, xs = np.meshgrid(np.arange(H, dtype=np.float64),
                         np.arange(W, dtype=np.float64), indexing="ij")
    c = np.array([(W - 1) / 2.0, (H - 1) / 2.0])
    px = np.stack([xs.ravel() - c[0], ys.ravel() - c[1]])  # [2, n]
    warped = A @ px + (c + t)[:, None]
    jit = rng.integers(-jitter, jitter + 1, size=(2, H * W), dtype=np.int64)
    sx = np.rint(warped[0]).astype(np.int64) + jit[0]
    sy = np.rint(warped[1]).astype(np.int64) + jit[1]
    ok = (sx >= 0) & (sx < W) & (sy >= 0) & (sy < H)
    return np.where(ok, sy * W + sx, -1)


def warped_pair_int8(seed: int, H: int = 384, W: int = 512, d: int = 24,
                     amp: int = 16, noise: int = 2,
                     outlier_frac: float = 0.3) -> PairMaps:
    """Map 1 uniform in [-amp, amp]; map 2 a noisy smooth warp of map 1.

    map2[p] = map1[src(p)] + U{-noise..noise} per entry (not clamped), then a
    seeded outlier_frac of the pixels, plus every pixel whose source fell
    outside map 1, are re-drawn uniformly in [-amp, amp].
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n = H * W
    m1 = rng.integers(-amp, amp + 1, size=(n, d), dtype=np.int64)
    src = _warp_sources(rng, H, W)
    m2 = m1[np.maximum(src, 0)] + rng.integers(-noise, noise + 1, size=(n, d),
                                               dtype=np.int64)
    k = int(round(outlier_frac * n))
    out = np.zeros(n, dtype=bool)
    out[rng.choice(n, size=k, replace=False)] = True
    out |= src < 0
    m2[out] = rng.integers(-amp, amp + 1, size=(int(out.sum()), d), dtype=np.int64)
    gt = np.where(out, -1, src)
    assert np.abs(m2).max() <= 127
    return PairMaps(m1.astype(np.int8).reshape(H, W, d),
                    m2.astype(np.int8).reshape(H, W, d), gt, "i8")


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def warped_pair_bf16(seed: int, H: int = 384, W: int = 512, d: int = 24,
                     sigma: float = 0.05, outlier_frac: float = 0.3,
                     storage: str = "bf16") -> PairMaps:
    """Unit-norm float descriptors stored as bfloat16.

    map1 ~ N(0, 1)^d per pixel, L2-normalised in float64. map2 = the warped
    float64 map1 plus N(0, sigma) per entry, re-normalised; outliers (a seeded
    outlier_frac plus out-of-bounds sources) are fresh normalised N(0, 1)
    vectors. Both maps are then rounded to bfloat16.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n = H * W
    m1 = _unit_rows(rng.standard_normal((n, d)))
    src = _warp_sources(rng, H, W)
    m2 = m1[np.maximum(src, 0)] + sigma * rng.standard_normal((n, d))
    k = int(round(outlier_frac * n))
    out = np.zeros(n, dtype=bool)
    out[rng.choice(n, size=k, replace=False)] = True
    out |= src < 0
    m2[out] = rng.standard_normal((int(out.sum()), d))
    m2 = _unit_rows(m2)
    gt = np.where(out, -1, src)
    cvt = f64_to_bf16_bits if storage == "bf16" else f64_to_f16_bits
    return PairMaps(cvt(m1).reshape(H, W, d), cvt(m2).reshape(H, W, d), gt, storage)


def pointmap_pair(seed: int, H: int = 384, W: int = 512, noise: float = 0.002,
                  outlier_frac: float = 0.3) -> PairMaps:
    """Two float32 pointmaps of one smooth surface in the first camera's frame.

    View 1: pinhole rays (focal 0.9 W px, principal point at the centre) hit a
    depth surface z(x, y) = 3 + 0.6 y / H + a seeded sum of four low-frequency
    sinusoids of amplitude up to 0.15 (metres). View 2: the warp generator of
    the descriptor pairs picks each pixel's source pixel in view 1 and the
    point is that view-1 point plus N(0, noise * z) per coordinate (regression
    blur); a seeded outlier_frac of the pixels, plus those whose source fell
    outside view 1, get fresh points uniform in the bounding box of view 1.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n = H * W
    ys, xs = np.meshgrid(np.arange(H, dtype=np.float64), np.arange(W, dtype=np.float64),
                         indexing="ij")
    f = 0.9 * W
    z = 3.0 + 0.6 * ys / H
    for _ in range(4):
        kx, ky = rng.uniform(0.5, 3.0, size=2)
        ph = rng.uniform(0, 2 * np.pi)
        z = z + rng.uniform(0.03, 0.15) * np.sin(2 * np.pi * (kx * xs / W + ky * ys / H) + ph)
    p1 = np.stack([(xs - (W - 1) / 2.0) / f * z, (ys - (H - 1) / 2.0) / f * z, z],
                  axis=-1).reshape(n, 3)
    src = _warp_sources(rng, H, W)
    p2 = p1[np.maximum(src, 0)]
    p2 = p2 + noise * p2[:, 2:3] * rng.standard_normal((n, 3))
    k = int(round(outlier_frac * n))
    out = np.zeros(n, dtype=bool)
    out[rng.choice(n, size=k, replace=False)] = True
    out |= src < 0
    lo, hi = p1.min(axis=0), p1.max(axis=0)
    p2[out] = rng.uniform(lo, hi, size=(int(out.sum()), 3))
    gt = np.where(out, -1, src)
    return PairMaps(p1.astype(np.float32).reshape(H, W, 3),
                    p2.astype(np.float32).reshape(H, W, 3), gt, "l2")


def confidence_maps(seed: int, H: int, W: int, gt_src: np.ndarray | None = None,
                    sky_frac: float = 0.12) -> tuple[np.ndarray, np.ndarray]:
    """Per-pixel confidences for the two views of a pair, float32 [H, W], >= 1.

    Shaped like the confidences DUSt3R predicts beside its pointmaps (1 plus
    an exponential): conf = 1 + exp(0.8 + 0.6 f) with f a seeded smooth
    field (four low-frequency sinusoids), a low-confidence band over the top
    sky_frac of the rows (conf in [1, 1.3]), and, in view 2, confidence in
    [1, 1.5] on 80% of the generator's outlier pixels (gt_src == -1).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    ys, xs = np.meshgrid(np.arange(H, dtype=np.float64), np.arange(W, dtype=np.float64),
                         indexing="ij")
    out = []
    for view in range(2):
        f = np.zeros((H, W))
        for _ in range(4):
            kx, ky = rng.uniform(0.5, 4.0, size=2)
            f += np.sin(2 * np.pi * (kx * xs / W + ky * ys / H) + rng.uniform(0, 2 * np.pi))
        conf = 1.0 + np.exp(0.8 + 0.6 * f / 2.0)
        sky = ys < sky_frac * H
        conf[sky] = rng.uniform(1.0, 1.3, size=int(sky.sum()))
        if view == 1 and gt_src is not None:
            o = (gt_src.reshape(H, W) < 0) & (rng.uniform(size=(H, W)) < 0.8)
            conf[o] = rng.uniform(1.0, 1.5, size=int(o.sum()))
        out.append(conf.astype(np.float32))
    return out[0], out[1]


def planted_sign_pair(seed: int, H: int, W: int, d: int, c: int = 8,
                      redraw_frac: float = 0.2) -> PairMaps:
    """Sign-vector maps with a planted permutation.

    Every descriptor lies in {-c, +c}^d and all descriptors of both maps are
    pairwise distinct, so all have the same norm and <x, y> < |x|^2 for any
    y != x. map2[pi(i)] = map1[i]; a seeded redraw_frac of map-2 pixels get
    fresh sign vectors distinct from every other descriptor.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n = H * W
    if 2 ** d < 2 * n:
        raise ValueError("d too small for distinct sign vectors")
    seen: set = set()

    def fresh(count):
        rows = []
        while len(rows) < count:
            bits = rng.integers(0, 2, size=d, dtype=np.int64)
            key = bits.tobytes()
            if key in seen:
                continue
            seen.add(key)
            rows.append(bits)
        return (np.array(rows, dtype=np.int64) * 2 - 1) * c

    m1 = fresh(n)
    perm = rng.permutation(n)
    m2 = np.empty_like(m1)
    m2[perm] = m1
    gt = np.empty(n, dtype=np.int64)
    gt[perm] = np.arange(n)
    k = int(round(redraw_frac * n))
    out = rng.choice(n, size=k, replace=False)
    m2[out] = fresh(k)
    gt[out] = -1
    return PairMaps(m1.astype(np.int8).reshape(H, W, d),
                    m2.astype(np.int8).reshape(H, W, d), gt, "i8")


# ---------------------------------------------------------------------------
# the named workloads
# ---------------------------------------------------------------------------

CONFIGS = {
    "tiny_64x48_d24_i8": dict(
        seed=BASE_SEED + 1,
        note="two 64x48 maps, d=24, int8 uniform in [-8,8]; map2 a seeded pixel "
             "permutation of map1 with 20% of pixels re-drawn; fast matching from "
             "an 8-px grid (48 seeds), max_iter=10; dense mutual over 3072x3072"),
    "pair_512x384_d24_i8": dict(
        seed=BASE_SEED + 2,
        note="one 512x384 pair, d=24, int8 uniform in [-16,16]; map2 a smooth warp "
             "(affine + 4 px jitter) with 30% outliers and +-2 noise; fast matching "
             "from an 8-px grid (3,072 seeds), max_iter=10"),
    "dense_512x384_d24_i8": dict(
        seed=BASE_SEED + 2,
        note="dense mutual nearest neighbours over all 196,608 pixels of the "
             "512x384 int8 pair above (same seed, same maps)"),
    "pair_512x384_d24_bf16": dict(
        seed=BASE_SEED + 4,
        note="one 512x384 pair, d=24, unit-norm bf16; map2 warped map1 plus "
             "N(0,0.05) noise, renormalised, 30% outliers; 8-px grid, max_iter=10"),
    "pair_512x384_d24_f16": dict(
        seed=BASE_SEED + 4,
        note="the bf16 512x384 pair above (same seed, same float maps) stored as "
             "IEEE half; 8-px grid, max_iter=10"),
    "pair_512x384_d64_i8": dict(
        seed=BASE_SEED + 6,
        note="one 512x384 pair, d=64, int8 uniform in [-16,16], warped as the d=24 "
             "pair; 8-px grid (3,072 seeds), max_iter=10"),
    "pair_512x384_pts3_f32": dict(
        seed=BASE_SEED + 7,
        note="one 512x384 pair of float32 pointmaps (d=3, metres, camera-1 frame): "
             "a smooth random depth surface at 3-3.6 m seen by view 1; view 2 the "
             "warp generator's sources with N(0, 0.002 z) noise and 30% outliers "
             "uniform in the scene's bounding box; nearest 3D point by Euclidean "
             "distance; 8-px grid (3,072 seeds), max_iter=10"),
    "dense_512x384_pts3_f32": dict(
        seed=BASE_SEED + 7,
        note="dense mutual nearest 3D points over all 196,608 pixels of the 512x384 "
             "pointmap pair above (same seed, same maps)"),
    "pair_512x384_d24_i8_conf": dict(
        seed=BASE_SEED + 2,
        note="the int8 512x384 pair (same seed, same maps) with per-pixel "
             "confidences (confidence_maps, seed + 50): a pixel takes part iff its "
             "confidence >= 2.0 (about 80% of view 1 and 60% of view 2 do); "
             "8-px grid, max_iter=10"),
    "batch16_512x288_d32_i8": dict(
        seed=BASE_SEED + 5,
        note="16 independent 512x288 pairs, d=32, int8 uniform in [-16,16], warped "
             "as above, pair b seeded with seed + 1000*b; 4-px grid (9,216 seeds "
             "per pair), max_iter=15, one launch sequence on one stream"),
}


def make_workload(name: str, batch: int | None = None) -> Workload:
    """Build one of the named workloads in ``CONFIGS``.

    ``batch`` (only for the 16-pair workload) builds the first ``batch`` pairs.
    """
    cfg = CONFIGS[name]
    seed = cfg["seed"]
    if name == "tiny_64x48_d24_i8":
        return Workload(name, [tiny_permuted_pair(seed)], subsample=8, max_iter=10,
                        dense=True, note=cfg["note"])
    if name == "pair_512x384_d24_i8":
        return Workload(name, [warped_pair_int8(seed)], subsample=8, max_iter=10,
                        note=cfg["note"])
    if name == "dense_512x384_d24_i8":
        return Workload(name, [warped_pair_int8(seed)], subsample=8, max_iter=10,
                        dense=True, note=cfg["note"])
    if name == "pair_512x384_d24_bf16":
        return Workload(name, [warped_pair_bf16(seed)], subsample=8, max_iter=10,
                        note=cfg["note"])
    if name == "pair_512x384_d24_f16":
        return Workload(name, [warped_pair_bf16(seed, storage="f16")], subsample=8,
                        max_iter=10, note=cfg["note"])
    if name == "pair_512x384_d64_i8":
        return Workload(name, [warped_pair_int8(seed, d=64)], subsample=8, max_iter=10,
                        note=cfg["note"])
    if name == "pair_512x384_pts3_f32":
        return Workload(name, [pointmap_pair(seed)], subsample=8, max_iter=10, note=cfg["note"])
    if name == "dense_512x384_pts3_f32":
        return Workload(name, [pointmap_pair(seed)], subsample=8, max_iter=10, dense=True,
                        note=cfg["note"])
    if name == "pair_512x384_d24_i8_conf":
        p = warped_pair_int8(seed)
        c1, c2 = confidence_maps(seed + 50, p.H1, p.W1, p.gt_src)
        return Workload(name, [p], subsample=8, max_iter=10, note=cfg["note"],
                        extra={"conf1": [c1], "conf2": [c2], "threshold": 2.0})
    if name == "batch16_512x288_d32_i8":
        nb = 16 if batch is None else batch
        pairs = [warped_pair_int8(seed + 1000 * b, H=288, W=512, d=32)
                 for b in range(nb)]
        return Workload(name, pairs, subsample=4, max_iter=15, note=cfg["note"])
    raise KeyError(name)
