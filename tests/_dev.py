"""Helpers shared by the GPU tests: device copies and parity comparisons."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

BF16_TOL = 1e-2  # absolute score tolerance for bfloat16 descriptors


def require_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(a: np.ndarray, half: str = "bf16") -> torch.Tensor:
    """int8 arrays stay int8; uint16 arrays are the bit patterns of bfloat16
    (``half="bf16"``) or IEEE half (``half="f16"``) descriptors."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.int8:
        return torch.from_numpy(a).cuda()
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).cuda()
        return t.view(torch.bfloat16 if half == "bf16" else torch.float16)
    raise TypeError(a.dtype)


def gpu_pairs(pairs: torch.Tensor, score: torch.Tensor, count: torch.Tensor, b: int = 0):
    n = int(count[b].item()) if count.dim() else int(count.item())
    p = pairs[b, :n] if pairs.dim() == 3 else pairs[:n]
    s = score[b, :n] if score.dim() == 2 else score[:n]
    return p.cpu().numpy().astype(np.int64), s.cpu().numpy()


def check_nn_exact(idx_g, score_g, ref: oracle.NNResult):
    idx_g = idx_g.cpu().numpy()
    score_g = score_g.cpu().numpy()
    bad = np.nonzero(idx_g != ref.idx)[0]
    assert bad.size == 0, f"{bad.size} index mismatches, first at {bad[:5]}: " \
        f"gpu {idx_g[bad[:5]]} vs oracle {ref.idx[bad[:5]]}"
    assert np.array_equal(score_g.astype(np.int64), ref.score)


def check_nn_bf16(idx_g, score_g, q, db, ref: oracle.NNResult, tol=BF16_TOL, dtype="bf16"):
    """Tolerance rule for float descriptors.

    The GPU score must be within tol of the exact score of the pair it chose,
    the chosen pair must be within tol of the exact best, and the index may
    differ from the oracle's only where the exact top-2 gap is below tol.
    """
    idx_g = idx_g.cpu().numpy().astype(np.int64)
    score_g = score_g.cpu().numpy().astype(np.float64)
    exact_chosen = oracle.score_of(q, np.arange(len(idx_g)), db, idx_g, dtype)
    assert np.all(np.abs(score_g - exact_chosen) <= tol)
    assert np.all(ref.score - exact_chosen <= tol)
    diff = idx_g != ref.idx
    assert np.all(ref.score[diff] - ref.second[diff] < tol)
    return int(diff.sum())
