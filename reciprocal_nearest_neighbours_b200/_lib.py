"""ctypes binding of libfastnn.so: argument marshalling only."""

from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libfastnn.so")

FASTNN_I8 = 0
FASTNN_BF16 = 1
FASTNN_F16 = 2
FASTNN_F32_L2 = 3
FASTNN_OP_NN = 0
FASTNN_OP_RECIPROCAL = 1
FASTNN_OP_MUTUAL_DENSE = 2
FASTNN_OP_MUTUAL_FROM_NN = 3
FASTNN_OP_RECIPROCAL_MASKED = 4
FASTNN_OP_MUTUAL_DENSE_MASKED = 5
FASTNN_OP_IMAGE_ROWS = 6

_lib = None


class FastNNError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {fastnn_status_str(status)} ({status})"
        if status == -4:
            msg += ": " + library().fastnn_last_cuda_error().decode()
        super().__init__(msg)


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load libfastnn.so (built in-tree by ``build()``); raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -m reciprocal_nearest_neighbours_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.fastnn_workspace_size.argtypes = [I, I64, I64, I, I, I, I64]
    lib.fastnn_workspace_size.restype = SZ
    lib.fastnn_nn.argtypes = [P, I64, P, I64, I, I, P, P, P, SZ, P]
    lib.fastnn_nn.restype = I
    lib.fastnn_reciprocal.argtypes = [P, I, I, P, I, I, I, I, I, I, I, P, P, I64, P, P, P, P, SZ, P]
    lib.fastnn_reciprocal.restype = I
    lib.fastnn_reciprocal_noalloc.argtypes = [P, I, I, P, I, I, I, I, I, I, I, P, P, I64, P, P, P, P]
    lib.fastnn_reciprocal_noalloc.restype = I
    lib.fastnn_mutual_dense.argtypes = [P, I64, P, I64, I, I, P, P, I64, P, P, SZ, P]
    lib.fastnn_mutual_dense.restype = I
    F = ctypes.c_float
    lib.fastnn_reciprocal_masked.argtypes = [P, P, I, I, P, P, I, I, I, I, F, I, I, I, P, P, I64,
                                             P, P, P, P, SZ, P]
    lib.fastnn_reciprocal_masked.restype = I
    lib.fastnn_mutual_dense_masked.argtypes = [P, P, I64, P, P, I64, I, I, F, P, P, I64, P, P, SZ,
                                               P]
    lib.fastnn_mutual_dense_masked.restype = I
    lib.fastnn_mutual_from_nn.argtypes = [P, P, I64, I64, P, I64, I64, I, P, P, I64, P, P, SZ, P]
    lib.fastnn_mutual_from_nn.restype = I
    lib.fastnn_image_rows.argtypes = [P, I64, I64, P, P, P, SZ, P]
    lib.fastnn_image_rows.restype = I
    lib.fastnn_device_status.argtypes = [P, P]
    lib.fastnn_device_status.restype = I
    lib.fastnn_noalloc_device_status.argtypes = [P]
    lib.fastnn_noalloc_device_status.restype = I
    lib.fastnn_kernel_timer_enable.argtypes = [I]
    lib.fastnn_kernel_timer_enable.restype = I
    lib.fastnn_kernel_timer_select.argtypes = [I]
    lib.fastnn_kernel_timer_select.restype = I
    lib.fastnn_kernel_timer_read.argtypes = [ctypes.POINTER(I), ctypes.POINTER(ctypes.c_double)]
    lib.fastnn_kernel_timer_read.restype = I
    lib.fastnn_last_cuda_error.argtypes = []
    lib.fastnn_last_cuda_error.restype = ctypes.c_char_p
    lib.fastnn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.fastnn_set_wait_timeout_ns.restype = None
    lib.fastnn_status_str.argtypes = [I]
    lib.fastnn_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def fastnn_status_str(status: int) -> str:
    return library().fastnn_status_str(int(status)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise FastNNError(rc, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.int8:
        return FASTNN_I8
    if t.dtype == torch.bfloat16:
        return FASTNN_BF16
    if t.dtype == torch.float16:
        return FASTNN_F16
    if t.dtype == torch.float32:
        return FASTNN_F32_L2
    raise TypeError(f"descriptors must be int8, bfloat16 or float16 (dot product) or float32 "
                    f"3D points (Euclidean distance), got {t.dtype}")


def _score_dtype(code: int):
    return torch.int32 if code == FASTNN_I8 else torch.float32


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        raise FastNNError(-1, "fastnn_workspace_size")
    if workspace is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise FastNNError(-3, "workspace")
    return workspace


def seed_count(H: int, W: int, subsample: int) -> int:
    return ((H + subsample - 1) // subsample) * ((W + subsample - 1) // subsample)


def fastnn_workspace_size(op: int, n1: int, n2: int, d: int, dtype: int, batch: int = 1,
                          max_queries: int = 0) -> int:
    return int(library().fastnn_workspace_size(op, n1, n2, d, dtype, batch, max_queries))


def fastnn_nn(q: torch.Tensor, db: torch.Tensor, out_idx=None, out_score=None,
              workspace=None, stream=None):
    """Nearest neighbour of each row of ``q`` [nq, d] among rows of ``db`` [ndb, d].

    Returns ``(idx int32 [nq], score [nq])`` (int32 scores for int8
    descriptors, float32 for bfloat16 and float16). float32 inputs are 3D
    points (d <= 3): the nearest point by Euclidean distance, with its
    squared distance as the score.
    """
    _need_cuda(q, db)
    code = _dtype_code(q)
    assert db.dtype == q.dtype and q.dim() == 2 and db.dim() == 2 and q.shape[1] == db.shape[1]
    nq, d = q.shape
    ndb = db.shape[0]
    if out_idx is None:
        out_idx = torch.empty(nq, dtype=torch.int32, device=q.device)
    if out_score is None:
        out_score = torch.empty(nq, dtype=_score_dtype(code), device=q.device)
    nbytes = fastnn_workspace_size(FASTNN_OP_NN, nq, ndb, d, code)
    ws = _workspace(nbytes, q.device, workspace)
    rc = library().fastnn_nn(_ptr(q), nq, _ptr(db), ndb, d, code, _ptr(out_idx), _ptr(out_score),
                             _ptr(ws), nbytes, _stream(stream))
    _check(rc, "fastnn_nn")
    return out_idx, out_score


def fastnn_reciprocal(desc1: torch.Tensor, desc2: torch.Tensor, subsample: int, max_iter: int,
                      capacity: int | None = None, out_pairs=None, out_score=None,
                      out_count=None, out_iters=None, out_frontier=None, workspace=None,
                      stream=None):
    """MASt3R fast reciprocal matching of ``desc1`` [B,H1,W1,d] against ``desc2`` [B,H2,W2,d].

    A 3-d input is a batch of one. Returns ``(pairs [B,cap,2] int32,
    score [B,cap], count [B] int32, iters [B] int32)``; pair b's matches are
    ``pairs[b, :count[b]]`` in order of discovery. ``out_frontier`` (optional,
    int32 [B, max_iter]) receives the frontier size of every round.
    """
    _need_cuda(desc1, desc2)
    code = _dtype_code(desc1)
    assert desc2.dtype == desc1.dtype
    if desc1.dim() == 3:
        desc1, desc2 = desc1.unsqueeze(0), desc2.unsqueeze(0)
    B, H1, W1, d = desc1.shape
    B2, H2, W2, d2 = desc2.shape
    assert B2 == B and d2 == d
    S = seed_count(H1, W1, subsample)
    cap = S if capacity is None else int(capacity)
    dev = desc1.device
    if out_pairs is None:
        out_pairs = torch.empty((B, cap, 2), dtype=torch.int32, device=dev)
    if out_score is None:
        out_score = torch.empty((B, cap), dtype=_score_dtype(code), device=dev)
    if out_count is None:
        out_count = torch.empty(B, dtype=torch.int32, device=dev)
    if out_iters is None:
        out_iters = torch.empty(B, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_RECIPROCAL, H1 * W1, H2 * W2, d, code, B, S)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_reciprocal(_ptr(desc1), H1, W1, _ptr(desc2), H2, W2, d, code,
                                     subsample, max_iter, B, _ptr(out_pairs), _ptr(out_score),
                                     cap, _ptr(out_count), _ptr(out_iters), _ptr(out_frontier),
                                     _ptr(ws), nbytes,
                                     _stream(stream))
    _check(rc, "fastnn_reciprocal")
    return out_pairs, out_score, out_count, out_iters


def fastnn_reciprocal_noalloc(desc1: torch.Tensor, desc2: torch.Tensor, subsample: int,
                              max_iter: int, out_pairs: torch.Tensor, out_score: torch.Tensor,
                              out_count: torch.Tensor, out_iters=None, out_frontier=None,
                              stream=None):
    """fastnn_reciprocal without a workspace, for callers that cannot allocate.

    The library's fixed device scratch array stands in for the workspace (see
    include/fastnn.h); the caller passes every output buffer. Calls on one
    device share that array, so they must not overlap on the GPU.
    """
    _need_cuda(desc1, desc2, out_pairs, out_score, out_count)
    code = _dtype_code(desc1)
    if desc1.dim() == 3:
        desc1, desc2 = desc1.unsqueeze(0), desc2.unsqueeze(0)
    B, H1, W1, d = desc1.shape
    _, H2, W2, _ = desc2.shape
    cap = out_pairs.shape[-2]
    rc = library().fastnn_reciprocal_noalloc(
        _ptr(desc1), H1, W1, _ptr(desc2), H2, W2, d, code, subsample, max_iter, B,
        _ptr(out_pairs), _ptr(out_score), cap, _ptr(out_count), _ptr(out_iters),
        _ptr(out_frontier), _stream(stream))
    _check(rc, "fastnn_reciprocal_noalloc")
    return out_pairs, out_score, out_count, out_iters


def fastnn_mutual_dense(desc1: torch.Tensor, desc2: torch.Tensor, capacity: int | None = None,
                        out_pairs=None, out_score=None, out_count=None, workspace=None,
                        stream=None):
    """Every mutual nearest-neighbour pair of ``desc1`` [n1, d] and ``desc2`` [n2, d].

    Returns ``(pairs [cap,2] int32, score [cap], count [1] int32)``; the pairs
    are ``pairs[:count]`` in ascending image-1 index.
    """
    _need_cuda(desc1, desc2)
    code = _dtype_code(desc1)
    desc1 = desc1.reshape(-1, desc1.shape[-1])
    desc2 = desc2.reshape(-1, desc2.shape[-1])
    n1, d = desc1.shape
    n2 = desc2.shape[0]
    cap = min(n1, n2) if capacity is None else int(capacity)
    dev = desc1.device
    if out_pairs is None:
        out_pairs = torch.empty((cap, 2), dtype=torch.int32, device=dev)
    if out_score is None:
        out_score = torch.empty(cap, dtype=_score_dtype(code), device=dev)
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_MUTUAL_DENSE, n1, n2, d, code)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_mutual_dense(_ptr(desc1), n1, _ptr(desc2), n2, d, code, _ptr(out_pairs),
                                       _ptr(out_score), cap, _ptr(out_count), _ptr(ws), nbytes,
                                       _stream(stream))
    _check(rc, "fastnn_mutual_dense")
    return out_pairs, out_score, out_count


def fastnn_mutual_from_nn(nn12: torch.Tensor, score12, i0: int, nn21: torch.Tensor,
                          n1_total: int, capacity: int | None = None, out_pairs=None,
                          out_score=None, out_count=None, workspace=None, stream=None):
    """Mutual pairs of a row shard of image 1 from nearest-neighbour indices.

    ``nn12`` [n1] int32 (partners of global rows i0 .. i0 + n1 - 1),
    ``score12`` [n1] int32 or float32 (or None), ``nn21`` [n2] int32 (global
    image-1 partner of every image-2 row). Returns ``(pairs [cap,2],
    score [cap], count [1])`` with pairs[:count] in ascending image-1 index.
    """
    _need_cuda(nn12, nn21)
    n1, n2 = nn12.numel(), nn21.numel()
    dev = nn12.device
    sdt = score12.dtype if score12 is not None else torch.int32
    code = FASTNN_BF16 if sdt == torch.float32 else FASTNN_I8
    cap = max(1, min(n1, n2)) if capacity is None else int(capacity)
    if out_pairs is None:
        out_pairs = torch.empty((cap, 2), dtype=torch.int32, device=dev)
    if out_score is None:
        out_score = torch.empty(cap, dtype=sdt, device=dev)
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_MUTUAL_FROM_NN, max(n1, 1), n2, 1, code)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_mutual_from_nn(_ptr(nn12), _ptr(score12), n1, int(i0), _ptr(nn21), n2,
                                         int(n1_total), code, _ptr(out_pairs), _ptr(out_score),
                                         cap, _ptr(out_count), _ptr(ws), nbytes, _stream(stream))
    _check(rc, "fastnn_mutual_from_nn")
    return out_pairs, out_score, out_count


def fastnn_image_rows(nn12: torch.Tensor, n2: int, out_rows=None, out_count=None,
                      workspace=None, stream=None):
    """Ascending distinct values of ``nn12`` [n1] int32 that lie in [0, n2):
    the image-2 rows some image-1 row matches. Returns ``(rows [cap], count
    [1])`` with rows[:count] valid (cap = min(n1, n2))."""
    _need_cuda(nn12)
    n1 = nn12.numel()
    dev = nn12.device
    cap = max(1, min(n1, int(n2)))
    if out_rows is None:
        out_rows = torch.empty(cap, dtype=torch.int32, device=dev)
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_IMAGE_ROWS, n1, int(n2), 1, FASTNN_I8)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_image_rows(_ptr(nn12) if n1 else None, n1, int(n2), _ptr(out_rows),
                                     _ptr(out_count), _ptr(ws), nbytes, _stream(stream))
    _check(rc, "fastnn_image_rows")
    return out_rows, out_count


def fastnn_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device status of the last call on ``workspace``."""
    return int(library().fastnn_device_status(_ptr(workspace), _stream(stream)))


def fastnn_noalloc_device_status(stream=None) -> int:
    """Synchronise and return the device status of the last allocation-free
    call on the current device (read from the library's static scratch)."""
    return int(library().fastnn_noalloc_device_status(_stream(stream)))


def fastnn_kernel_timer_enable(capacity: int) -> None:
    """Time the next ``capacity`` nearest-neighbour kernel launches with CUDA events."""
    _check(library().fastnn_kernel_timer_enable(int(capacity)), "fastnn_kernel_timer_enable")


FASTNN_TIME_MATCHING = 1
FASTNN_TIME_REPACK = 2
FASTNN_TIME_MUTUAL = 4
FASTNN_TIME_MASK = 8


def fastnn_kernel_timer_select(kinds: int) -> int:
    """Choose which launch kinds the timer brackets (FASTNN_TIME_* bit mask);
    returns the previous selection."""
    return int(library().fastnn_kernel_timer_select(int(kinds)))


def fastnn_kernel_timer_read():
    """Return (launches, total device milliseconds) since the last read; resets."""
    n = ctypes.c_int(0)
    ms = ctypes.c_double(0.0)
    _check(library().fastnn_kernel_timer_read(ctypes.byref(n), ctypes.byref(ms)),
           "fastnn_kernel_timer_read")
    return int(n.value), float(ms.value)


def _conf(conf, n_expected, dev):
    if conf is None:
        return None
    if not (conf.is_cuda and conf.is_contiguous() and conf.dtype == torch.float32):
        raise ValueError("confidence maps must be contiguous float32 CUDA tensors")
    if conf.numel() != n_expected:
        raise ValueError("confidence map size does not match the descriptor map")
    return conf


def fastnn_reciprocal_masked(desc1: torch.Tensor, desc2: torch.Tensor, subsample: int,
                             max_iter: int, conf1: torch.Tensor | None = None,
                             conf2: torch.Tensor | None = None, threshold: float = 0.0,
                             capacity: int | None = None, out_pairs=None, out_score=None,
                             out_count=None, out_iters=None, out_frontier=None, workspace=None,
                             stream=None):
    """Fast reciprocal matching among confident pixels (conf >= threshold).

    ``conf1`` [B,H1,W1] / ``conf2`` [B,H2,W2] float32, or None (every pixel of
    that image takes part). Everything else as ``fastnn_reciprocal``; the
    pairs are pixel indices of the full maps.
    """
    _need_cuda(desc1, desc2)
    code = _dtype_code(desc1)
    assert desc2.dtype == desc1.dtype
    if desc1.dim() == 3:
        desc1, desc2 = desc1.unsqueeze(0), desc2.unsqueeze(0)
    B, H1, W1, d = desc1.shape
    B2, H2, W2, d2 = desc2.shape
    assert B2 == B and d2 == d
    conf1 = _conf(conf1, B * H1 * W1, desc1.device)
    conf2 = _conf(conf2, B * H2 * W2, desc1.device)
    S = seed_count(H1, W1, subsample)
    cap = S if capacity is None else int(capacity)
    dev = desc1.device
    if out_pairs is None:
        out_pairs = torch.empty((B, cap, 2), dtype=torch.int32, device=dev)
    if out_score is None:
        out_score = torch.empty((B, cap), dtype=_score_dtype(code), device=dev)
    if out_count is None:
        out_count = torch.empty(B, dtype=torch.int32, device=dev)
    if out_iters is None:
        out_iters = torch.empty(B, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_RECIPROCAL_MASKED, H1 * W1, H2 * W2, d, code, B, S)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_reciprocal_masked(
        _ptr(desc1), _ptr(conf1), H1, W1, _ptr(desc2), _ptr(conf2), H2, W2, d, code,
        float(threshold), subsample, max_iter, B, _ptr(out_pairs), _ptr(out_score), cap,
        _ptr(out_count), _ptr(out_iters), _ptr(out_frontier), _ptr(ws), nbytes, _stream(stream))
    _check(rc, "fastnn_reciprocal_masked")
    return out_pairs, out_score, out_count, out_iters


def fastnn_mutual_dense_masked(desc1: torch.Tensor, desc2: torch.Tensor,
                               conf1: torch.Tensor | None = None,
                               conf2: torch.Tensor | None = None, threshold: float = 0.0,
                               capacity: int | None = None, out_pairs=None, out_score=None,
                               out_count=None, workspace=None, stream=None):
    """Every mutual nearest-neighbour pair among the confident pixels of two maps."""
    _need_cuda(desc1, desc2)
    code = _dtype_code(desc1)
    desc1 = desc1.reshape(-1, desc1.shape[-1])
    desc2 = desc2.reshape(-1, desc2.shape[-1])
    n1, d = desc1.shape
    n2 = desc2.shape[0]
    conf1 = _conf(conf1, n1, desc1.device)
    conf2 = _conf(conf2, n2, desc1.device)
    cap = min(n1, n2) if capacity is None else int(capacity)
    dev = desc1.device
    if out_pairs is None:
        out_pairs = torch.empty((cap, 2), dtype=torch.int32, device=dev)
    if out_score is None:
        out_score = torch.empty(cap, dtype=_score_dtype(code), device=dev)
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
    nbytes = fastnn_workspace_size(FASTNN_OP_MUTUAL_DENSE_MASKED, n1, n2, d, code)
    ws = _workspace(nbytes, dev, workspace)
    rc = library().fastnn_mutual_dense_masked(
        _ptr(desc1), _ptr(conf1), n1, _ptr(desc2), _ptr(conf2), n2, d, code, float(threshold),
        _ptr(out_pairs), _ptr(out_score), cap, _ptr(out_count), _ptr(ws), nbytes,
        _stream(stream))
    _check(rc, "fastnn_mutual_dense_masked")
    return out_pairs, out_score, out_count


def fastnn_set_wait_timeout_ns(ns: int) -> None:
    """Limit of the kernels' bounded waits for later calls (0: the 2 s default)."""
    library().fastnn_set_wait_timeout_ns(int(ns))
