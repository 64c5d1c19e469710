"""Host-side checks of the C ABI (no GPU, no compute calls).

The library must load, export every function include/fastnn.h declares, size
workspaces consistently, and reject bad arguments on the host before it
touches the device.
"""

from __future__ import annotations

import ctypes
import os
import re

import pytest

import reciprocal_nearest_neighbours_b200 as fnn
from reciprocal_nearest_neighbours_b200 import build as fnn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    fnn_build.build()
    return fnn.library()


def _declared():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(fastnn_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"fastnn_nn", "fastnn_reciprocal", "fastnn_mutual_dense",
            "fastnn_workspace_size", "fastnn_device_status", "fastnn_status_str"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings(lib):
    assert fnn.fastnn_status_str(0) == "FASTNN_OK"
    assert fnn.fastnn_status_str(-3) == "FASTNN_ERR_CAPACITY"
    assert fnn.fastnn_status_str(-5) == "FASTNN_ERR_TIMEOUT"
    assert fnn.fastnn_status_str(42) == "FASTNN_UNKNOWN_STATUS"


def test_workspace_sizes(lib):
    ws = fnn.fastnn_workspace_size
    a = ws(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 24, fnn.FASTNN_I8, 1, 3072)
    b = ws(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 24, fnn.FASTNN_BF16, 1, 3072)
    c = ws(fnn.FASTNN_OP_RECIPROCAL, 147456, 147456, 32, fnn.FASTNN_I8, 16, 9216)
    assert 0 < a < b and c > 16 * a // 2
    assert a % 256 == 0
    # int8 repacked maps: 2 x (N + 256) rows x 32 B, plus claims and frontier state
    assert a >= 2 * (196608 + 256) * 32 + 196608 * 4
    assert ws(fnn.FASTNN_OP_NN, 10, 1000, 24, fnn.FASTNN_I8) > 1000 * 32
    assert ws(fnn.FASTNN_OP_MUTUAL_DENSE, 3072, 3072, 24, fnn.FASTNN_I8) > 2 * 3072 * 40
    # half descriptors take the bf16 layout; 32 < d <= 64 doubles the repacked rows
    assert ws(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 24, fnn.FASTNN_F16, 1, 3072) == b
    e = ws(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 64, fnn.FASTNN_I8, 1, 3072)
    assert e == b and e - a >= 2 * 196608 * 32
    assert ws(fnn.FASTNN_OP_NN, 10, 1000, 48, fnn.FASTNN_BF16) > 1000 * 128
    # pointmaps: one 16-byte row per point, d <= 3
    assert ws(fnn.FASTNN_OP_NN, 10, 1000, 3, fnn.FASTNN_F32_L2) > 1000 * 16
    assert ws(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 3, fnn.FASTNN_F32_L2, 1, 3072) > \
        2 * 196608 * 16
    assert ws(fnn.FASTNN_OP_NN, 10, 10, 4, fnn.FASTNN_F32_L2) == 0
    # masked ops: the unmasked workspace plus compaction state
    am = ws(fnn.FASTNN_OP_RECIPROCAL_MASKED, 196608, 196608, 24, fnn.FASTNN_I8, 1, 3072)
    assert am >= a + 3 * 196608 * 4
    dm = ws(fnn.FASTNN_OP_MUTUAL_DENSE_MASKED, 3072, 3072, 24, fnn.FASTNN_I8)
    assert dm > ws(fnn.FASTNN_OP_MUTUAL_DENSE, 3072, 3072, 24, fnn.FASTNN_I8) + 2 * 3072 * 4
    # unsupported arguments size to 0
    assert ws(fnn.FASTNN_OP_NN, 10, 10, 65, fnn.FASTNN_I8) == 0
    assert ws(fnn.FASTNN_OP_NN, 10, 10, 65, fnn.FASTNN_F16) == 0
    assert ws(fnn.FASTNN_OP_NN, 10, 10, 0, fnn.FASTNN_I8) == 0
    assert ws(fnn.FASTNN_OP_NN, 10, 10, 24, 7) == 0
    assert ws(7, 10, 10, 24, fnn.FASTNN_I8) == 0
    assert ws(fnn.FASTNN_OP_RECIPROCAL, 10, 10, 24, fnn.FASTNN_I8, 0, 5) == 0


def test_argument_errors_are_reported_on_the_host(lib):
    """Every call here fails validation before any CUDA API is reached."""
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: validation rejects first
    big = 1 << 30
    I8 = fnn.FASTNN_I8
    # unsupported d / dtype
    assert lib.fastnn_nn(fake, 4, fake, 4, 65, I8, fake, None, fake, big, None) == -2
    assert lib.fastnn_nn(fake, 4, fake, 4, 0, fnn.FASTNN_F16, fake, None, fake, big, None) == -2
    assert lib.fastnn_nn(fake, 4, fake, 4, 4, fnn.FASTNN_F32_L2, fake, None, fake, big, None) == -2
    assert lib.fastnn_nn(fake, 4, fake, 4, 24, 5, fake, None, fake, big, None) == -2
    # empty query set is a no-op, even with null pointers
    assert lib.fastnn_nn(None, 0, None, 4, 24, I8, None, None, None, 0, None) == 0
    # empty database, null output, misaligned workspace, small workspace
    assert lib.fastnn_nn(fake, 4, fake, 0, 24, I8, fake, None, fake, big, None) == -1
    assert lib.fastnn_nn(fake, 4, fake, 4, 24, I8, None, None, fake, big, None) == -1
    assert lib.fastnn_nn(fake, 4, fake, 4, 24, I8, fake, None, P((1 << 20) + 8), big, None) == -1
    assert lib.fastnn_nn(fake, 4, fake, 4, 24, I8, fake, None, fake, 16, None) == -3
    # reciprocal: capacity below the seed count, bad rounds, bad batch
    rec = lib.fastnn_reciprocal
    S = fnn.seed_count(48, 64, 8)
    assert S == 48
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 8, 10, 1, fake, None, S - 1, fake, None,
               None, fake, big, None) == -3
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 8, 0, 1, fake, None, S, fake, None,
               None, fake, big, None) == -1
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 8, 256, 1, fake, None, S, fake, None,
               None, fake, big, None) == -1
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 0, 10, 1, fake, None, S, fake, None,
               None, fake, big, None) == -1
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 8, 10, 0, fake, None, S, fake, None,
               None, fake, big, None) == -1
    assert rec(fake, 48, 64, fake, 48, 64, 24, I8, 8, 10, 1, fake, None, S, fake, None,
               None, fake, 64, None) == -3
    # masked calls: a NaN threshold, then the unmasked calls' own checks
    nan = float("nan")
    recm = lib.fastnn_reciprocal_masked
    assert recm(fake, None, 48, 64, fake, None, 48, 64, 24, I8, nan, 8, 10, 1, fake, None, S,
                fake, None, None, fake, big, None) == -1
    assert recm(fake, None, 48, 64, fake, None, 48, 64, 24, I8, 1.0, 8, 10, 1, fake, None, S - 1,
                fake, None, None, fake, big, None) == -3
    assert recm(fake, None, 48, 64, fake, None, 48, 64, 65, I8, 1.0, 8, 10, 1, fake, None, S,
                fake, None, None, fake, big, None) == -2
    mutm = lib.fastnn_mutual_dense_masked
    assert mutm(fake, None, 100, fake, None, 50, 24, I8, nan, fake, None, 50, fake, fake, big,
                None) == -1
    assert mutm(fake, None, 100, fake, None, 50, 24, I8, 0.5, fake, None, 49, fake, fake, big,
                None) == -3
    # dense: capacity below min(n1, n2)
    mut = lib.fastnn_mutual_dense
    assert mut(fake, 100, fake, 50, 24, I8, fake, None, 49, fake, fake, big, None) == -3
    assert mut(fake, 0, fake, 50, 24, I8, fake, None, 49, fake, fake, big, None) == -1
    assert mut(fake, 100, fake, 50, 24, I8, None, None, 50, fake, fake, big, None) == -1


def test_noalloc_argument_errors_are_reported_on_the_host(lib):
    """The allocation-free entry point rejects bad arguments, with
    fastnn_reciprocal's statuses, before its first CUDA call (the scratch
    lookup): every call here returns without touching a device."""
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: validation rejects first
    I8 = fnn.FASTNN_I8
    na = lib.fastnn_reciprocal_noalloc
    S = fnn.seed_count(48, 64, 8)
    count = (ctypes.c_int32 * 16)(*([-7] * 16))
    cnt = ctypes.cast(count, P)

    def call(H1=48, W1=64, H2=48, W2=64, d=24, dt=I8, sub=8, it=10, batch=1, cap=S,
             pairs=fake, d1=fake):
        return na(d1, H1, W1, fake, H2, W2, d, dt, sub, it, batch, pairs, None, cap, cnt,
                  None, None, None)
    # bad sizes, rounds, batch and pointers: FASTNN_ERR_INVALID
    assert call(sub=0) == -1
    assert call(H1=0) == -1 and call(W2=0) == -1
    assert call(batch=0) == -1
    assert call(it=0) == -1 and call(it=256) == -1
    assert call(pairs=None) == -1 and call(d1=None) == -1
    # unsupported d or dtype: FASTNN_ERR_UNSUPPORTED, as fastnn_reciprocal says
    assert call(d=65) == -2 and call(d=0) == -2 and call(dt=9) == -2
    assert call(d=4, dt=fnn.FASTNN_F32_L2) == -2
    rec = lib.fastnn_reciprocal
    assert rec(fake, 48, 64, fake, 48, 64, 65, I8, 8, 10, 1, fake, None, S, fake, None, None,
               fake, 1 << 30, None) == -2
    # capacity below the seed count, and workloads beyond the scratch array
    assert call(cap=S - 1) == -3
    need = fnn.fastnn_workspace_size(fnn.FASTNN_OP_RECIPROCAL, 288 * 512, 288 * 512, 32, I8,
                                     16, 9216)
    assert need > (32 << 20)
    assert call(H1=288, W1=512, H2=288, W2=512, d=32, sub=4, it=15, batch=16, cap=9216) == -3
    # one 512x384 pair fits (int8 and bf16); nothing was written by any call above
    assert fnn.fastnn_workspace_size(fnn.FASTNN_OP_RECIPROCAL, 196608, 196608, 24,
                                     fnn.FASTNN_BF16, 1, 3072) <= (32 << 20)
    assert list(count) == [-7] * 16
