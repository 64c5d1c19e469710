"""B200-native reciprocal nearest-neighbour matching of dense descriptor maps.

Python binding of ``libfastnn.so`` (declared in ``include/fastnn.h``). The
functions here only marshal arguments: they take CUDA tensors, allocate the
outputs and the workspace with PyTorch when the caller does not pass them, and
call the C ABI on the current CUDA stream. Every step of the matching runs in
the library's sm_100a kernels; there is no other implementation to fall back
to, and loading fails loudly when the library is missing.
"""

from __future__ import annotations

from ._lib import (  # noqa: F401
    FASTNN_BF16,
    FASTNN_F16,
    FASTNN_F32_L2,
    FASTNN_I8,
    FASTNN_OP_MUTUAL_DENSE,
    FASTNN_OP_IMAGE_ROWS,
    FASTNN_OP_MUTUAL_DENSE_MASKED,
    FASTNN_OP_MUTUAL_FROM_NN,
    FASTNN_OP_NN,
    FASTNN_OP_RECIPROCAL,
    FASTNN_OP_RECIPROCAL_MASKED,
    FASTNN_TIME_MASK,
    FASTNN_TIME_MATCHING,
    FASTNN_TIME_MUTUAL,
    FASTNN_TIME_REPACK,
    FastNNError,
    fastnn_device_status,
    fastnn_image_rows,
    fastnn_kernel_timer_enable,
    fastnn_kernel_timer_read,
    fastnn_kernel_timer_select,
    fastnn_mutual_dense,
    fastnn_mutual_dense_masked,
    fastnn_mutual_from_nn,
    fastnn_nn,
    fastnn_noalloc_device_status,
    fastnn_reciprocal,
    fastnn_reciprocal_masked,
    fastnn_reciprocal_noalloc,
    fastnn_set_wait_timeout_ns,
    fastnn_status_str,
    fastnn_workspace_size,
    library,
    library_path,
    seed_count,
)
