// Launcher of the tensor-core nearest-neighbour kernel (nn_tc.cu).
#pragma once

#include "common.cuh"

namespace fastnn {

// Smallest database row count the kernel's TMA descriptor accepts (one full
// tile); callers pad the repacked database to at least this many rows.
int nn_tc_min_rows();
// Largest batch (independent pairs) one launch takes.
int nn_tc_max_batch();

// Launch on `stream`. a.db_rows holds `db_total_rows` repacked rows (all
// pairs back to back plus zero padding), 16-byte aligned. Returns a
// fastnn_status.
// Benchmark instrumentation behind fastnn_kernel_timer_enable/_read.
int kernel_timer_enable(int capacity);
int kernel_timer_read(int* launches, double* total_ms);

int launch_nn_tc(const NNArgs& a, int dtype, int64_t db_total_rows, cudaStream_t stream);

}  // namespace fastnn
