// Launcher of the tensor-core nearest-neighbour kernel (nn_tc.cu).
#pragma once

#include "common.cuh"
#include "frontier.cuh"

namespace fastnn {

// Smallest database row count the kernel's TMA descriptor accepts (one full
// tile); callers pad the repacked database to at least this many rows.
int nn_tc_min_rows();
// Largest batch (independent pairs) one launch takes.
int nn_tc_max_batch();

// Launch on `stream`. a.db_rows holds `db_total_rows` repacked rows (all
// pairs back to back plus zero padding), 16-byte aligned. Returns a
// fastnn_status.
// Benchmark instrumentation behind fastnn_kernel_timer_enable/_select/_read.
// A launcher brackets its kernel(s) of one kind with kernel_timer_begin
// (returns a slot; -1 when the timer is off, full or not selecting that
// kind; -2 on a CUDA error) and kernel_timer_end.
constexpr int kTimeMatching = 1;  // nearest-neighbour and persistent matching kernels
constexpr int kTimeRepack = 2;    // repack of a descriptor map
constexpr int kTimeMutual = 4;    // mutual test and ordered emit (and the dense image list)
constexpr int kTimeMask = 8;      // confidence-mask compaction of a map
int kernel_timer_enable(int capacity);
int kernel_timer_select(int kinds);
int kernel_timer_read(int* launches, double* total_ms);
int kernel_timer_begin(cudaStream_t stream, int kind);
int kernel_timer_end(int slot, cudaStream_t stream);
// Multiprocessors of the current device.
int device_sm_count(int* sms);

int launch_nn_tc(const NNArgs& a, int dtype, int64_t db_total_rows, cudaStream_t stream);

// Cooperative launch of the persistent fast-matching kernel on `stream`.
// d1_rows / d2_rows: repacked rows (all pairs plus zero padding) behind
// r.bwd.db_rows / r.fwd.db_rows. Returns a fastnn_status.
int launch_reciprocal(const RecArgs& r, int dtype, int64_t d1_rows, int64_t d2_rows,
                      cudaStream_t stream);

}  // namespace fastnn
