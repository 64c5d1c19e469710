// Launcher of the tensor-core nearest-neighbour kernel (nn_tc.cu).
#pragma once

#include "common.cuh"
#include "frontier.cuh"

namespace fastnn {

// Everything the persistent fast-matching kernel needs (device pointers).
struct RecArgs {
  NNArgs fwd;        // forward pass template: queries = image-1 rows, database = image 2
  NNArgs bwd;        // backward pass template: queries = image-2 rows of the forward keys
  CompactArgs cmp;   // per-round check/compaction template
  int32_t* F[2];     // frontier ping-pong [batch][S]
  int32_t* cnt[2];   // frontier sizes ping-pong [batch]
  int64_t N1;        // pixels of image 1
  int64_t S;         // seeds per pair
  int W1, sub, max_iter, batch;
  uint32_t* grid_count;  // grid-barrier arrival counter (zero before the launch)
  int* grid_abort;       // set when any CTA gives up (zero before the launch)
  int* status;
};

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

// Cooperative launch of the persistent fast-matching kernel on `stream`.
// d1_rows / d2_rows: repacked rows (all pairs plus zero padding) behind
// r.bwd.db_rows / r.fwd.db_rows. Returns a fastnn_status.
int launch_reciprocal(const RecArgs& r, int dtype, int64_t d1_rows, int64_t d2_rows,
                      cudaStream_t stream);

}  // namespace fastnn
