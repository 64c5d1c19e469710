// Launchers of the pointmap (nearest 3D point) kernels (l2_nn.cu).
#pragma once

#include "common.cuh"
#include "frontier.cuh"

namespace fastnn {

// Nearest point of every query row: a.q_rows / a.db_rows hold repacked
// float4 rows (x, y, z, -|p|^2), a.ndb rows per pair. Keys merge into
// a.out_key (zeroed by the caller) with atomicMax. Returns a fastnn_status.
int launch_nn_l2(const NNArgs& a, cudaStream_t stream);

// Cooperative launch of the persistent fast-matching kernel for pointmaps.
int launch_reciprocal_l2(const RecArgs& r, cudaStream_t stream);

// Largest batch (independent pairs) one launch takes.
int nn_l2_max_batch();

}  // namespace fastnn
