// Shared device helpers for the fastnn kernels (sm_100a).
//
// Score/index packing: a nearest-neighbour result is carried as one 64-bit
// key whose unsigned order is (score ascending, index descending):
//   key = (ordered_bits(score) << 32) | (0xFFFFFFFF - index)
// so the maximum key over a set of candidates is the highest score with the
// LOWEST index among equal scores, and partial results from any number of
// CTAs merge with one 64-bit atomicMax in any order, deterministically.
// key == 0 means "no candidate yet". Pointmap keys carry the score
// -(squared distance), so the maximum is the nearest point.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/fastnn.h"

namespace fastnn {

constexpr int kStatusTimeout = 1;  // bit set in the device status word
// Every bounded wait in the kernels (mbarrier phases, grid barriers) gives up
// after this long (or after NNArgs::wait_ns when set), sets kStatusTimeout
// and unwinds. The waits that drain in-flight copies and MMAs before a kernel
// exits always use kTimeoutNs.
constexpr uint64_t kTimeoutNs = 2000000000ull;

// A wait's limit: the configured one, or kTimeoutNs.
__host__ __device__ __forceinline__ uint64_t wait_limit(uint64_t configured) {
  return configured ? configured : kTimeoutNs;
}

__host__ __device__ __forceinline__ uint32_t ord_i32(int32_t s) {
  return static_cast<uint32_t>(s) ^ 0x80000000u;
}
__host__ __device__ __forceinline__ int32_t unord_i32(uint32_t h) {
  return static_cast<int32_t>(h ^ 0x80000000u);
}
__device__ __forceinline__ uint32_t ord_f32(float s) {
  s += 0.0f;  // -0 -> +0 so that equal scores share one key
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t h) {
  uint32_t u = (h & 0x80000000u) ? (h & 0x7FFFFFFFu) : ~h;
  return __uint_as_float(u);
}
__host__ __device__ __forceinline__ uint64_t make_key(uint32_t ord_score, uint32_t idx) {
  return (static_cast<uint64_t>(ord_score) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - idx);
}
__host__ __device__ __forceinline__ uint32_t key_index(uint64_t key) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(key);
}
__host__ __device__ __forceinline__ uint32_t key_score_bits(uint64_t key) {
  return static_cast<uint32_t>(key >> 32);
}

// Bytes of one repacked descriptor row: d elements zero-padded to K = 32
// (d <= 32) or K = 64 (d <= 64) elements of 1 (int8) or 2 (bf16, half) bytes.
// Pointmap rows (FASTNN_F32_L2, d <= 3) become one float4 (x, y, z, -|p|^2).
__host__ __device__ constexpr int elem_bytes(int dtype) {
  return dtype == FASTNN_I8 ? 1 : dtype == FASTNN_F32_L2 ? 4 : 2;
}
__host__ __device__ constexpr int row_bytes(int dtype, int d) {
  return dtype == FASTNN_F32_L2 ? 16 : elem_bytes(dtype) * (d <= 32 ? 32 : 64);
}


// Where the query rows of one nearest-neighbour pass come from.
//   row id of slot k of pair b:
//     q_index != nullptr : q_index[b * q_cap + k]
//     q_key   != nullptr : key_index(q_key[b * q_cap + k])   (chained pass)
//     otherwise          : k
//   rows live in q_rows + (b * q_rows_per_pair + row) * row_bytes.
//   Active slots of pair b: q_count ? q_count[b] : nq_static.
// Database rows per chunk of the pointmap kernels (a chunk's points also
// have a bounding box, for skipping chunks a query cannot be near).
constexpr int kL2Chunk = 1024;

struct NNArgs {
  const uint8_t* q_rows;
  int64_t q_rows_per_pair;
  const int32_t* q_index;
  const uint64_t* q_key;
  int64_t q_cap;
  const int32_t* q_count;
  int64_t nq_static;
  const uint8_t* db_rows;  // repacked database rows [batch][ndb][row_bytes]
  int64_t ndb;             // database rows per pair, and the stride between pairs
  const int32_t* ndb_dev;  // optional [batch]: pair b searches only its first ndb_dev[b]
                           // (<= ndb) rows (device counts of masked, compacted maps)
  uint64_t* out_key;       // [batch][q_cap], merged with atomicMax
  int batch;
  int* status;
  int d;                   // descriptor length (<= 64; <= 3 for pointmaps)
  const int* q_absmax;     // int8: max |element| of the query map (or nullptr)
  const int* db_absmax;    // int8: max |element| of the database map (or nullptr)
  uint64_t wait_ns;        // limit of the pipeline's bounded waits (0: kTimeoutNs)
  const uint32_t* q_bound; // optional [batch][q_cap]: ordered bits of a score each query is
                           // known to reach (0: none), for the standalone passes
  const float4* db_box;    // pointmaps, optional: [batch][ceil(ndb / kL2Chunk)][2] box (lo, hi)
                           // of each database chunk's points
};

// The parts of a pass's query description that change from round to round
// (the rest of NNArgs stays in kernel-parameter space).
struct PhaseQ {
  const int32_t* q_index;
  const int32_t* q_count;
  // Optional lower bound on each query's best score, as ordered score bits
  // (0: none) at bound[(b * q_cap + k) * bstride]: a score the query is known
  // to reach, so that only larger-or-equal scores need a record.
  const uint32_t* bound;
  int bstride;
  // 1: the CTA's per-pair count cache in shared memory already holds this
  // phase's query counts (read by the previous phase, or by the round loop's
  // check after the compaction), so the planner skips their load.
  int cached = 0;
};

// Counts, frontier indices and keys may have been written by other CTAs of
// the same (persistent) kernel: read them through L2 (ld.global.cg).
__device__ __forceinline__ int64_t nn_count(const NNArgs& a, const PhaseQ& q, int b) {
  return q.q_count ? static_cast<int64_t>(__ldcg(q.q_count + b)) : a.nq_static;
}

__device__ __forceinline__ int64_t nn_query_row(const NNArgs& a, const PhaseQ& q, int b,
                                                int64_t k) {
  if (q.q_index) return __ldcg(q.q_index + b * a.q_cap + k);
  if (a.q_key) return key_index(__ldcg(a.q_key + b * a.q_cap + k));
  return k;
}

}  // namespace fastnn

namespace fastnn {
// Records the most recent CUDA runtime error seen by the library (read with
// fastnn_last_cuda_error()).
void note_cuda_error(cudaError_t e);
}  // namespace fastnn

#define FASTNN_CUDA_TRY(expr)                              \
  do {                                                     \
    cudaError_t e_ = (expr);                               \
    if (e_ != cudaSuccess) {                               \
      ::fastnn::note_cuda_error(e_);                       \
      return FASTNN_ERR_CUDA;                              \
    }                                                      \
  } while (0)
