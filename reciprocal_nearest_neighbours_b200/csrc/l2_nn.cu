// Nearest 3D point of pointmap rows on the FP32 pipes (sm_100a).
//
// Pointmap matching ("DUSt3R / MASt3R explained", the paragraph on recovering
// the cameras: pixels of two views match when their predicted 3D points are
// nearest neighbours in the shared frame) has d = 3, far too short a
// contraction for the tensor cores, so the scores are plain FP32 arithmetic.
// For a query a and a database point p
//     s(a, p) = 2<a, p> - |p|^2 = |a|^2 - |a - p|^2,
// so argmax_p s is the nearest point. A repacked row holds (x, y, z, -|p|^2)
// (the norm computed once per point by the repack kernel); one score is three
// fused multiply-adds, issued as FFMA2 on a pair of database rows, and a
// three-input max folds both scores of the pair into the running maximum.
//
// Work: units (pair b, 128-query tile m, 1024-row database chunk n), split
// into contiguous ranges over persistent CTAs of 16 warps. Each chunk comes
// into shared memory with one bulk copy on the TMA engine (double-buffered,
// completion on an mbarrier, every wait bounded). Each warp holds 8 queries
// in registers and its lanes stride over the chunk (lane l scores rows
// 64 s + l and 64 s + 32 + l). Per chunk a lane keeps only the maximum score
// of each query; when a warp vote finds a lane above the warp's best so far,
// the warp reduces the maximum, and all 32 lanes re-score the 32 rows of the
// lane holding it (same FMA order, so bit-identical scores) to find its
// first, i.e. lowest-index, row with that score. Consecutive chunks of one
// (pair, tile) form a segment; at its end lane q of each warp merges query
// q's (score, index) into the 64-bit key with atomicMax: the highest score
// (nearest point) with the lowest index, whatever the order of the merges.
#include <cuda_runtime.h>

#include "common.cuh"
#include "frontier_dev.cuh"
#include "l2_nn.cuh"
#include "nn_tc.cuh"
#include "ptx.cuh"

namespace fastnn {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kQW = 8;              // queries per warp, held by every lane
constexpr int kQT = kWarps * kQW;   // queries per tile
constexpr int kDC = 1024;           // database rows per chunk (16 KB)
constexpr int kSteps = kDC / 64;    // 64-row steps per chunk: two rows per lane per step
constexpr int kMaxBatchL2 = 1024;
constexpr unsigned kFull = 0xffffffffu;

struct __align__(16) L2Smem {
  float4 buf[2][kDC];
  unsigned long long bar[2];
  uint32_t bar_phase[2];
  int pending[2];  // a bulk copy into buffer i is in flight (thread 0's view)
  int abort_flag;
  int grid_ok;
  int more;
  int b0;
  long long nt, u0, u1, m0, n0;
  int scan[66];
  int cnt[kMaxBatchL2];
  int mt[kMaxBatchL2];
};

__device__ __forceinline__ void l2_setup(L2Smem& s) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(ptx::smem_u32(&s.bar[i]), 1);
      s.bar_phase[i] = 0;
      s.pending[i] = 0;
    }
    s.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
}

// Bounded wait for buffer i's copy. False when it ran out (status and the
// CTA's abort flag are raised) or the CTA already aborted.
__device__ __noinline__ bool l2_wait_slow(L2Smem& s, int i, uint32_t parity, int* status) {
  const uint32_t bar = ptx::smem_u32(&s.bar[i]);
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 255) == 0) {
      if (*reinterpret_cast<volatile int*>(&s.abort_flag)) return false;
      if (ptx::globaltimer_ns() - t0 > kTimeoutNs) {
        *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool l2_wait(L2Smem& s, int i, uint32_t parity, int* status) {
  if (ptx::mbar_try_wait(ptx::smem_u32(&s.bar[i]), parity)) return true;
  return l2_wait_slow(s, i, parity, status);
}

// Thread 0: wait (bounded) for copies still in flight so that none lands
// after the CTA has moved on; called before exit.
__device__ void l2_teardown(L2Smem& s, int* status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i)
      if (s.pending[i]) {
        const uint32_t bar = ptx::smem_u32(&s.bar[i]);
        const uint64_t t0 = ptx::globaltimer_ns();
        while (!ptx::mbar_try_wait(bar, s.bar_phase[i]))
          if (ptx::globaltimer_ns() - t0 > kTimeoutNs) {
            atomicOr(status, kStatusTimeout);
            break;
          }
        s.pending[i] = 0;
      }
  }
  __syncthreads();
}

// Thread 0: this CTA's contiguous range of units for one pass.
__device__ void l2_plan(const NNArgs& a, const PhaseQ& q, L2Smem& s) {
  const int64_t nt = (a.ndb + kDC - 1) / kDC;
  int64_t total = 0;
  for (int b = 0; b < a.batch; ++b) {
    const int64_t c = nn_count(a, q, b);
    s.cnt[b] = static_cast<int>(c);
    s.mt[b] = static_cast<int>((c + kQT - 1) / kQT);
    total += static_cast<int64_t>(s.mt[b]) * nt;
  }
  const int64_t G = gridDim.x;
  const int64_t u0 = total * blockIdx.x / G;
  s.nt = nt;
  s.u0 = u0;
  s.u1 = total * (blockIdx.x + 1) / G;
  int64_t acc = 0;
  int b = 0;
  while (b < a.batch && acc + static_cast<int64_t>(s.mt[b]) * nt <= u0) {
    acc += static_cast<int64_t>(s.mt[b]) * nt;
    ++b;
  }
  s.b0 = b;
  s.m0 = nt > 0 ? (u0 - acc) / nt : 0;
  s.n0 = nt > 0 ? (u0 - acc) % nt : 0;
}

// Thread 0: bring chunk n of pair b's database into buffer i.
__device__ __forceinline__ void l2_issue(const NNArgs& a, L2Smem& s, int i, int b, int64_t n) {
  const int64_t r0 = n * kDC;
  const int64_t rows = min(static_cast<int64_t>(kDC), a.ndb - r0);
  const uint32_t bytes = static_cast<uint32_t>(rows) * 16u;
  const uint32_t bar = ptx::smem_u32(&s.bar[i]);
  ptx::fence_proxy_async_smem();
  ptx::mbar_arrive_expect_tx(bar, bytes);
  ptx::bulk_load(ptx::smem_u32(&s.buf[i][0]), a.db_rows + (b * a.ndb + r0) * 16, bytes, bar);
  s.pending[i] = 1;
}

struct Queries {
  float2 x[kQW], y[kQW], z[kQW];  // (2 q, 2 q) per coordinate, both halves equal
};

__device__ __forceinline__ void load_queries(const NNArgs& a, const PhaseQ& q, int b, int64_t k0,
                                             int cnt, int lane, Queries& Q) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t k = k0 + lane;
  if (lane < kQW && k < cnt) {
    const int64_t row = nn_query_row(a, q, b, k);
    if (row >= 0 && row < a.q_rows_per_pair)
      v = __ldg(reinterpret_cast<const float4*>(a.q_rows) + b * a.q_rows_per_pair + row);
  }
#pragma unroll
  for (int i = 0; i < kQW; ++i) {
    const float x = 2.f * __shfl_sync(kFull, v.x, i);
    const float y = 2.f * __shfl_sync(kFull, v.y, i);
    const float z = 2.f * __shfl_sync(kFull, v.z, i);
    Q.x[i] = make_float2(x, x);
    Q.y[i] = make_float2(y, y);
    Q.z[i] = make_float2(z, z);
  }
}

// Scores of two rows against the 8 queries, folded into mx.
__device__ __forceinline__ void score_pair(const float4 p0, const float4 p1, const Queries& Q,
                                           float (&mx)[kQW]) {
  const float2 X = make_float2(p0.x, p1.x), Y = make_float2(p0.y, p1.y);
  const float2 Z = make_float2(p0.z, p1.z), N = make_float2(p0.w, p1.w);
#pragma unroll
  for (int i = 0; i < kQW; ++i) {
    float2 t = __ffma2_rn(Q.x[i], X, N);
    t = __ffma2_rn(Q.y[i], Y, t);
    t = __ffma2_rn(Q.z[i], Z, t);
    mx[i] = ptx::fmax3(mx[i], t.x, t.y);
  }
}

// One chunk (rows valid rows at database index base) for one warp.
__device__ __forceinline__ void l2_chunk(const float4* __restrict__ buf, int rows, uint32_t base,
                                         const Queries& Q, float (&best)[kQW],
                                         uint32_t (&bidx)[kQW], int lane) {
  float mx[kQW];
#pragma unroll
  for (int i = 0; i < kQW; ++i) mx[i] = -INFINITY;
  if (rows == kDC) {
#pragma unroll 2
    for (int st = 0; st < kSteps; ++st)
      score_pair(buf[64 * st + lane], buf[64 * st + 32 + lane], Q, mx);
  } else {
    // Ragged last chunk: missing rows score -inf (0 * q + -inf).
    const float4 never = make_float4(0.f, 0.f, 0.f, -INFINITY);
    for (int st = 0; 64 * st < rows; ++st) {
      const int j0 = 64 * st + lane, j1 = j0 + 32;
      score_pair(j0 < rows ? buf[j0] : never, j1 < rows ? buf[j1] : never, Q, mx);
    }
  }
#pragma unroll
  for (int i = 0; i < kQW; ++i) {
    if (!__any_sync(kFull, mx[i] > best[i])) continue;
    float M = mx[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    // Lanes holding the maximum; lane t re-scores the t-th row of each
    // (rows of lane L in increasing order: 64 (t >> 1) + 32 (t & 1) + L).
    unsigned cand = __ballot_sync(kFull, mx[i] == M);
    uint32_t J = 0xFFFFFFFFu;
    const int jt = 64 * (lane >> 1) + 32 * (lane & 1);
    while (cand) {
      const int L = __ffs(cand) - 1;
      cand &= cand - 1;
      float sc = -INFINITY;
      if (jt + L < rows) {
        const float4 p = buf[jt + L];
        sc = __fmaf_rn(Q.z[i].x, p.z, __fmaf_rn(Q.y[i].x, p.y, __fmaf_rn(Q.x[i].x, p.x, p.w)));
      }
      const unsigned hit = __ballot_sync(kFull, sc == M);
      if (hit) {
        const int t = __ffs(hit) - 1;
        J = min(J, static_cast<uint32_t>(64 * (t >> 1) + 32 * (t & 1) + L));
      }
    }
    if (J != 0xFFFFFFFFu) {
      best[i] = M;
      bidx[i] = base + J;
    }
  }
}

// One nearest-neighbour pass over this CTA's units; ends with a CTA barrier
// after which every result of the pass has been merged into a.out_key.
__device__ void l2_phase(const NNArgs& a, const PhaseQ q, L2Smem& s) {
  if (threadIdx.x == 0) l2_plan(a, q, s);
  __syncthreads();
  const int64_t u0 = s.u0, u1 = s.u1, nt = s.nt;
  if (u0 >= u1 || *reinterpret_cast<volatile int*>(&s.abort_flag)) {
    __syncthreads();
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t ph[2] = {s.bar_phase[0], s.bar_phase[1]};
  int b = s.b0;
  int64_t m = s.m0, n = s.n0;
  if (threadIdx.x == 0) l2_issue(a, s, 0, b, n);
  Queries Q;
  float best[kQW];
  uint32_t bidx[kQW];
  bool seg_start = true, ok = true;
  for (int64_t u = u0; u < u1; ++u) {
    const int i = static_cast<int>((u - u0) & 1);
    // Position of the next unit.
    int nb = b;
    int64_t nm = m, nn = n + 1;
    if (nn == nt) {
      nn = 0;
      if (++nm == s.mt[nb]) {
        nm = 0;
        do {
          ++nb;
        } while (nb < a.batch && s.mt[nb] == 0);
      }
    }
    if (threadIdx.x == 0 && u + 1 < u1) l2_issue(a, s, i ^ 1, nb, nn);
    const int64_t k0 = m * kQT + warp * kQW;
    const bool active = k0 < s.cnt[b];  // warp-uniform
    if (seg_start) {
      load_queries(a, q, b, k0, s.cnt[b], lane, Q);
#pragma unroll
      for (int j = 0; j < kQW; ++j) {
        best[j] = -INFINITY;
        bidx[j] = 0xFFFFFFFFu;
      }
    }
    ok = l2_wait(s, i, ph[i], a.status) && ok;
    ph[i] ^= 1u;
    if (threadIdx.x == 0 && ok) s.pending[i] = 0;
    const int rows = static_cast<int>(min(static_cast<int64_t>(kDC), a.ndb - n * kDC));
    if (active && ok) l2_chunk(s.buf[i], rows, static_cast<uint32_t>(n * kDC), Q, best, bidx, lane);
    const bool seg_end = (nn == 0) || (u + 1 == u1);
    if (seg_end && active && ok) {
#pragma unroll
      for (int j = 0; j < kQW; ++j)
        if (lane == j && k0 + j < s.cnt[b] && bidx[j] != 0xFFFFFFFFu)
          atomicMax(reinterpret_cast<unsigned long long*>(&a.out_key[b * a.q_cap + k0 + j]),
                    static_cast<unsigned long long>(make_key(ord_f32(best[j]), bidx[j])));
    }
    seg_start = seg_end;
    b = nb;
    m = nm;
    n = nn;
    // Buffer i is free for the copy issued at the top of the next iteration.
    if (!__syncthreads_and(ok)) break;
  }
  if (threadIdx.x == 0) {
    s.bar_phase[0] = ph[0];
    s.bar_phase[1] = ph[1];
    if (!ok) s.abort_flag = 1;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) nn_l2_kernel(const __grid_constant__ NNArgs a) {
  __shared__ L2Smem s;
  l2_setup(s);
  l2_phase(a, PhaseQ{a.q_index, a.q_count}, s);
  l2_teardown(s, a.status);
}

// Fast reciprocal matching of pointmaps: the shared round loop with the
// passes above.
__global__ void __launch_bounds__(kThreads, 1)
    reciprocal_l2_kernel(const __grid_constant__ RecArgs r) {
  __shared__ L2Smem s;
  l2_setup(s);
  auto pass = [&](int dir, const PhaseQ& q) { l2_phase(dir == 0 ? r.fwd : r.bwd, q, s); };
  fast_rounds<FASTNN_F32_L2>(r, pass, &s.abort_flag, &s.grid_ok, &s.more, s.scan);
  l2_teardown(s, r.status);
}

}  // namespace

int nn_l2_max_batch() { return kMaxBatchL2; }

int launch_nn_l2(const NNArgs& a, cudaStream_t stream) {
  if (a.batch < 1 || a.batch > kMaxBatchL2 || a.ndb < 1) return FASTNN_ERR_INVALID;
  int sms = 0, rc = device_sm_count(&sms);
  if (rc != FASTNN_OK) return rc;
  const int slot = kernel_timer_begin(stream);
  if (slot == -2) return FASTNN_ERR_CUDA;
  nn_l2_kernel<<<sms, kThreads, 0, stream>>>(a);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return kernel_timer_end(slot, stream);
}

int launch_reciprocal_l2(const RecArgs& r, cudaStream_t stream) {
  if (r.batch < 1 || r.batch > kMaxBatchL2 || r.fwd.ndb < 1 || r.bwd.ndb < 1)
    return FASTNN_ERR_INVALID;
  int sms = 0, rc = device_sm_count(&sms);
  if (rc != FASTNN_OK) return rc;
  const void* fn = reinterpret_cast<const void*>(reciprocal_l2_kernel);
  int per_sm = 0;
  FASTNN_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0));
  if (per_sm < 1) return FASTNN_ERR_UNSUPPORTED;
  RecArgs args = r;
  void* params[] = {&args};
  const int slot = kernel_timer_begin(stream);
  if (slot == -2) return FASTNN_ERR_CUDA;
  FASTNN_CUDA_TRY(cudaLaunchCooperativeKernel(fn, dim3(sms), dim3(kThreads), params, 0, stream));
  return kernel_timer_end(slot, stream);
}

}  // namespace fastnn
