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
// fused multiply-adds, and a three-input max folds the scores of two rows
// into the running maximum. (Packed FFMA2 on pairs of rows measured no
// faster on B200: the packing moves cost more than they save, and with a
// pre-paired layout the gain was 3%.)
//
// Exact ranking. The fp32 score s~ is within E = 8 u (|a| + R)^2 of s
// (u = 2^-24, R = the largest |p| of the database, measured by the repack
// kernel; the rounding analysis of the six operations gives 6 u plus
// second-order terms). A point whose s~ is more than 2E below the largest s~
// seen cannot be the nearest, so only the points inside that window are
// ranked again, by their squared distance computed in fp64 from the
// coordinate differences -- (dx^2 + dy^2) + dz^2, each operation rounded
// once, the order of a plain loop over the coordinates. Within the share of
// the database one CTA scans, the winner is the smallest fp64 value, lowest
// index among exact ties (the definition). Winners of different CTAs are
// merged on the fp64 value rounded to fp32, lowest index among equal fp32
// values, and the score reported is that fp32 value; the two rules can
// differ only for two points in different CTAs' shares whose fp64 distances
// differ yet round to one fp32 value. In the fast scheme's passes a query usually
// comes with the fp32 distance D of a point it is known to reach (its partner
// in the previous pass); the window then starts at the floor that D implies
// instead of opening at every chunk until a near point has been seen.
//
// Work: units (pair b, 128-query tile m, 1024-row database chunk n), split
// into contiguous ranges over persistent CTAs of 16 warps. Chunks come into a
// 4-deep ring of shared-memory buffers by bulk copies on the TMA engine,
// completing on one mbarrier per buffer (every wait bounded). There is no
// CTA-wide barrier per chunk: each warp counts itself out of a buffer when it
// is done with it, and the last warp out issues the copy of the unit four
// ahead into it, so warps drift up to three chunks apart and uneven work
// evens out. Each warp holds 8 queries in registers and its lanes stride over
// the chunk (lane l scores rows 64 s + l and 64 s + 32 + l). Per chunk a lane
// keeps only the maximum s~ of each query; a warp vote asks whether any lane
// reached the query's window. Only then does the warp reduce the maximum and
// walk the lanes inside the window: all 32 lanes re-score the 32 rows of one
// such lane (same FMA order, so bit-identical s~), rank the rows inside the
// window by fp64 distance and keep the best (fp64 distance, index) as the
// query's winner. Consecutive units of one (pair, tile) form a segment,
// visiting the database chunks in a scrambled order (the ranking does not
// depend on the order, and spatially ordered rows would otherwise open the
// re-ranking at nearly every chunk); at its end lane q of each warp merges
// query q's winner into the 64-bit key with atomicMax on (ordered -distance,
// inverted index): the nearest point with the lowest index, whatever the
// order of the merges.
#include <cfloat>
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
constexpr int kDC = kL2Chunk;       // database rows per chunk (16 KB)
constexpr int kSteps = kDC / 64;    // 64-row steps per chunk: two rows per lane per step
constexpr int kNS = 4;              // chunk ring depth
constexpr int kMaxBatchL2 = 1024;
constexpr unsigned kFull = 0xffffffffu;

// Per-warp, per-query state of the exact ranking that only a vote that fires
// touches (warp-uniform values).
struct WarpState {
  unsigned long long dbits[kQW];  // winner's exact fp64 squared distance (bits; ~0: none)
  uint32_t idx[kQW];              // winner's index (lowest among exact ties)
  float smax[kQW];              // largest fp32 score s~ seen in the segment
  float win2[kQW];              // window width 2E
  float floor[kQW];             // lowest window edge the query's bound allows, or -FLT_MAX
  float4 qlo, qhi;              // box of the warp's queries; qlo.w = largest bound distance
                                // (+inf if a query has none)
};

struct __align__(16) L2Smem {
  float4 buf[kNS][kDC];
  WarpState ws[kWarps];
  unsigned long long bar[kNS];
  uint32_t bar_phase[kNS];  // consumers' next parity per buffer, carried across passes
  uint32_t issued[kNS];     // copies issued into each buffer (teardown waits for the last)
  int empty_cnt[kNS];       // warps done with the buffer's current chunk
  int abort_flag;
  int grid_ok;
  int b0;
  unsigned long long wait_ns;  // limit of the pipeline's bounded waits
  long long u0, u1, m0, n0;
  int scan[66];
  int cnt[kMaxBatchL2];   // queries per pair
  int mt[kMaxBatchL2];    // query tiles per pair (0 when the pair has no database row)
  int nt[kMaxBatchL2];    // database chunks per pair
  int rows[kMaxBatchL2];  // database rows per pair
  int step[kMaxBatchL2];  // chunk n of a segment is chunk (n * step) mod nt; step < nt
};

constexpr size_t kSmemBytes = sizeof(L2Smem);

__device__ __forceinline__ L2Smem& l2_smem() {
  extern __shared__ __align__(16) unsigned char l2_dyn[];
  return *reinterpret_cast<L2Smem*>(l2_dyn);
}

__device__ __forceinline__ void l2_setup(L2Smem& s) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      ptx::mbar_init(ptx::smem_u32(&s.bar[i]), 1);
      s.bar_phase[i] = 0;
      s.issued[i] = 0;
      s.empty_cnt[i] = 0;
    }
    s.abort_flag = 0;
    s.wait_ns = kTimeoutNs;
    ptx::fence_mbar_init();
  }
  __syncthreads();
}

// Bounded wait for buffer i's copy. False when it ran out (status and the
// CTA's abort flag are raised) or the CTA already aborted.
__device__ __noinline__ bool l2_wait_slow(L2Smem& s, int i, uint32_t parity, int* status) {
  const uint32_t bar = ptx::smem_u32(&s.bar[i]);
  const uint64_t t0 = ptx::globaltimer_ns();
  const uint64_t limit = s.wait_ns;
  for (uint32_t n = 1;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 255) == 0 || n == 8) {
      if (*reinterpret_cast<volatile int*>(&s.abort_flag)) return false;
      if (ptx::globaltimer_ns() - t0 > limit) {
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

// Thread 0: wait (bounded) for the last copy issued into every buffer, so
// that none lands after the CTA has exited; called before exit.
__device__ void l2_teardown(L2Smem& s, int* status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i)
      if (s.issued[i]) {
        const uint32_t bar = ptx::smem_u32(&s.bar[i]);
        const uint32_t parity = (s.issued[i] - 1u) & 1u;
        const uint64_t t0 = ptx::globaltimer_ns();
        while (!ptx::mbar_try_wait(bar, parity))
          if (ptx::globaltimer_ns() - t0 > kTimeoutNs) {
            atomicOr(status, kStatusTimeout);
            break;
          }
      }
  }
  __syncthreads();
}

// Position of a unit: pair b, query tile m, position n in the segment and
// the database chunk c it visits.
struct Walk {
  int b;
  int64_t m, n, c;
};

__device__ __forceinline__ void walk_next(Walk& w, const L2Smem& s, int batch) {
  const int nt = s.nt[w.b];
  ++w.n;
  w.c += s.step[w.b];
  if (w.c >= nt) w.c -= nt;
  if (w.n == nt) {
    w.n = 0;
    w.c = 0;
    if (++w.m == s.mt[w.b]) {
      w.m = 0;
      do {
        ++w.b;
      } while (w.b < batch && s.mt[w.b] == 0);
    }
  }
}

// Issue the copy of database chunk w.c of pair w.b into buffer i.
__device__ __forceinline__ void l2_issue(const NNArgs& a, L2Smem& s, int i, const Walk& w) {
  const int64_t r0 = w.c * kDC;
  const int64_t rows = min(static_cast<int64_t>(kDC), s.rows[w.b] - r0);
  const uint32_t bytes = static_cast<uint32_t>(rows) * 16u;
  const uint32_t bar = ptx::smem_u32(&s.bar[i]);
  ptx::fence_proxy_async_smem();
  ptx::mbar_arrive_expect_tx(bar, bytes);
  ptx::bulk_load(ptx::smem_u32(&s.buf[i][0]), a.db_rows + (w.b * a.ndb + r0) * 16, bytes, bar);
  s.issued[i] += 1u;
}

__device__ __forceinline__ int gcd_i(int x, int y) {
  while (y) {
    const int t = x % y;
    x = y;
    y = t;
  }
  return x;
}

// Thread 0: this CTA's contiguous range of units for one pass, and the
// copies of its first kNS units.
__device__ void l2_plan(const NNArgs& a, const PhaseQ& q, L2Smem& s) {
  s.wait_ns = wait_limit(a.wait_ns);
  int64_t total = 0;
  for (int b = 0; b < a.batch; ++b) {
    const int64_t c = q.cached ? s.cnt[b] : nn_count(a, q, b);
    const int64_t rows = a.ndb_dev ? min(static_cast<int64_t>(__ldcg(a.ndb_dev + b)), a.ndb)
                                   : a.ndb;
    const int nt = static_cast<int>(rows > 0 ? (rows + kDC - 1) / kDC : 0);
    s.cnt[b] = static_cast<int>(c);
    s.rows[b] = static_cast<int>(rows);
    s.nt[b] = nt;
    s.mt[b] = nt > 0 ? static_cast<int>((c + kQT - 1) / kQT) : 0;
    // A stride coprime with nt near 0.618 nt scatters the chunks of every
    // segment over the database: rows of a pointmap are spatially ordered,
    // and in storage order nearly every chunk would bring a point nearer
    // than all before it, each time opening the exact re-ranking.
    int st = nt > 1 ? static_cast<int>(0.618 * nt) : 0;
    if (nt > 1) {
      if (st < 1) st = 1;
      while (gcd_i(st, nt) != 1) ++st;
      st %= nt;
    }
    s.step[b] = st;
    total += static_cast<int64_t>(s.mt[b]) * nt;
  }
  const int64_t G = gridDim.x;
  const int64_t u0 = total * blockIdx.x / G;
  s.u0 = u0;
  s.u1 = total * (blockIdx.x + 1) / G;
  int64_t acc = 0;
  int b = 0;
  while (b < a.batch && acc + static_cast<int64_t>(s.mt[b]) * s.nt[b] <= u0) {
    acc += static_cast<int64_t>(s.mt[b]) * s.nt[b];
    ++b;
  }
  const int64_t nt = b < a.batch ? s.nt[b] : 0;
  s.b0 = b;
  s.m0 = nt > 0 ? (u0 - acc) / nt : 0;
  s.n0 = nt > 0 ? (u0 - acc) % nt : 0;
  if (!s.abort_flag && u0 < s.u1) {
    Walk w{b, s.m0, s.n0, (s.n0 * s.step[b]) % nt};
    for (int64_t u = u0; u < s.u1 && u < u0 + kNS; ++u) {
      l2_issue(a, s, static_cast<int>(u - u0), w);
      walk_next(w, s, a.batch);
    }
  }
}

struct Queries {
  float x[kQW], y[kQW], z[kQW];  // 2 q per coordinate
};

// Per-query lower edge of the re-ranking window, max(smax - 2E, floor), or
// the floor before any score (warp-uniform values, read every chunk).
struct Window {
  float thr[kQW];
};

// Loads the warp's 8 queries and resets its ranking state. max_p2 = largest
// |p|^2 (fp32) over the database.
__device__ __forceinline__ void load_queries(const NNArgs& a, const PhaseQ& q, int b, int64_t k0,
                                             int cnt, int lane, float max_p2, WarpState& W,
                                             Queries& Q, Window& Wn) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t k = k0 + lane;
  uint32_t bound = 0u;
  if (lane < kQW && k < cnt) {
    const int64_t row = nn_query_row(a, q, b, k);
    if (row >= 0 && row < a.q_rows_per_pair)
      v = __ldg(reinterpret_cast<const float4*>(a.q_rows) + b * a.q_rows_per_pair + row);
    if (q.bound) bound = __ldcg(q.bound + (b * a.q_cap + k) * q.bstride);
  }
  float floor = -FLT_MAX;
  // Box of the warp's queries and the largest of their bound distances
  // (+inf if one has none): a chunk whose box is farther from this box than
  // that holds none of their answers.
  const bool valid = lane < kQW && k < cnt;
  float lx = valid ? v.x : INFINITY, ly = valid ? v.y : INFINITY, lz = valid ? v.z : INFINITY;
  float hx = valid ? v.x : -INFINITY, hy = valid ? v.y : -INFINITY, hz = valid ? v.z : -INFINITY;
  float bd = valid ? (bound != 0u ? -unord_f32(bound) : INFINITY) : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lx = fminf(lx, __shfl_xor_sync(kFull, lx, o));
    ly = fminf(ly, __shfl_xor_sync(kFull, ly, o));
    lz = fminf(lz, __shfl_xor_sync(kFull, lz, o));
    hx = fmaxf(hx, __shfl_xor_sync(kFull, hx, o));
    hy = fmaxf(hy, __shfl_xor_sync(kFull, hy, o));
    hz = fmaxf(hz, __shfl_xor_sync(kFull, hz, o));
    bd = fmaxf(bd, __shfl_xor_sync(kFull, bd, o));
  }
  if (lane == 0) {
    W.qlo = make_float4(lx, ly, lz, bd);
    W.qhi = make_float4(hx, hy, hz, 0.f);
  }
  if (lane < kQW) {
    // 2E = 16 u (|a| + R)^2; the norms come from fp32 sums (relative error
    // below 3 u), inflated by 2^-20 to stay an upper bound.
    const float ra = sqrtf(fmaxf(-v.w, 0.f)) * (1.f + 0x1p-20f);
    const float rp = sqrtf(max_p2) * (1.f + 0x1p-20f);
    const float win2 = 0x1p-20f * (ra + rp) * (ra + rp) * (1.f + 0x1p-20f);
    // A bound (ordered bits of -D, D the fp32 distance of a point this query
    // is known to reach) means the answer r has |a - r|^2 <= D (1 + 2u), so
    // s(r) >= |a|^2 - D (1 + 2u) and s~(r) >= that - E. The floor lowers
    // both terms by 2^-20 (16 u, above the rounding of |a|^2, of D and of
    // these operations) and subtracts 2E.
    if (bound != 0u) {
      const float D = -unord_f32(bound);
      floor = (-v.w) * (1.f - 0x1p-20f) - D * (1.f + 0x1p-20f) - win2;
    }
    W.win2[lane] = win2;
    W.floor[lane] = floor;
    W.smax[lane] = -INFINITY;
    W.dbits[lane] = ~0ull;
    W.idx[lane] = 0xFFFFFFFFu;
  }
#pragma unroll
  for (int i = 0; i < kQW; ++i) {
    Q.x[i] = 2.f * __shfl_sync(kFull, v.x, i);
    Q.y[i] = 2.f * __shfl_sync(kFull, v.y, i);
    Q.z[i] = 2.f * __shfl_sync(kFull, v.z, i);
    Wn.thr[i] = __shfl_sync(kFull, floor, i);
  }
  __syncwarp();
}

// Score of point p for query i (2q scaled): 2<q, p> - |p|^2.
__device__ __forceinline__ float l2_score(const Queries& Q, int i, const float4 p) {
  return __fmaf_rn(Q.z[i], p.z, __fmaf_rn(Q.y[i], p.y, __fmaf_rn(Q.x[i], p.x, p.w)));
}

// Scores of two rows against the 8 queries, folded into mx.
__device__ __forceinline__ void score_pair(const float4 p0, const float4 p1, const Queries& Q,
                                           float (&mx)[kQW]) {
#pragma unroll
  for (int i = 0; i < kQW; ++i) mx[i] = ptx::fmax3(mx[i], l2_score(Q, i, p0), l2_score(Q, i, p1));
}

// fp64 squared distance of query (ax, ay, az) and point p in the order of a
// plain loop over the coordinates, one rounding per operation.
__device__ __forceinline__ double dist2_f64(float ax, float ay, float az, const float4 p) {
  const double dx = __dsub_rn(static_cast<double>(ax), static_cast<double>(p.x));
  const double dy = __dsub_rn(static_cast<double>(ay), static_cast<double>(p.y));
  const double dz = __dsub_rn(static_cast<double>(az), static_cast<double>(p.z));
  return __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
}

// One chunk (rows valid rows at database index base) for one warp.
__device__ __forceinline__ void l2_chunk(const float4* __restrict__ buf, int rows, uint32_t base,
                                         const Queries& Q, Window& Wn, WarpState& W, int lane) {
  float mx[kQW];
#pragma unroll
  for (int i = 0; i < kQW; ++i) mx[i] = -INFINITY;
  if (rows == kDC) {
#pragma unroll 4
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
  // Row t of lane L in increasing order: 64 (t >> 1) + 32 (t & 1) + L.
  const int jt = 64 * (lane >> 1) + 32 * (lane & 1);
#pragma unroll
  for (int i = 0; i < kQW; ++i) {
    if (!__any_sync(kFull, mx[i] >= Wn.thr[i])) continue;
    float M = mx[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    const float smax = fmaxf(W.smax[i], M);
    const float thr = fmaxf(smax - W.win2[i], W.floor[i]);
    Wn.thr[i] = thr;
    const float ax = 0.5f * Q.x[i], ay = 0.5f * Q.y[i], az = 0.5f * Q.z[i];
    unsigned long long best = W.dbits[i];
    uint32_t best_j = W.idx[i];
    unsigned cand = __ballot_sync(kFull, mx[i] >= thr);
    while (cand) {
      const int L = __ffs(cand) - 1;
      cand &= cand - 1;
      // The exact fp64 squared distance of this lane's row (bits: non-negative
      // doubles order like their bits; ~0 outside the window) and its index;
      // the warp minimum of (distance, index) in three 32-bit reductions.
      unsigned long long db = ~0ull;
      uint32_t jidx = 0xFFFFFFFFu;
      const int j = jt + L;
      if (j < rows) {
        const float4 p = buf[j];
        if (l2_score(Q, i, p) >= thr) {
          db = static_cast<unsigned long long>(__double_as_longlong(dist2_f64(ax, ay, az, p)));
          jidx = base + static_cast<uint32_t>(j);
        }
      }
      const uint32_t hi = static_cast<uint32_t>(db >> 32), lo = static_cast<uint32_t>(db);
      const uint32_t hmin = __reduce_min_sync(kFull, hi);
      const uint32_t lmin = __reduce_min_sync(kFull, hi == hmin ? lo : 0xFFFFFFFFu);
      const uint32_t jmin =
          __reduce_min_sync(kFull, (hi == hmin && lo == lmin) ? jidx : 0xFFFFFFFFu);
      const unsigned long long dmin = (static_cast<unsigned long long>(hmin) << 32) | lmin;
      if (dmin < best || (dmin == best && jmin < best_j)) {
        best = dmin;
        best_j = jmin;
      }
    }
    __syncwarp();
    if (lane == 0) {
      W.dbits[i] = best;
      W.idx[i] = best_j;
      W.smax[i] = smax;
    }
    __syncwarp();
  }
}

// One nearest-neighbour pass over this CTA's units; ends with a CTA barrier
// after which every result of the pass has been merged into a.out_key.
__device__ void l2_phase(const NNArgs& a, const PhaseQ q, L2Smem& s) {
  if (threadIdx.x == 0) l2_plan(a, q, s);
  __syncthreads();
  const int64_t u0 = s.u0, u1 = s.u1;
  if (u0 >= u1 || *reinterpret_cast<volatile int*>(&s.abort_flag)) {
    __syncthreads();
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t ph[kNS];
#pragma unroll
  for (int i = 0; i < kNS; ++i) ph[i] = s.bar_phase[i];
  Walk w{s.b0, s.m0, s.n0, (s.n0 * s.step[s.b0]) % s.nt[s.b0]};
  Walk ahead = w;  // the unit kNS ahead: the one a released buffer receives
  for (int k = 0; k < kNS; ++k) walk_next(ahead, s, a.batch);
  WarpState& W = s.ws[warp];
  const float max_p2 = a.db_absmax ? __int_as_float(__ldcg(a.db_absmax)) : INFINITY;
  Queries Q;
  Window Wn;
  bool seg_start = true, ok = true;
  int i = 0;
  for (int64_t u = u0; u < u1; ++u) {
    const int64_t k0 = w.m * kQT + warp * kQW;
    const int cnt = s.cnt[w.b];
    const bool active = k0 < cnt;  // warp-uniform
    if (seg_start) load_queries(a, q, w.b, k0, cnt, lane, max_p2, W, Q, Wn);
    float4 blo = make_float4(0.f, 0.f, 0.f, 0.f), bhi = blo;
    if (a.db_box && active) {
      const float4* bx = a.db_box + 2 * (w.b * ((a.ndb + kDC - 1) / kDC) + w.c);
      blo = __ldcg(bx);
      bhi = __ldcg(bx + 1);
    }
    ok = __all_sync(kFull, l2_wait(s, i, ph[i], a.status));
    ph[i] ^= 1u;
    // Skip the chunk when its box is farther from the queries' box than every
    // bound: each of its points is then beyond every query's answer. The
    // box distance loses at most a few ulps in fp32; the 2^-20 margins on
    // both sides cover that and the rounding of the bounds themselves.
    bool skip = false;
    if (a.db_box && active) {
      const float4 ql = W.qlo, qh = W.qhi;
      const float dx = fmaxf(fmaxf(blo.x - qh.x, ql.x - bhi.x), 0.f);
      const float dy = fmaxf(fmaxf(blo.y - qh.y, ql.y - bhi.y), 0.f);
      const float dz = fmaxf(fmaxf(blo.z - qh.z, ql.z - bhi.z), 0.f);
      const float d2 = __fmaf_rn(dz, dz, __fmaf_rn(dy, dy, dx * dx));
      skip = d2 * (1.f - 0x1p-20f) > ql.w * (1.f + 0x1p-20f);
    }
    if (ok && active && !skip) {
      const int rows = static_cast<int>(min(static_cast<int64_t>(kDC), s.rows[w.b] - w.c * kDC));
      l2_chunk(s.buf[i], rows, static_cast<uint32_t>(w.c * kDC), Q, Wn, W, lane);
    }
    Walk nx = w;
    walk_next(nx, s, a.batch);
    const bool seg_end = (nx.n == 0) || (u + 1 == u1);
    if (seg_end && active && ok && lane < kQW && k0 + lane < cnt) {
      const uint32_t jw = W.idx[lane];
      if (jw != 0xFFFFFFFFu) {
        // Across CTAs the merge compares the fp32 rounding of the distance
        // (lowest index among equal fp32 values).
        const float d2 = __double2float_rn(__longlong_as_double(static_cast<long long>(W.dbits[lane])));
        atomicMax(reinterpret_cast<unsigned long long*>(&a.out_key[w.b * a.q_cap + k0 + lane]),
                  static_cast<unsigned long long>(make_key(ord_f32(-d2), jw)));
      }
    }
    if (!ok) {
      *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
      break;
    }
    // Count this warp out of buffer i; the last one refills it.
    __syncwarp();
    if (lane == 0 && atomicAdd(&s.empty_cnt[i], 1) == kWarps - 1) {
      atomicExch(&s.empty_cnt[i], 0);
      if (u + kNS < u1 && !*reinterpret_cast<volatile int*>(&s.abort_flag))
        l2_issue(a, s, i, ahead);
    }
    __syncwarp();
    walk_next(ahead, s, a.batch);
    seg_start = seg_end;
    w = nx;
    i = i + 1 == kNS ? 0 : i + 1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < kNS; ++k) s.bar_phase[k] = ph[k];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) nn_l2_kernel(const __grid_constant__ NNArgs a) {
  L2Smem& s = l2_smem();
  l2_setup(s);
  l2_phase(a, PhaseQ{a.q_index, a.q_count, a.q_bound, 1}, s);
  l2_teardown(s, a.status);
}

// Fast reciprocal matching of pointmaps: the shared round loop with the
// passes above.
// Box (lo, hi) of the points of every database chunk of both maps, one
// chunk per warp (32 rows per lane), written into the passes' db_box arrays
// (workspace) before the first grid barrier; the passes read them through L2.
__device__ void l2_boxes(const RecArgs& r) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nc1 = (r.bwd.ndb + kDC - 1) / kDC, nc2 = (r.fwd.ndb + kDC - 1) / kDC;
  const int64_t total = r.batch * (nc1 + nc2);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < total;
       t += static_cast<int64_t>(gridDim.x) * kWarps) {
    const bool img1 = t < r.batch * nc1;
    const NNArgs& a = img1 ? r.bwd : r.fwd;  // the pass whose database this map is
    const int64_t nc = img1 ? nc1 : nc2, tt = img1 ? t : t - r.batch * nc1;
    const int b = static_cast<int>(tt / nc);
    const int64_t c = tt % nc;
    const int64_t n = a.ndb_dev ? min(static_cast<int64_t>(__ldg(a.ndb_dev + b)), a.ndb) : a.ndb;
    const float4* rows = reinterpret_cast<const float4*>(a.db_rows) + b * a.ndb;
    float v[6] = {INFINITY, INFINITY, INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 8
    for (int h = 0; h < kDC / 32; ++h) {
      const int64_t row = c * kDC + h * 32 + lane;
      if (row < n) {
        const float4 p = __ldg(rows + row);
        v[0] = fminf(v[0], p.x);
        v[1] = fminf(v[1], p.y);
        v[2] = fminf(v[2], p.z);
        v[3] = fmaxf(v[3], p.x);
        v[4] = fmaxf(v[4], p.y);
        v[5] = fmaxf(v[5], p.z);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int k = 0; k < 6; ++k) {
        const float y = __shfl_xor_sync(kFull, v[k], o);
        v[k] = k < 3 ? fminf(v[k], y) : fmaxf(v[k], y);
      }
    if (lane == 0) {
      float4* box = const_cast<float4*>(a.db_box) + 2 * (b * nc + c);
      box[0] = make_float4(v[0], v[1], v[2], 0.f);
      box[1] = make_float4(v[3], v[4], v[5], 0.f);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    reciprocal_l2_kernel(const __grid_constant__ RecArgs r) {
  L2Smem& s = l2_smem();
  l2_setup(s);
  auto pass = [&](int dir, const PhaseQ& q) { l2_phase(dir == 0 ? r.fwd : r.bwd, q, s); };
  auto boxes = [&] {
    if (r.fwd.db_box && r.bwd.db_box) l2_boxes(r);
  };
  fast_rounds<FASTNN_F32_L2>(r, pass, boxes, &s.abort_flag, &s.grid_ok, s.scan, s.cnt);
  l2_teardown(s, r.status);
}

}  // namespace

int nn_l2_max_batch() { return kMaxBatchL2; }

int launch_nn_l2(const NNArgs& a, cudaStream_t stream) {
  if (a.batch < 1 || a.batch > kMaxBatchL2 || a.ndb < 1) return FASTNN_ERR_INVALID;
  int sms = 0, rc = device_sm_count(&sms);
  if (rc != FASTNN_OK) return rc;
  FASTNN_CUDA_TRY(cudaFuncSetAttribute(nn_l2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes)));
  const int slot = kernel_timer_begin(stream, kTimeMatching);
  if (slot == -2) return FASTNN_ERR_CUDA;
  nn_l2_kernel<<<sms, kThreads, kSmemBytes, stream>>>(a);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return kernel_timer_end(slot, stream);
}

int launch_reciprocal_l2(const RecArgs& r, cudaStream_t stream) {
  if (r.batch < 1 || r.batch > kMaxBatchL2 || r.fwd.ndb < 1 || r.bwd.ndb < 1)
    return FASTNN_ERR_INVALID;
  int sms = 0, rc = device_sm_count(&sms);
  if (rc != FASTNN_OK) return rc;
  const void* fn = reinterpret_cast<const void*>(reciprocal_l2_kernel);
  FASTNN_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes)));
  int per_sm = 0;
  FASTNN_CUDA_TRY(
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, kSmemBytes));
  if (per_sm < 1) return FASTNN_ERR_UNSUPPORTED;
  RecArgs args = r;
  void* params[] = {&args};
  const int slot = kernel_timer_begin(stream, kTimeMatching);
  if (slot == -2) return FASTNN_ERR_CUDA;
  FASTNN_CUDA_TRY(
      cudaLaunchCooperativeKernel(fn, dim3(sms), dim3(kThreads), params, kSmemBytes, stream));
  return kernel_timer_end(slot, stream);
}

}  // namespace fastnn
