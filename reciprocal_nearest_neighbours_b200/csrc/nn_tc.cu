// Nearest neighbour by dot product on the 5th-generation tensor cores.
//
// For every active query slot k of every pair b:
//     out_key[b][k] = max over db rows j of key(<q_k, db_j>, j)
// i.e. the highest score with the lowest index among ties ("MASt3R
// dissection", section 3 Napkin Formula: argmax of dot products, the
// primitive of both the dense reciprocal set and the fast scheme).
//
// Design (one persistent CTA per SM, warp-specialised):
//   epilogue warps (two groups of 8): group g owns TMEM accumulator g, so
//       one group loads a score tile while the other folds the previous one
//       into a running (max score, lowest index) per query row. Warp w of a
//       group reads TMEM lanes 32 (w mod 4) .. +31 and one half (128
//       columns) of the tile. The score matrix never leaves the SM.
//   producer warp: gathers the 128 query rows of a tile into shared memory
//       (swizzled, K-major) and streams kBN-row database tiles with TMA
//       (cp.async.bulk.tensor, no multicast) into a 4- or 6-deep ring.
//   MMA warps (one thread each): tcgen05.mma kind::i8 (int8 -> int32,
//       K = 32) or kind::f16 (bf16 -> fp32, 2 x K = 16); issuer g fills
//       TMEM accumulator g (two of 256 columns) for every other unit;
//       tcgen05.commit frees the database stage and hands the accumulator to
//       its epilogue group.
// Work: units (pair, 128-query tile, kBN-row database tile) in row-major
// order, split into contiguous ranges of equal cost over the CTAs. A run of
// units that share a query tile is a segment; at its end the four warps that
// share a TMEM lane quarter merge their partial results in shared memory
// (int8), and each row's best is merged into the global key with one 64-bit
// atomicMax, which is order independent. A query may come with a score it is known to reach (the fast
// scheme's previous pass); its running best then starts just below that
// score, so that only tiles reaching it search for the column.
// Descriptors are zero-padded to 32 elements (32 B int8 rows, 64 B bf16 rows)
// by the repack kernel, so the padding adds nothing to any score.
// Every mbarrier wait is bounded; on expiry the kernel records
// FASTNN_ERR_TIMEOUT in the status word, drains what it issued and exits.
#include <cuda.h>

#include "common.cuh"
#include "frontier_dev.cuh"
#include "nn_tc.cuh"
#include "ptx.cuh"

namespace fastnn {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;                        // database rows per unit = accumulator columns
constexpr int kAcc = 2;                         // TMEM accumulators (2 x 256 = 512 columns)
constexpr int kMaxStages = 6;                   // database ring slots laid out in Ctl

// Database ring depth for RB-byte rows: 6 x 256-row tiles (48 KB / 96 KB) for
// 32- and 64-byte rows, 4 (128 KB) for 128-byte rows.
__host__ __device__ constexpr int stages_for(int rb) { return rb == 128 ? 4 : 6; }
constexpr int kGroupWarps = 8;                  // epilogue warps per accumulator
constexpr int kPreTiles = 1;                    // database tiles requested before a phase's first gather
constexpr int kEpiWarps = kAcc * kGroupWarps;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp0 = kEpiWarps + 1;        // MMA issuers: warp kMmaWarp0 + g feeds accumulator g
constexpr int kThreads = 32 * (kEpiWarps + 1 + kAcc);
constexpr int kEpiCols = kBN / 2;               // columns of a tile per epilogue thread
constexpr int kChunks = kEpiCols / 32;          // 32-column TMEM loads per unit and thread
constexpr int kMaxBatch = 1024;
// Work-split cost of starting a segment, in units (measured: a CTA whose
// range holds two segments ran ~5 us, about 10 units, longer than one with
// a single segment of the same length).
constexpr int64_t kSegCost = 8;
constexpr int kStashBytes = kEpiWarps * 32 * 32;  // 32 B per epilogue thread
// Segment-end partial results of the int8 epilogue (two parities); the
// 16-bit float paths search their columns exactly and need none.
constexpr int kPartBytes = 2 * kEpiWarps * 32 * 16;
__host__ __device__ constexpr int part_bytes(int dtype) { return dtype == FASTNN_I8 ? kPartBytes : 0; }

// Barrier slots inside the barrier block.
constexpr int kBarBFull = 0;
constexpr int kBarBEmpty = kBarBFull + kMaxStages;
constexpr int kBarAFull = kBarBEmpty + kMaxStages;
constexpr int kBarAEmpty = kBarAFull + 2;
constexpr int kBarAccFull = kBarAEmpty + 2;
constexpr int kBarAccEmpty = kBarAccFull + kAcc;
constexpr int kBarDone = kBarAccEmpty + kAcc;
constexpr int kNumBars = kBarDone + 1;
static_assert(stages_for(32) % kAcc == 0 && stages_for(128) % kAcc == 0 && (kAcc & (kAcc - 1)) == 0,
              "issuer g owns stages g, g + kAcc, ...");

struct Ctl {
  uint64_t bars[kNumBars];
  // Producer and MMA ring positions, kept here between phases so that only
  // the one or two threads that use them hold them in registers.
  int64_t p_seg;
  int p_st_idx;
  uint32_t p_st_phase;
  int64_t m_seg[kAcc];
  int m_st_idx[kAcc], m_par[kAcc];
  uint32_t m_st_phase[kAcc], m_ac_phase[kAcc];
  int p_last_phase[kMaxStages];
  uint32_t tmem_base;
  int abort_flag;
  int pack16;
  int grid_ok;
  uint64_t wait_ns;  // limit of the bounded waits in force (kTimeoutNs while draining)
  int scan[66];  // block-scan scratch of the per-pair compaction
  int b0;
  int64_t m0, n0, u0, u1;
  int mt[kMaxBatch];      // query tiles per pair (0 when the pair has no database row)
  int cnt[kMaxBatch];     // queries per pair
  int nt[kMaxBatch];      // database tiles per pair
  int rows[kMaxBatch];    // database rows per pair
};

__host__ __device__ constexpr size_t tile_bytes_a(int rb) { return static_cast<size_t>(kBM) * rb; }
__host__ __device__ constexpr size_t tile_bytes_b(int rb) { return static_cast<size_t>(kBN) * rb; }
__host__ __device__ constexpr size_t ctl_bytes() { return (sizeof(Ctl) + 15) & ~static_cast<size_t>(15); }

size_t smem_bytes(int rb, int dtype) {
  return 1024 /* alignment slack */ + 2 * tile_bytes_a(rb) + stages_for(rb) * tile_bytes_b(rb) +
         ctl_bytes() + kStashBytes + part_bytes(dtype);
}

// Bounded wait on an mbarrier phase. Returns false (and raises the abort flag
// and the device status) if the phase did not complete within kTimeoutNs, or
// if another role already aborted.
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, Ctl* ctl, int* status) {
  const uint64_t t0 = ptx::globaltimer_ns();
  const uint64_t limit = ctl->wait_ns;
  for (uint32_t n = 1;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 255) == 0 || n == 8) {
      if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) return false;
      if (ptx::globaltimer_ns() - t0 > limit) {
        *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, Ctl* ctl, int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, ctl, status);
}

// Bounded wait that polls with the non-blocking test first: used where the
// wait is on the critical path of the accumulator hand-off (the MMA issuer
// waiting for an epilogue group to free its accumulator), since a thread
// suspended in try_wait resumes later than a polling one notices the phase.
// After kSpinPolls polls it continues as wait_bounded. With TIGHT, the first
// 64 polls run in a loop of eight tests per counter step, so that the poll
// needs almost no ALU issue slots while the epilogue warps of the same SM
// sub-partitions keep the ALU pipe busy with the fold (measured on the int8
// paths: dense step 3.27 -> 3.19 ms, 16-pair batch 3.91 -> 3.82 ms; on the
// 16-bit float path it cost 2.5%, so that path keeps the plain loop).
constexpr int kSpinPolls = 2048;
template <bool TIGHT>
__device__ __forceinline__ bool spin_wait_bounded(uint32_t bar, uint32_t parity, Ctl* ctl,
                                                  int* status) {
  if constexpr (TIGHT) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .u32 c;\n\t"
        "mov.u32 c, %3;\n\t"
        "SPIN_%=:\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t@p bra DONE_%=;\n\t"
        "sub.u32 c, c, 1;\n\tsetp.ne.u32 q, c, 0;\n\t@q bra SPIN_%=;\n\t"
        "DONE_%=:\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(8u)
        : "memory");
    if (ok) return true;
  }
  for (int n = 0; n < kSpinPolls; ++n)
    if (ptx::mbar_test_wait(bar, parity)) return true;
  return wait_slow(bar, parity, ctl, status);
}

// Index and phase bit of a ring of mbarrier-guarded slots.
struct Ring {
  int idx = 0;
  uint32_t phase = 0;
  template <int N>
  __device__ __forceinline__ void next() {
    if (++idx == N) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

// Warp-uniform bounded wait: every lane polls, the warp proceeds only if all
// lanes saw the phase complete.
__device__ bool warp_wait_bounded(uint32_t bar, uint32_t parity, Ctl* ctl, int* status) {
  const bool ok = wait_bounded(bar, parity, ctl, status);
  return __all_sync(0xffffffffu, ok);
}

// Position of the next unit: pair b, query tile m, database tile n.
struct Pos {
  int b;
  int64_t m, n;
};

// Units left in the current segment (same pair and query tile).
__device__ __forceinline__ int64_t seg_len(const Pos& p, int64_t u, int64_t u1, const Ctl* ctl) {
  return min(u1 - u, static_cast<int64_t>(ctl->nt[p.b]) - p.n);
}

// Move to the first unit of the next segment.
__device__ __forceinline__ void next_segment(Pos& p, const Ctl* ctl, int batch) {
  p.n = 0;
  if (++p.m == ctl->mt[p.b]) {
    p.m = 0;
    do {
      ++p.b;
    } while (p.b < batch && ctl->mt[p.b] == 0);
  }
}

// Query-tile gather: 32 lanes copy 128 rows of `rb` bytes into a K-major tile
// with the 32B / 64B / 128B swizzle (rb = 32 / 64 / 128) the MMA descriptor
// names: the 16-byte chunk c of row r lands at r * rb + 16 * (c ^ swz(r)).
// All row indices are loaded first, then the rows in batches of kRB: the
// loads of a batch are in flight together instead of one dependent index
// and row load per row.
template <int RB>
__device__ __forceinline__ void gather_a(uint8_t* tile, const NNArgs& a, const PhaseQ& q, int b,
                                         int64_t m, int cnt, int lane) {
  constexpr int kC = RB / 16;
  constexpr int kR = kBM / 32;             // rows per lane
  constexpr int kRB = RB == 32 ? kR : 2;   // rows per batch of loads
  int64_t row[kR];
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int64_t k = m * kBM + lane + 32 * i;
    row[i] = k < cnt ? nn_query_row(a, q, b, k) : -1;
  }
#pragma unroll
  for (int i0 = 0; i0 < kR; i0 += kRB) {
    uint4 v[kRB][kC];
#pragma unroll
    for (int i = 0; i < kRB; ++i) {
      // Rows outside the query source (never produced by a healthy
      // pipeline) read as zeros instead of faulting.
      const int64_t rw = row[i0 + i];
      if (rw >= 0 && rw < a.q_rows_per_pair) {
        const uint4* src = reinterpret_cast<const uint4*>(
            a.q_rows + (static_cast<int64_t>(b) * a.q_rows_per_pair + rw) * RB);
#pragma unroll
        for (int c = 0; c < kC; ++c) v[i][c] = __ldg(src + c);
      } else {
#pragma unroll
        for (int c = 0; c < kC; ++c) v[i][c] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < kRB; ++i) {
      const int r = lane + 32 * (i0 + i);
      const int swz = RB == 32 ? ((r >> 2) & 1) : RB == 64 ? ((r >> 1) & 3) : (r & 7);
#pragma unroll
      for (int c = 0; c < kC; ++c)
        *reinterpret_cast<uint4*>(tile + r * RB + 16 * (c ^ swz)) = v[i][c];
    }
  }
}

template <int DT>
struct Epi;

// int8 descriptors: int32 scores.
template <>
struct Epi<FASTNN_I8> {
  using S = int32_t;
  static __device__ __forceinline__ S lowest() { return INT32_MIN; }
  static __device__ __forceinline__ S as_score(uint32_t r) { return static_cast<int32_t>(r); }
  static __device__ __forceinline__ S mx(S x, S y) { return max(x, y); }
  static __device__ __forceinline__ S mx3(S x, S y, S z) { return max(max(x, y), z); }
  static __device__ __forceinline__ uint32_t ord(S s) { return ord_i32(s); }
  // Running best that a score equal to the bound beats (scores are exact).
  static __device__ __forceinline__ S below_bound(uint32_t bits) { return unord_i32(bits) - 1; }
};

// bf16 and half descriptors: fp32 scores.
template <>
struct Epi<FASTNN_BF16> {
  using S = float;
  static __device__ __forceinline__ S lowest() { return -INFINITY; }
  static __device__ __forceinline__ S as_score(uint32_t r) { return __uint_as_float(r); }
  static __device__ __forceinline__ S mx(S x, S y) { return fmaxf(x, y); }
  static __device__ __forceinline__ S mx3(S x, S y, S z) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
    return r;
  }
  static __device__ __forceinline__ uint32_t ord(S s) { return ord_f32(s); }
  // Running best that the bound's own dot product beats: the bound was
  // accumulated with the operands' roles swapped, so it is lowered by a margin
  // far above any difference in rounding between the two sums.
  static __device__ __forceinline__ S below_bound(uint32_t bits) {
    const float s = unord_f32(bits);
    return s - (fabsf(s) + 1.0f) * 0x1p-12f;
  }
};

template <>
struct Epi<FASTNN_F16> : Epi<FASTNN_BF16> {};

// Fold 32 consecutive columns (global index col0 + j) into (best, bidx).
// Used for the ragged last database tile: `valid` < 32 masks the tail.
template <int DT>
__device__ __forceinline__ void fold32_masked(const uint32_t (&r)[32], uint32_t col0, int valid,
                                              typename Epi<DT>::S& best, uint32_t& bidx,
                                              bool& exact) {
  using E = Epi<DT>;
  using S = typename E::S;
  S v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = (j < valid) ? E::as_score(r[j]) : E::lowest();
  S m = v[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) m = E::mx(m, v[j]);
  if (m > best) {
    int first = 31;
#pragma unroll
    for (int j = 31; j >= 0; --j)
      if (v[j] == m) first = j;
    best = m;
    bidx = col0 + first;
    exact = true;
  }
}

// ---- fast epilogue for full tiles ------------------------------------------
// Each thread owns one query row and kEpiCols columns of the tile. Their
// maximum is formed with a reduction tree; only when it beats the running best
// strictly (a new record for this row) is the first column holding it
// searched for: the 8-register group holding it is found from the tree's
// group maxima, staged to this thread's 32-byte slot in shared memory, and
// scanned there, so the search needs no dynamic register indexing. The lowest
// index among equal scores survives.

__device__ __forceinline__ uint32_t vmax3_s16x2(uint32_t a, uint32_t b, uint32_t c) {
  return ptx::vmax_s16x2(ptx::vmax_s16x2(a, b), c);
}

__device__ __forceinline__ uint32_t tree8_s16x2(const uint32_t* r) {
  const uint32_t x = vmax3_s16x2(r[0], r[1], r[2]);
  const uint32_t y = vmax3_s16x2(r[3], r[4], r[5]);
  const uint32_t z = ptx::vmax_s16x2(r[6], r[7]);
  return vmax3_s16x2(x, y, z);
}

__device__ __forceinline__ int lo16(uint32_t x) { return static_cast<int>(static_cast<int16_t>(x & 0xFFFFu)); }
__device__ __forceinline__ int hi16(uint32_t x) { return static_cast<int>(x) >> 16; }

__device__ __forceinline__ void stash8(uint4* slot, const uint32_t* r) {
  slot[0] = make_uint4(r[0], r[1], r[2], r[3]);
  slot[1] = make_uint4(r[4], r[5], r[6], r[7]);
}

// int8 scores that fit in 16 bits: r[c][i] holds columns 32c + 2i (low half)
// and 32c + 2i + 1 (high half) of this thread's block. On a strict new
// record the first 16-column group holding it is found from the tree's group
// maxima. DEFER == false: that group is staged to this thread's 32-byte slot
// in shared memory and scanned for the first column. DEFER == true: only the
// group is noted (bidx = its first column, exact = false) and resolve_group
// finds the column once, at the end of the segment (measured: the dense
// 512x384 mutual set 3.85 -> 3.40 ms, the 16-pair batch 4.23 -> 3.93 ms).
template <int NC, bool DEFER>
__device__ __forceinline__ void fold_pack16(const uint32_t (&r)[NC][16], uint32_t colbase,
                                            int& best, uint32_t& bidx, bool& exact,
                                            uint4* slot) {
  constexpr int G = 2 * NC;  // groups of 8 registers = 16 columns
  uint32_t g[G];
#pragma unroll
  for (int i = 0; i < G; ++i) g[i] = tree8_s16x2(&r[i / 2][(i % 2) * 8]);
  uint32_t u;
  if constexpr (G == 2) {
    u = ptx::vmax_s16x2(g[0], g[1]);
  } else if constexpr (G == 4) {
    u = ptx::vmax_s16x2(ptx::vmax_s16x2(g[0], g[1]), ptx::vmax_s16x2(g[2], g[3]));
  } else {
    u = vmax3_s16x2(vmax3_s16x2(g[0], g[1], g[2]), vmax3_s16x2(g[3], g[4], g[5]),
                    ptx::vmax_s16x2(g[6], g[7]));
  }
  const int m = max(lo16(u), hi16(u));
  if (m > best) {
    best = m;
    int gi = G - 1;
#pragma unroll
    for (int i = G - 1; i >= 0; --i)
      if (lo16(g[i]) == m || hi16(g[i]) == m) gi = i;
    if constexpr (DEFER) {
      bidx = colbase + 16 * gi;
      exact = false;
    } else {
#pragma unroll
      for (int i = 0; i < G; ++i)
        if (i == gi) stash8(slot, &r[i / 2][(i % 2) * 8]);
      const uint4 a = slot[0], b = slot[1];
      const uint32_t x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      int w = 15;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (hi16(x[j]) == m) w = 2 * j + 1;
        if (lo16(x[j]) == m) w = 2 * j;
      }
      bidx = colbase + 16 * gi + w;
      exact = true;
    }
  }
}

// The lowest column among the 16 from bidx whose int8 dot product with the
// query equals best (one exists: the tile's tree found best in this group).
// The query is row r of the segment's query tile in shared memory (RB bytes of
// zero-padded int8, 16-byte chunks swizzled as the gather wrote them); the
// candidate rows are read from the repacked database (L2) in batches of
// four, a lane stopping at the batch that holds its column.
template <int RB>
__device__ __noinline__ uint32_t resolve_group(const uint8_t* qtile, int r,
                                               const uint8_t* __restrict__ db, uint32_t bidx,
                                               int best) {
  constexpr int NV = RB / 16;           // 16-byte words per row
  constexpr int kRows = 4;              // candidate rows per batch of loads
  const int swz = RB == 32 ? ((r >> 2) & 1) : ((r >> 1) & 3);
  int4 qv[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i)
    qv[i] = *reinterpret_cast<const int4*>(qtile + r * RB + 16 * (i ^ swz));
  uint32_t found = 0xFFFFFFFFu;
#pragma unroll 1
  for (int c0 = 0; c0 < 16 && found == 0xFFFFFFFFu; c0 += kRows) {
    int4 rv[kRows][NV];
#pragma unroll
    for (int c = 0; c < kRows; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i)
        rv[c][i] = __ldg(reinterpret_cast<const int4*>(db + static_cast<int64_t>(bidx + c0 + c) * RB) + i);
#pragma unroll
    for (int c = kRows - 1; c >= 0; --c) {
      int s = 0;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        s = __dp4a(qv[i].x, rv[c][i].x, s);
        s = __dp4a(qv[i].y, rv[c][i].y, s);
        s = __dp4a(qv[i].z, rv[c][i].z, s);
        s = __dp4a(qv[i].w, rv[c][i].w, s);
      }
      if (s == best) found = bidx + c0 + c;
    }
  }
  return found != 0xFFFFFFFFu ? found : bidx;
}

// 32-bit scores (int32, or fp32 for bf16 descriptors): r[c][i] = column 32c + i.
template <int DT, int NC>
__device__ __forceinline__ void fold_wide(const uint32_t (&r)[NC][32], uint32_t colbase,
                                          typename Epi<DT>::S& best, uint32_t& bidx,
                                          bool& exact, uint4* slot) {
  using E = Epi<DT>;
  using S = typename E::S;
  constexpr int G = 4 * NC;  // groups of 8 registers = 8 columns
  S g[G];
#pragma unroll
  for (int i = 0; i < G; ++i) {
    const uint32_t* q = &r[i / 4][(i % 4) * 8];
    const S a0 = E::mx3(E::as_score(q[0]), E::as_score(q[1]), E::as_score(q[2]));
    const S a1 = E::mx3(E::as_score(q[3]), E::as_score(q[4]), E::as_score(q[5]));
    g[i] = E::mx3(a0, a1, E::mx(E::as_score(q[6]), E::as_score(q[7])));
  }
  S m = g[0];
#pragma unroll
  for (int i = 1; i < G; ++i) m = E::mx(m, g[i]);
  if (m > best) {
    best = m;
    int gi = G - 1;
#pragma unroll
    for (int i = G - 1; i >= 0; --i)
      if (g[i] == m) gi = i;
#pragma unroll
    for (int i = 0; i < G; ++i)
      if (i == gi) stash8(slot, &r[i / 4][(i % 4) * 8]);
    const uint4 a = slot[0], b = slot[1];
    const uint32_t x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    int w = 7;
#pragma unroll
    for (int j = 7; j >= 0; --j)
      if (E::as_score(x[j]) == m) w = j;
    bidx = colbase + 8 * gi + w;
    exact = true;
  }
}

// ---- pipeline set-up, phases and teardown --------------------------------
// A "phase" is one nearest-neighbour pass over a work list. The standalone
// kernel runs one phase; the persistent fast-matching kernel runs two per
// round. Barrier phases, ring positions and the TMEM allocation carry over
// from phase to phase, so a phase costs no set-up.

struct SmemLayout {
  uint8_t* tileA;  // 2 x kBM x RB query tiles
  uint8_t* tileB;  // stages_for(RB) x kBN x RB database tiles
  Ctl* ctl;
  uint4* stash;    // 32 B per epilogue thread
  uint4* part;     // 2 x kEpiWarps x 32 segment-end partial results
};

template <int RB>
__device__ __forceinline__ SmemLayout smem_layout() {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SmemLayout L;
  L.tileA = base;
  L.tileB = base + 2 * tile_bytes_a(RB);
  L.ctl = reinterpret_cast<Ctl*>(L.tileB + stages_for(RB) * tile_bytes_b(RB));
  L.stash = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(L.ctl) + ctl_bytes());
  L.part = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(L.stash) + kStashBytes);  // int8 only
  return L;
}

// Epilogue state that persists across phases (per thread). The producer's and
// the MMA thread's ring positions live in Ctl.
struct PipeState {
  uint32_t ephase = 0;  // phase bit of this group's accumulator barrier
  int epar = 0;         // parity of the running unit index
  int eseg = 0;         // parity of the running segment index (the query tile)
};

// Barrier init and TMEM allocation; ends with a CTA barrier.
template <int DT>
__device__ __forceinline__ void pipe_setup(Ctl* ctl) {
  if (threadIdx.x == 0) {
    ctl->abort_flag = 0;
    ctl->pack16 = -1;
    ctl->wait_ns = kTimeoutNs;
    ctl->p_seg = 0;
    ctl->p_st_idx = 0;
    ctl->p_st_phase = 0;
    for (int g = 0; g < kAcc; ++g) {
      ctl->m_seg[g] = 0;
      ctl->m_st_idx[g] = g;  // issuer g handles units g, g + kAcc, ... -> stages g, g + kAcc, ...
      ctl->m_st_phase[g] = 0;
      ctl->m_ac_phase[g] = 0;
      ctl->m_par[g] = 0;
    }
    for (int s = 0; s < kMaxStages; ++s) ctl->p_last_phase[s] = -1;
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= kBarAFull && i < kBarAFull + 2) count = 32;    // producer lanes
      // One commit per MMA issuer; with int8 scores also one arrival per
      // lane quarter's leader, whose column searches read the query tile.
      if (i >= kBarAEmpty && i < kBarAEmpty + 2) count = kAcc + (DT == FASTNN_I8 ? 4 : 0);
      if (i == kBarDone) count = kAcc;
      if (i >= kBarAccEmpty && i < kBarAccEmpty + kAcc) count = kGroupWarps;
      ptx::mbar_init(ptx::smem_u32(&ctl->bars[i]), count);
    }
    ptx::fence_mbar_init();
  }
  if ((threadIdx.x >> 5) == 0) {
    ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
}

// Work list of this CTA for one phase (thread 0).
template <int DT>
__device__ void plan_phase(const NNArgs& a, const PhaseQ& q, Ctl* ctl) {
  const int batch = a.batch;
  // int8 scores fit in 16 bits when d * max|q| * max|db| < 2^15; the repack
  // pass measured both maxima before the launch, and the test is symmetric in
  // the two maps, so it is decided once per launch (pack16 < 0: not yet).
  if (ctl->pack16 < 0) {
    const bool have_absmax = DT == FASTNN_I8 && a.q_absmax && a.db_absmax;
    const int q_absmax = have_absmax ? __ldcg(a.q_absmax) : 0;
    const int db_absmax = have_absmax ? __ldcg(a.db_absmax) : 0;
    ctl->pack16 =
        (have_absmax && static_cast<int64_t>(q_absmax) * db_absmax * a.d <= 32767) ? 1 : 0;
  }
  ctl->wait_ns = wait_limit(a.wait_ns);
  for (int b = 0; b < batch; ++b) {
    const int64_t c = q.cached ? ctl->cnt[b] : nn_count(a, q, b);
    const int64_t rows = a.ndb_dev ? min(static_cast<int64_t>(__ldcg(a.ndb_dev + b)), a.ndb)
                                   : a.ndb;
    const int64_t nt = rows > 0 ? (rows + kBN - 1) / kBN : 0;
    ctl->cnt[b] = static_cast<int>(c);
    ctl->rows[b] = static_cast<int>(rows);
    ctl->nt[b] = static_cast<int>(nt);
    ctl->mt[b] = nt > 0 ? static_cast<int>((c + kBM - 1) / kBM) : 0;
  }
  // Contiguous ranges of equal cost, where a segment (one query tile of one
  // pair: nt units on the same query tile) costs its units plus kSegCost for
  // starting it (query gather, pipeline refill, result flush), so that a CTA
  // whose range starts a new segment takes that many fewer units.
  const int64_t G = gridDim.x;
  // Quotients of non-negative values; 32-bit division when both fit (the
  // 64-bit one is a long dependent sequence on this single thread).
  auto div = [](int64_t x, int64_t y) -> int64_t {
    return (x <= 0x7fffffff && y <= 0x7fffffff)
               ? static_cast<int64_t>(static_cast<uint32_t>(x) / static_cast<uint32_t>(y))
               : x / y;
  };
  int64_t cost = 0;
  for (int b = 0; b < batch; ++b) cost += static_cast<int64_t>(ctl->mt[b]) * (ctl->nt[b] + kSegCost);
  // Unit index at cost position C (monotone in C; 0 at 0, total at cost).
  auto unit_at = [&](int64_t C, int& b_out, int64_t& m_out, int64_t& n_out) {
    int64_t units = 0, acc = 0;
    int b = 0;
    while (b < batch) {
      const int64_t segc = ctl->nt[b] + kSegCost;
      const int64_t pc = static_cast<int64_t>(ctl->mt[b]) * segc;
      if (acc + pc > C) break;
      acc += pc;
      units += static_cast<int64_t>(ctl->mt[b]) * ctl->nt[b];
      ++b;
    }
    b_out = b;
    m_out = n_out = 0;
    if (b >= batch) return units;
    const int64_t segc = ctl->nt[b] + kSegCost;
    const int64_t j = div(C - acc, segc);
    const int64_t off = max(static_cast<int64_t>(0), (C - acc) - j * segc - kSegCost);
    m_out = j;
    n_out = off;
    return units + j * ctl->nt[b] + off;
  };
  int b, b_end;
  int64_t m0, n0, m_end, n_end;
  ctl->u0 = unit_at(div(cost * blockIdx.x, G), b, m0, n0);
  ctl->u1 = unit_at(div(cost * (blockIdx.x + 1), G), b_end, m_end, n_end);
  ctl->b0 = b;
  ctl->m0 = m0;
  ctl->n0 = n0;
}

// One nearest-neighbour phase: plan (thread 0), then each role runs its loop
// over this CTA's units. Ends with a CTA barrier, after which every MMA of the
// phase has completed and every result has been merged into a.out_key.
template <int DT, int RB, bool DEFER>
__device__ void run_phase(const CUtensorMap* tmap_db, const NNArgs& a, const PhaseQ q,
                          const SmemLayout& L, uint32_t tmem, PipeState& ps) {
  constexpr int NS = stages_for(RB);  // database ring depth
  constexpr int KS = RB / 32;         // MMAs per tile: 32 bytes of K each
  using E = Epi<DT>;
  Ctl* ctl = L.ctl;
  uint8_t* tileA = L.tileA;
  uint8_t* tileB = L.tileB;
  if (threadIdx.x == 0) plan_phase<DT>(a, q, ctl);
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int batch = a.batch;
  const int64_t u0 = ctl->u0, u1 = ctl->u1;
  auto bar = [&](int i) { return ptx::smem_u32(&ctl->bars[i]); };
  const Pos start{ctl->b0, ctl->m0, ctl->n0};

  if (u0 < u1 && !ctl->abort_flag) {
    if (warp == kProducerWarp) {
      // -------------------------------------------------------------- producer
      Pos p = start;
      bool ok = true;
      int64_t seg = ctl->p_seg;
      Ring st;
      st.idx = ctl->p_st_idx;
      st.phase = ctl->p_st_phase;
      // At the phase start every stage is free: the first kPreTiles database
      // tiles are requested before the query gather, so that their latency
      // overlaps the gather's dependent loads. (All free stages at once was
      // measured slower: every CTA's burst of tile loads delays the gathers.)
      auto load_b = [&](int32_t row) {
        if (!wait_bounded(bar(kBarBEmpty + st.idx), st.phase ^ 1u, ctl, a.status)) return false;
        ptx::mbar_arrive_expect_tx(bar(kBarBFull + st.idx), static_cast<uint32_t>(tile_bytes_b(RB)));
        ptx::tma_load_2d(ptx::smem_u32(tileB + st.idx * tile_bytes_b(RB)), tmap_db, 0, row,
                         bar(kBarBFull + st.idx));
        ctl->p_last_phase[st.idx] = static_cast<int>(st.phase);
        st.next<NS>();
        return true;
      };
      for (int64_t u = u0; ok && u < u1; ++seg) {
        const int len = static_cast<int>(seg_len(p, u, u1, ctl));
        const int as = static_cast<int>(seg & 1);
        const int32_t row0 = static_cast<int32_t>(static_cast<int64_t>(p.b) * a.ndb + p.n * kBN);
        const int pre = u == u0 ? min(len, kPreTiles) : 0;
        if (lane == 0)
          for (int j = 0; ok && j < pre; ++j) ok = load_b(row0 + j * kBN);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (!warp_wait_bounded(bar(kBarAEmpty + as), static_cast<uint32_t>(((seg >> 1) & 1) ^ 1),
                               ctl, a.status))
          break;
        gather_a<RB>(tileA + as * tile_bytes_a(RB), a, q, p.b, p.m, ctl->cnt[p.b], lane);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar(kBarAFull + as));
        if (lane == 0) {
          int32_t row = row0 + pre * kBN;
          for (int j = pre; j < len; ++j, row += kBN) {
            if (!load_b(row)) {
              ok = false;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        u += len;
        next_segment(p, ctl, batch);
      }
      if (lane == 0) {
        ctl->p_seg = seg;
        ctl->p_st_idx = st.idx;
        ctl->p_st_phase = st.phase;
      }
    } else if (warp >= kMmaWarp0) {
      // ------------------------------------------------------------- MMA issue
      // Issuer g (one thread) handles the units whose running index is
      // congruent to g mod kAcc: accumulator g, stages g, g + kAcc, ... The
      // issuers sit in different warps, so their per-unit waits and commits
      // overlap.
      if (lane == 0) {
        // Instruction descriptor: accumulator format (S32 / F32), A and B formats
        // (S8 / BF16 / F16), both K-major, N >> 3, M >> 4.
        constexpr uint32_t kFmt = DT == FASTNN_I8 ? 1u : DT == FASTNN_BF16 ? 1u : 0u;
        constexpr uint32_t kIdesc = ((DT == FASTNN_I8 ? 2u : 1u) << 4) | (kFmt << 7) |
                                    (kFmt << 10) | ((kBN >> 3) << 17) | ((kBM >> 4) << 24);
        const int g = warp - kMmaWarp0;
        Pos p = start;
        bool ok = true;
        int64_t seg = ctl->m_seg[g];
        int st_idx = ctl->m_st_idx[g];
        uint32_t st_phase = ctl->m_st_phase[g];
        uint32_t ac_phase = ctl->m_ac_phase[g];
        int par = ctl->m_par[g];
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(g * kBN);
        for (int64_t u = u0; ok && u < u1; ++seg) {
          const int len = static_cast<int>(seg_len(p, u, u1, ctl));
          const int as = static_cast<int>(seg & 1);
          if (!wait_bounded(bar(kBarAFull + as), static_cast<uint32_t>((seg >> 1) & 1), ctl,
                            a.status))
            break;
          ptx::tc_fence_after();
          const uint64_t adesc =
              ptx::smem_desc_kmajor(ptx::smem_u32(tileA + as * tile_bytes_a(RB)), RB);
          const uint64_t bdesc0 = ptx::smem_desc_kmajor(ptx::smem_u32(tileB), RB);
          for (int j = (g - par) & (kAcc - 1); j < len; j += kAcc) {
            // The database stage is loaded long before the accumulator frees
            // up: check it first, so that only the MMA issue follows the
            // accumulator's hand-back.
            const uint64_t bdesc =
                bdesc0 + static_cast<uint64_t>((st_idx * tile_bytes_b(RB)) >> 4);
            if (!wait_bounded(bar(kBarBFull + st_idx), st_phase, ctl, a.status) ||
                !spin_wait_bounded<DT == FASTNN_I8>(bar(kBarAccEmpty + g), ac_phase ^ 1u, ctl,
                                                    a.status)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            // K steps of 32 bytes (32 int8 or 16 16-bit elements); step s
            // starts 32 * s bytes into the swizzled rows.
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              if constexpr (DT == FASTNN_I8)
                ptx::mma_i8(d_tmem, adesc + 2 * ks, bdesc + 2 * ks, kIdesc, ks > 0 ? 1u : 0u);
              else
                ptx::mma_bf16(d_tmem, adesc + 2 * ks, bdesc + 2 * ks, kIdesc, ks > 0 ? 1u : 0u);
            }
            ptx::mma_commit(bar(kBarAccFull + g));
            ptx::mma_commit(bar(kBarBEmpty + st_idx));
            ac_phase ^= 1u;
            st_idx += kAcc;
            if (st_idx >= NS) {
              st_idx -= NS;
              st_phase ^= 1u;
            }
          }
          if (!ok) break;
          // The query tile may be refilled once both issuers' MMAs on it completed.
          ptx::mma_commit(bar(kBarAEmpty + as));
          u += len;
          par ^= len & 1;
          next_segment(p, ctl, batch);
        }
        ctl->m_seg[g] = seg;
        ctl->m_st_idx[g] = st_idx;
        ctl->m_st_phase[g] = st_phase;
        ctl->m_ac_phase[g] = ac_phase;
        ctl->m_par[g] = par;
      }
    } else {
      // -------------------------------------------------------------- epilogue
      // Group g folds the units whose running index is congruent to g mod 2,
      // i.e. the ones the MMA wrote into accumulator g.
      const int grp = warp / kGroupWarps;
      const int gw = warp % kGroupWarps;
      const int lg = gw & 3;  // TMEM lane quarter (warp id mod 4)
      const int h = gw >> 2;  // column half of the tile
      const bool pack16 = ctl->pack16 != 0;
      const uint32_t acc_bar = bar(kBarAccFull + grp);
      const uint32_t rel_bar = bar(kBarAccEmpty + grp);
      const uint32_t taddr = tmem + (static_cast<uint32_t>(lg * 32) << 16) +
                             static_cast<uint32_t>(grp * kBN + h * kEpiCols);
      uint4* slot = L.stash + 2 * threadIdx.x;
      Pos p = start;
      bool ok = true;
      for (int64_t u = u0; ok && u < u1;) {
        const int len = static_cast<int>(seg_len(p, u, u1, ctl));
        const int n0 = static_cast<int>(p.n);
        const int last_n = ctl->nt[p.b] - 1;
        const int tail = ctl->rows[p.b] - last_n * kBN;  // valid columns of the last tile
        // A row with a score bound starts just below it: only tiles that
        // reach the bound can hold the row's maximum, and only they search
        // for its column. A row whose tiles all stay below keeps no result
        // here; another CTA's range holds the bound's own column.
        const int64_t krow = p.m * kBM + lg * 32 + lane;
        typename E::S best = E::lowest();
        if (q.bound && krow < ctl->cnt[p.b]) {
          const uint32_t bits = __ldcg(q.bound + (p.b * a.q_cap + krow) * q.bstride);
          if (bits != 0u) best = E::below_bound(bits);
        }
        uint32_t bidx = 0xFFFFFFFFu;
        bool exact = true;  // false: bidx is a 16-column group still to resolve
        for (int j = (grp - ps.epar) & 1; j < len; j += kAcc) {
          const int n = n0 + j;
          const uint32_t colbase = static_cast<uint32_t>(n) * kBN + h * kEpiCols;
          const bool ragged = n == last_n && tail < kBN;
          if (!warp_wait_bounded(acc_bar, ps.ephase, ctl, a.status)) {
            ok = false;
            break;
          }
          ps.ephase ^= 1u;
          ptx::tc_fence_after();
          if (ragged) {
            // Ragged last tile of the database: column-masked fold.
            const int valid_blk = tail - h * kEpiCols;
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
              uint32_t r[32];
              ptx::tmem_ld32(taddr + c * 32, r);
              ptx::tmem_ld_wait();
              const int valid = min(32, max(0, valid_blk - c * 32));
              fold32_masked<DT>(r, colbase + c * 32, valid, best, bidx, exact);
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(rel_bar);
          } else if (DT == FASTNN_I8 && pack16) {
            uint32_t r[kChunks][16];
            static_assert(kChunks * 16 == 64, "one packed 128-column load");
            ptx::tmem_ld64_pack(taddr, reinterpret_cast<uint32_t(&)[64]>(r));
            ptx::tmem_ld_wait_regs(reinterpret_cast<uint32_t(&)[64]>(r));
            // The accumulator is free for the next MMA once it is in registers:
            // release it before any of the fold (the pin keeps the fold's
            // register-only work from being scheduled ahead of the arrive).
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(rel_bar);
            ptx::pin_regs(reinterpret_cast<uint32_t(&)[64]>(r));
            if constexpr (DT == FASTNN_I8)
              fold_pack16<kChunks, DEFER>(r, colbase, best, bidx, exact, slot);
          } else {
            // 32-bit scores: two 64-column halves, the accumulator is released
            // after the second load.
            uint32_t r[2][32];
            ptx::tmem_ld64(taddr, reinterpret_cast<uint32_t(&)[64]>(r));
            ptx::tmem_ld_wait_regs(reinterpret_cast<uint32_t(&)[64]>(r));
            fold_wide<DT, 2>(r, colbase, best, bidx, exact, slot);
            ptx::tmem_ld64(taddr + 64, reinterpret_cast<uint32_t(&)[64]>(r));
            ptx::tmem_ld_wait_regs(reinterpret_cast<uint32_t(&)[64]>(r));
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(rel_bar);
            ptx::pin_regs(reinterpret_cast<uint32_t(&)[64]>(r));
            fold_wide<DT, 2>(r, colbase + 64, best, bidx, exact, slot);
          }
        }
        const int par = ps.eseg;
        if constexpr (DT == FASTNN_I8) {
          // The four warps of this lane quarter (two accumulator groups x
          // two column halves) hold partial results for the same 32 rows over
          // disjoint columns. They meet in shared memory (double-buffered by
          // segment parity); the leader, warp (0, 0), keeps each row's best
          // (higher score, then lower index: the column groups are disjoint,
          // so a group start orders like any column in it), finds its column
          // if it is still a 16-column group, and merges it into the global
          // key: one column search and one atomic per row instead of four.
          // Every warp of the quarter reaches the named barrier (all waits
          // above are bounded), and all leave the loop together when any of
          // them failed.
          const bool valid = ok && krow < ctl->cnt[p.b] && bidx != 0xFFFFFFFFu;
          uint4* part = L.part + par * (kEpiWarps * 32);
          part[warp * 32 + lane] = make_uint4(E::ord(best), bidx, exact ? 1u : 0u,
                                              (valid ? 1u : 0u) | (ok ? 2u : 0u));
          ptx::named_bar_sync(1 + lg, 4 * 32);
          const int w4[4] = {lg, kGroupWarps + lg, 4 + lg, kGroupWarps + 4 + lg};
          bool all_ok = true;
#pragma unroll
          for (int i = 0; i < 4; ++i) all_ok = all_ok && (part[w4[i] * 32 + lane].w & 2u) != 0u;
          if (!__all_sync(0xffffffffu, all_ok)) break;
          if (grp == 0 && h == 0) {
            uint4 bst = part[lg * 32 + lane];
#pragma unroll
            for (int i = 1; i < 4; ++i) {
              const uint4 v = part[w4[i] * 32 + lane];
              if ((v.w & 1u) && (!(bst.w & 1u) || v.x > bst.x || (v.x == bst.x && v.y < bst.y)))
                bst = v;
            }
            if (bst.w & 1u) {
              const uint32_t col =
                  bst.z != 0u ? bst.y
                              : resolve_group<RB>(tileA + par * tile_bytes_a(RB), lg * 32 + lane,
                                                  a.db_rows + static_cast<int64_t>(p.b) * a.ndb * RB,
                                                  bst.y, unord_i32(bst.x));
              atomicMax(reinterpret_cast<unsigned long long*>(&a.out_key[p.b * a.q_cap + krow]),
                        static_cast<unsigned long long>(make_key(bst.x, col)));
            }
            // The query tile may be refilled once the column searches have
            // read their rows (one arrival per lane quarter).
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(kBarAEmpty + par));
          }
        } else {
          // Exact columns: each warp merges its own partial results.
          if (!ok) break;
          if (krow < ctl->cnt[p.b] && bidx != 0xFFFFFFFFu)
            atomicMax(reinterpret_cast<unsigned long long*>(&a.out_key[p.b * a.q_cap + krow]),
                      static_cast<unsigned long long>(make_key(E::ord(best), bidx)));
        }
        ps.eseg ^= 1;
        u += len;
        ps.epar ^= len & 1;
        next_segment(p, ctl, batch);
      }
    }
  }
  __syncthreads();
}

// Drain (every issued MMA and TMA load completes) and release TMEM.
__device__ __forceinline__ void pipe_teardown(Ctl* ctl, uint32_t tmem, int* status) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) { return ptx::smem_u32(&ctl->bars[i]); };
  // Draining waits for work already issued: always the long limit.
  if (threadIdx.x == 0) ctl->wait_ns = kTimeoutNs;
  __syncthreads();
  if (warp >= kMmaWarp0 && lane == 0) {
    ptx::mma_commit(bar(kBarDone));
    wait_bounded(bar(kBarDone), 0, ctl, status);
  }
  if (warp == kProducerWarp && lane == 0) {
    for (int s = 0; s < kMaxStages; ++s)
      if (ctl->p_last_phase[s] >= 0)
        wait_bounded(bar(kBarBFull + s), static_cast<uint32_t>(ctl->p_last_phase[s]), ctl, status);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

template <int DT, int RB>
__global__ void __launch_bounds__(kThreads, 1)
    nn_tc_kernel(const __grid_constant__ CUtensorMap tmap_db, const __grid_constant__ NNArgs a) {
  const SmemLayout L = smem_layout<RB>();
  if ((threadIdx.x >> 5) == kProducerWarp && (threadIdx.x & 31) == 0) ptx::prefetch_tmap(&tmap_db);
  pipe_setup<DT>(L.ctl);
  const uint32_t tmem = L.ctl->tmem_base;
  PipeState ps;
  run_phase<DT, RB, true>(&tmap_db, a, PhaseQ{a.q_index, a.q_count, a.q_bound, 1}, L, tmem, ps);
  pipe_teardown(L.ctl, tmem, a.status);
}

// ---- persistent fast reciprocal matching ----------------------------------

// MASt3R fast reciprocal matching of `batch` pairs in one launch (the round
// loop is fast_rounds); its nearest-neighbour passes run the tensor-core
// pipeline above, whose barrier phases, ring positions and TMEM allocation
// carry over from pass to pass.
template <int DT, int RB>
__global__ void __launch_bounds__(kThreads, 1)
    reciprocal_kernel(const __grid_constant__ CUtensorMap tmap_d2,
                      const __grid_constant__ CUtensorMap tmap_d1,
                      const __grid_constant__ RecArgs r) {
  const SmemLayout L = smem_layout<RB>();
  Ctl* ctl = L.ctl;
  if ((threadIdx.x >> 5) == kProducerWarp && (threadIdx.x & 31) == 0) {
    ptx::prefetch_tmap(&tmap_d1);
    ptx::prefetch_tmap(&tmap_d2);
  }
  pipe_setup<DT>(ctl);
  const uint32_t tmem = ctl->tmem_base;
  PipeState ps;
  auto pass = [&](int dir, const PhaseQ& q) {
    if (dir == 0)
      run_phase<DT, RB, true>(&tmap_d2, r.fwd, q, L, tmem, ps);
    else
      run_phase<DT, RB, true>(&tmap_d1, r.bwd, q, L, tmem, ps);
  };
  // The repack of both maps, when the launcher left it to the kernel, runs in
  // the clearing pass, before the first grid barrier.
  auto repack = [&] {
    if (r.src_nbytes > 0) {
      const int64_t gtid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
      const int64_t gsize = static_cast<int64_t>(gridDim.x) * blockDim.x;
      const int64_t pad = 256;
      repack_in_kernel(r.src1, r.batch * r.N1, r.src_nbytes, RB, const_cast<uint8_t*>(r.bwd.db_rows),
                       pad, DT == FASTNN_I8 ? const_cast<int*>(r.fwd.q_absmax) : nullptr, gtid,
                       gsize);
      repack_in_kernel(r.src2, r.batch * r.N2, r.src_nbytes, RB, const_cast<uint8_t*>(r.fwd.db_rows),
                       pad, DT == FASTNN_I8 ? const_cast<int*>(r.fwd.db_absmax) : nullptr, gtid,
                       gsize);
    }
  };
  fast_rounds<DT>(r, pass, repack, &ctl->abort_flag, &ctl->grid_ok, ctl->scan, ctl->cnt);
  pipe_teardown(ctl, tmem, r.status);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// Optional event pairs around launches (benchmark instrumentation).
struct KernelTimer {
  cudaEvent_t* ev = nullptr;  // 2 * cap events
  int cap = 0;
  int used = 0;
  int kinds = kTimeMatching;  // which launch kinds are bracketed
};
KernelTimer g_timer;

}  // namespace

int kernel_timer_enable(int capacity) {
  const int kinds = g_timer.kinds;
  if (g_timer.ev) {
    for (int i = 0; i < 2 * g_timer.cap; ++i) cudaEventDestroy(g_timer.ev[i]);
    delete[] g_timer.ev;
    g_timer = KernelTimer{};
  }
  g_timer.kinds = kinds;
  if (capacity <= 0) return FASTNN_OK;
  g_timer.ev = new cudaEvent_t[2 * capacity];
  for (int i = 0; i < 2 * capacity; ++i)
    if (cudaEventCreate(&g_timer.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_timer.ev[j]);
      delete[] g_timer.ev;
      g_timer = KernelTimer{};
      g_timer.kinds = kinds;
      return FASTNN_ERR_CUDA;
    }
  g_timer.cap = capacity;
  return FASTNN_OK;
}

int kernel_timer_select(int kinds) {
  const int old = g_timer.kinds;
  if (kinds > 0) g_timer.kinds = kinds;
  return old;
}

int kernel_timer_read(int* launches, double* total_ms) {
  double ms = 0.0;
  for (int i = 0; i < g_timer.used; ++i) {
    FASTNN_CUDA_TRY(cudaEventSynchronize(g_timer.ev[2 * i + 1]));
    float x = 0.f;
    FASTNN_CUDA_TRY(cudaEventElapsedTime(&x, g_timer.ev[2 * i], g_timer.ev[2 * i + 1]));
    ms += x;
  }
  if (launches) *launches = g_timer.used;
  if (total_ms) *total_ms = ms;
  g_timer.used = 0;
  return FASTNN_OK;
}

int nn_tc_min_rows() { return kBN; }
int nn_tc_max_batch() { return kMaxBatch; }

namespace {

int make_tmap(CUtensorMap* tm, const uint8_t* rows, int64_t total_rows, int rb) {
  EncodeFn encode = get_encode();
  if (!encode) return FASTNN_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(total_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(rb), static_cast<cuuint32_t>(kBN)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(rows), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            rb == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                            : rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                       : CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FASTNN_OK : FASTNN_ERR_INVALID;
}

int sm_count(int* sms) {
  int dev = 0;
  FASTNN_CUDA_TRY(cudaGetDevice(&dev));
  FASTNN_CUDA_TRY(cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev));
  return FASTNN_OK;
}

int timer_begin(cudaStream_t stream, int kind) {
  if (!(g_timer.kinds & kind)) return -1;
  const int slot = (g_timer.ev && g_timer.used < g_timer.cap) ? g_timer.used++ : -1;
  if (slot >= 0 && cudaEventRecord(g_timer.ev[2 * slot], stream) != cudaSuccess) return -2;
  return slot;
}

int timer_end(int slot, cudaStream_t stream) {
  if (slot >= 0) FASTNN_CUDA_TRY(cudaEventRecord(g_timer.ev[2 * slot + 1], stream));
  return FASTNN_OK;
}

}  // namespace

int kernel_timer_begin(cudaStream_t stream, int kind) { return timer_begin(stream, kind); }
int kernel_timer_end(int slot, cudaStream_t stream) { return timer_end(slot, stream); }
int device_sm_count(int* sms) { return sm_count(sms); }

namespace {

// Kernel instance for (dtype, row bytes), or nullptr for an unsupported pair.
const void* nn_kernel_for(int dtype, int rb) {
  if (dtype == FASTNN_I8 && rb == 32) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_I8, 32>);
  if (dtype == FASTNN_I8 && rb == 64) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_I8, 64>);
  if (dtype == FASTNN_BF16 && rb == 64) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_BF16, 64>);
  if (dtype == FASTNN_BF16 && rb == 128) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_BF16, 128>);
  if (dtype == FASTNN_F16 && rb == 64) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_F16, 64>);
  if (dtype == FASTNN_F16 && rb == 128) return reinterpret_cast<const void*>(nn_tc_kernel<FASTNN_F16, 128>);
  return nullptr;
}

const void* rec_kernel_for(int dtype, int rb) {
  if (dtype == FASTNN_I8 && rb == 32) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_I8, 32>);
  if (dtype == FASTNN_I8 && rb == 64) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_I8, 64>);
  if (dtype == FASTNN_BF16 && rb == 64) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_BF16, 64>);
  if (dtype == FASTNN_BF16 && rb == 128) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_BF16, 128>);
  if (dtype == FASTNN_F16 && rb == 64) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_F16, 64>);
  if (dtype == FASTNN_F16 && rb == 128) return reinterpret_cast<const void*>(reciprocal_kernel<FASTNN_F16, 128>);
  return nullptr;
}

}  // namespace

int launch_nn_tc(const NNArgs& a, int dtype, int64_t db_total_rows, cudaStream_t stream) {
  const int rb = row_bytes(dtype, a.d);
  if (db_total_rows < kBN || a.batch < 1 || a.batch > kMaxBatch) return FASTNN_ERR_INVALID;
  const void* fn = nn_kernel_for(dtype, rb);
  if (!fn) return FASTNN_ERR_UNSUPPORTED;
  CUtensorMap tm;
  int rc = make_tmap(&tm, a.db_rows, db_total_rows, rb);
  if (rc != FASTNN_OK) return rc;
  int sms = 0;
  if ((rc = sm_count(&sms)) != FASTNN_OK) return rc;
  const size_t smem = smem_bytes(rb, dtype);
  FASTNN_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
  NNArgs args = a;
  void* params[] = {&tm, &args};
  const int slot = timer_begin(stream, kTimeMatching);
  if (slot == -2) return FASTNN_ERR_CUDA;
  FASTNN_CUDA_TRY(cudaLaunchKernel(fn, dim3(sms), dim3(kThreads), params, smem, stream));
  return timer_end(slot, stream);
}

int launch_reciprocal(const RecArgs& r, int dtype, int64_t d1_rows, int64_t d2_rows,
                      cudaStream_t stream) {
  const int rb = row_bytes(dtype, r.fwd.d);
  if (d1_rows < kBN || d2_rows < kBN || r.batch < 1 || r.batch > kMaxBatch)
    return FASTNN_ERR_INVALID;
  const void* fn = rec_kernel_for(dtype, rb);
  if (!fn) return FASTNN_ERR_UNSUPPORTED;
  CUtensorMap tm2, tm1;
  int rc = make_tmap(&tm2, r.fwd.db_rows, d2_rows, rb);
  if (rc != FASTNN_OK) return rc;
  if ((rc = make_tmap(&tm1, r.bwd.db_rows, d1_rows, rb)) != FASTNN_OK) return rc;
  int sms = 0;
  if ((rc = sm_count(&sms)) != FASTNN_OK) return rc;
  const size_t smem = smem_bytes(rb, dtype);
  FASTNN_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
  int per_sm = 0;
  FASTNN_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem));
  if (per_sm < 1) return FASTNN_ERR_UNSUPPORTED;
  RecArgs args = r;
  void* params[] = {&tm2, &tm1, &args};
  const int slot = timer_begin(stream, kTimeMatching);
  if (slot == -2) return FASTNN_ERR_CUDA;
  FASTNN_CUDA_TRY(cudaLaunchCooperativeKernel(fn, dim3(sms), dim3(kThreads), params, smem, stream));
  return timer_end(slot, stream);
}

}  // namespace fastnn
