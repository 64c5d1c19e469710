// Memory-bound kernels around the nearest-neighbour passes:
//   repack          descriptor rows [rows][d] -> zero-padded [rows][32 elems]
//   mutual_*        dense mutual-pair test and ordered emission
//   decode_nn       packed keys -> (index, score)
// (The fast scheme's seeds and per-round check/compaction run inside the
// persistent matching kernel, see frontier_dev.cuh and nn_tc.cu.)
#include "common.cuh"
#include "frontier.cuh"
#include "frontier_dev.cuh"
#include "nn_tc.cuh"

namespace fastnn {

namespace {

// ---------------------------------------------------------------- repack ---
// One thread per output row. Source rows of d elements (ESIZE bytes each) are
// copied into RB-byte rows (K = 32 or 64 elements) with zero padding, so every
// row is 16-byte aligned for TMA and the MMA's K extent is a whole number of
// 32-byte steps.
// For int8 maps, `absmax` (if given) receives max |element| over the map
// (atomicMax), which tells the nearest-neighbour kernel whether every score
// fits in 16 bits.
template <int ESIZE, int RB>
__global__ void repack_kernel(const uint8_t* __restrict__ src, int64_t rows, int d,
                              uint8_t* __restrict__ dst, int64_t pad_rows, int* absmax) {
  constexpr int NW = RB / 4;
  const int nbytes = d * ESIZE;
  const bool words = (nbytes % 4) == 0 && (reinterpret_cast<uintptr_t>(src) % 4) == 0;
  int amax = 0;
  for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       row < rows + pad_rows; row += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint32_t w[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0;
    if (row < rows) {
      const uint8_t* s = src + row * nbytes;
      if (words) {
        const uint32_t* s32 = reinterpret_cast<const uint32_t*>(s);
#pragma unroll
        for (int i = 0; i < NW; ++i)
          if (i < nbytes / 4) w[i] = __ldg(s32 + i);
      } else {
#pragma unroll
        for (int i = 0; i < RB; ++i)
          if (i < nbytes) w[i / 4] |= static_cast<uint32_t>(__ldg(s + i)) << (8 * (i % 4));
      }
    }
    if (ESIZE == 1 && absmax) {
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        const uint32_t x = w[i];
#pragma unroll
        for (int k = 0; k < 4; ++k) amax = max(amax, abs(static_cast<int>(static_cast<int8_t>(x >> (8 * k)))));
      }
    }
    uint4* o = reinterpret_cast<uint4*>(dst + row * RB);
#pragma unroll
    for (int i = 0; i < RB / 16; ++i) o[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
  if (ESIZE == 1 && absmax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0 && amax > 0) atomicMax(absmax, amax);
  }
}

// Staged repack for source rows of a whole number of 8-byte words (int8
// d = 8, 16, 24, 32, ...; 16-bit d = 4, 8, 12, ...) from a 16-byte aligned
// source: a block copies a run of kRepackRows rows with coalesced 16-byte
// loads into shared memory (kRepackRows * nbytes is a multiple of 16, so every
// run starts 16-byte aligned), then writes the run's padded rows with
// coalesced 16-byte stores, each thread assembling its output chunk from two
// 8-byte words of the staged rows. This is a pure stream: every input byte is
// read once and every output byte written once.
constexpr int kRepackRows = 256;
constexpr int kRepackThreads = 256;

template <int RB>
__global__ void __launch_bounds__(kRepackThreads)
    repack_staged_kernel(const uint8_t* __restrict__ src, int64_t rows, int nbytes,
                         uint8_t* __restrict__ dst, int64_t pad_rows, int* absmax) {
  constexpr int kOutChunks = kRepackRows * RB / 16;  // 16-byte output chunks of a run
  __shared__ __align__(16) uint8_t stage[kRepackRows * RB];  // nbytes <= RB per row
  const int64_t total = rows + pad_rows;
  const int64_t runs = (total + kRepackRows - 1) / kRepackRows;
  const int64_t in_bytes = rows * nbytes;
  uint32_t amax = 0;  // per-byte maxima of |x| (int8 maps only)
  for (int64_t run = blockIdx.x; run < runs; run += gridDim.x) {
    const int64_t r0 = run * kRepackRows;
    const int64_t b0 = r0 * nbytes;  // first source byte of the run (16-byte aligned)
    const int run_bytes = static_cast<int>(
        max(static_cast<int64_t>(0), min(static_cast<int64_t>(kRepackRows) * nbytes, in_bytes - b0)));
    // Load: full 16-byte chunks, then the run's ragged tail (at most 15 bytes).
    const int full = run_bytes / 16;
    for (int c = threadIdx.x; c < full; c += kRepackThreads) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + b0) + c);
      reinterpret_cast<uint4*>(stage)[c] = v;
      if (absmax) {
        amax = __vmaxu4(amax, __vabs4(v.x));
        amax = __vmaxu4(amax, __vabs4(v.y));
        amax = __vmaxu4(amax, __vabs4(v.z));
        amax = __vmaxu4(amax, __vabs4(v.w));
      }
    }
    if (static_cast<int>(threadIdx.x) < run_bytes - 16 * full) {
      const int i = 16 * full + threadIdx.x;
      const uint8_t x = __ldg(src + b0 + i);
      stage[i] = x;
      if (absmax) amax = __vmaxu4(amax, __vabs4(static_cast<uint32_t>(x) * 0x01010101u) & 0xFFu);
    }
    __syncthreads();
    // Store: output chunk k covers bytes [16 (k mod RB/16), +16) of row k / (RB/16).
    for (int k = threadIdx.x; k < kOutChunks; k += kRepackThreads) {
      const int r = k / (RB / 16);
      const int off = 16 * (k % (RB / 16));
      const int64_t row = r0 + r;
      if (row >= total) break;
      uint2 lo = make_uint2(0, 0), hi = make_uint2(0, 0);
      if (row < rows) {
        const uint8_t* srow = stage + r * nbytes;  // 8-byte aligned: nbytes % 8 == 0
        if (off < nbytes) lo = *reinterpret_cast<const uint2*>(srow + off);
        if (off + 8 < nbytes) hi = *reinterpret_cast<const uint2*>(srow + off + 8);
      }
      reinterpret_cast<uint4*>(dst + row * RB)[off / 16] = make_uint4(lo.x, lo.y, hi.x, hi.y);
    }
    __syncthreads();
  }
  if (absmax) {
    int m = static_cast<int>(max(max(amax & 0xFFu, (amax >> 8) & 0xFFu),
                                 max((amax >> 16) & 0xFFu, amax >> 24)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0) atomicMax(absmax, m);
  }
}

// ---------------------------------------------------------- dense mutual ---
// flag(i) = NN21(NN12(i)) == i0 + i for local image-1 row i. The NN results
// come either as packed keys (single-GPU dense path) or as index arrays plus
// scores (a row shard of image 1 checked against the full NN21 gathered from
// every rank). Three passes keep the output in ascending i without inter-CTA
// waiting: per-block counts, one scan block, ordered emit.
// A block covers kMutBlockRows rows. In the mutual test thread t of
// kMutThreads takes the eight consecutive rows 8t .. 8t + 7, two groups of
// four read with 16-byte loads where aligned, whose gathers of the partners'
// back-matches are in flight together.
constexpr int kMutBlockRows = 4096;
constexpr int kMutRowsPerThread = 8;
constexpr int kMutThreads = kMutBlockRows / kMutRowsPerThread;

// Partners NN12 of rows i .. i + 3 (local indices).
__device__ __forceinline__ void mutual_partners4(const MutualSrc& m, int64_t i,
                                                 uint32_t (&j)[4]) {
  const bool full = i + 3 < m.n1;
  if (m.k12) {
    uint64_t k[4] = {0, 0, 0, 0};
    if (full && (reinterpret_cast<uintptr_t>(m.k12 + i) & 15) == 0) {
      const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(m.k12 + i);
      const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(m.k12 + i + 2);
      k[0] = a.x; k[1] = a.y; k[2] = b.x; k[3] = b.y;
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r) k[r] = i + r < m.n1 ? m.k12[i + r] : 0;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) j[r] = key_index(k[r]);
  } else {
    if (full && (reinterpret_cast<uintptr_t>(m.nn12 + i) & 15) == 0) {
      const int4 a = *reinterpret_cast<const int4*>(m.nn12 + i);
      j[0] = a.x; j[1] = a.y; j[2] = a.z; j[3] = a.w;
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r) j[r] = i + r < m.n1 ? static_cast<uint32_t>(m.nn12[i + r]) : 0xFFFFFFFFu;
    }
  }
}

// Flags (and partners) of rows i .. i + 3. The partners' back-matches are
// loaded together, after all four partners are known.
__device__ __forceinline__ void mutual_flags4(const MutualSrc& m, int64_t i, bool (&f)[4],
                                              uint32_t (&j)[4]) {
  mutual_partners4(m, i, j);
  uint32_t back[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const bool ok = i + r < m.n1 && j[r] < static_cast<uint64_t>(m.n2);
    back[r] = !ok ? 0xFFFFFFFFu
              : m.k21 ? key_index(m.k21[m.pos21 ? m.pos21[j[r]] : j[r]])
                      : static_cast<uint32_t>(m.nn21[j[r]]);
    f[r] = ok && back[r] == static_cast<uint32_t>(m.i0 + i + r);
  }
}

// Output score bits of rows i .. i + 3, loaded whatever the keep flags say
// (at the usual share of kept rows every sector holds some), so that the
// loads go out with the partners' and not after the flags: the key's score in
// the output type (the keys were just read for the partners: cache hits), or
// score12[i] (read once: streamed), or 0 when there is neither.
template <int DT>
__device__ __forceinline__ void mutual_scores4(const MutualSrc& m, int64_t i, uint32_t (&sv)[4]) {
  const bool full = i + 3 < m.n1;
  if (m.k12) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const uint32_t h = i + r < m.n1 ? key_score_bits(m.k12[i + r]) : 0u;
      sv[r] = DT == FASTNN_I8      ? static_cast<uint32_t>(unord_i32(h))
              : DT == FASTNN_F32_L2 ? __float_as_uint(-unord_f32(h))
                                    : __float_as_uint(unord_f32(h));
    }
  } else if (m.score12) {
    const uint32_t* s = static_cast<const uint32_t*>(m.score12) + i;
    if (full && (reinterpret_cast<uintptr_t>(s) & 15) == 0) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(s));
      sv[0] = v.x; sv[1] = v.y; sv[2] = v.z; sv[3] = v.w;
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r) sv[r] = i + r < m.n1 ? s[r] : 0u;
    }
  } else {
#pragma unroll
    for (int r = 0; r < 4; ++r) sv[r] = 0u;
  }
}

// The count pass also records each thread's eight keep flags as one byte, so
// that the emit pass reads them instead of gathering the back-matches again.
__global__ void __launch_bounds__(kMutThreads) mutual_count_kernel(MutualSrc m,
                                                                   int32_t* __restrict__ block_cnt,
                                                                   uint8_t* __restrict__ keep) {
  __shared__ int sm[32];
  const int64_t i =
      blockIdx.x * static_cast<int64_t>(kMutBlockRows) + kMutRowsPerThread * threadIdx.x;
  bool f[2][4];
  uint32_t j[2][4];
  mutual_flags4(m, i, f[0], j[0]);
  mutual_flags4(m, i + 4, f[1], j[1]);
  uint32_t bits = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r) bits |= (f[r >> 2][r & 3] ? 1u : 0u) << r;
  keep[blockIdx.x * static_cast<int64_t>(kMutThreads) + threadIdx.x] = static_cast<uint8_t>(bits);
  int c = __popc(bits);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += sm[w];
    block_cnt[blockIdx.x] = t;
  }
}

// Block-wide exclusive scan of one small count per thread; `sm` holds 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int c, int* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < warp; ++w) off += sm[w];
  return off + x - c;
}

// Exclusive scan, in place, of the nblocks counts of segment blockIdx.x
// (block_cnt + blockIdx.x * nblocks); the segment's total goes to
// out_count[blockIdx.x]. The counts go through shared memory in tiles of
// kScanTile: coalesced loads, kScanPer consecutive counts per thread (the
// index is padded by one word per 32 so that those reads are free of bank
// conflicts), one block scan of the per-thread sums, coalesced stores; the
// running total carries from tile to tile.
constexpr int kScanPer = 8;
constexpr int kScanTile = 1024 * kScanPer;

__device__ __forceinline__ int scan_slot(int k) { return k + (k >> 5); }

__global__ void __launch_bounds__(1024) mutual_scan_kernel(int32_t* __restrict__ block_cnt,
                                                           int nblocks,
                                                           int32_t* __restrict__ out_count) {
  block_cnt += static_cast<int64_t>(blockIdx.x) * nblocks;
  out_count += blockIdx.x;
  __shared__ int buf[kScanTile + kScanTile / 32];
  __shared__ int sm[32];
  __shared__ int carry_s;
  int carry = 0;
  for (int t0 = 0; t0 < nblocks; t0 += kScanTile) {
    const int n = min(kScanTile, nblocks - t0);
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      const int k = static_cast<int>(threadIdx.x) + 1024 * i;
      buf[scan_slot(k)] = k < n ? block_cnt[t0 + k] : 0;
    }
    __syncthreads();
    int v[kScanPer];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      v[i] = buf[scan_slot(static_cast<int>(threadIdx.x) * kScanPer + i)];
      sum += v[i];
    }
    int run = carry + block_exclusive_scan(sum, sm);
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      buf[scan_slot(static_cast<int>(threadIdx.x) * kScanPer + i)] = run;
      run += v[i];
    }
    if (threadIdx.x == blockDim.x - 1) carry_s = run;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      const int k = static_cast<int>(threadIdx.x) + 1024 * i;
      if (k < n) block_cnt[t0 + k] = buf[scan_slot(k)];
    }
    carry = carry_s;
    __syncthreads();  // buf, sm and carry_s are reused by the next tile
  }
  if (threadIdx.x == 0) *out_count = carry;
}

// The emit pass: the block's kept pairs (and scores) are placed in shared
// memory in row order, then stored to consecutive output slots by
// consecutive threads.
constexpr int kMutEmitSmem = kMutBlockRows * (8 + 4);

template <int DT>
__global__ void __launch_bounds__(kMutThreads) mutual_emit_kernel(
    MutualSrc m, const int32_t* __restrict__ block_off, const uint8_t* __restrict__ keep,
    int32_t* __restrict__ out_pairs, void* __restrict__ out_score, int64_t cap) {
  extern __shared__ __align__(16) uint8_t mut_stage[];
  int2* sp = reinterpret_cast<int2*>(mut_stage);
  uint32_t* ss = reinterpret_cast<uint32_t*>(mut_stage + kMutBlockRows * 8);
  __shared__ int sm[32];
  const int64_t i =
      blockIdx.x * static_cast<int64_t>(kMutBlockRows) + kMutRowsPerThread * threadIdx.x;
  const uint32_t bits = keep[blockIdx.x * static_cast<int64_t>(kMutThreads) + threadIdx.x];
  uint32_t j[2][4], sv[2][4];
  mutual_partners4(m, i, j[0]);
  mutual_partners4(m, i + 4, j[1]);
  if (out_score) {
    mutual_scores4<DT>(m, i, sv[0]);
    mutual_scores4<DT>(m, i + 4, sv[1]);
  }
  int local = block_exclusive_scan(__popc(bits), sm);
  int total = 0;
  for (int w = 0; w < kMutThreads / 32; ++w) total += sm[w];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (!((bits >> r) & 1u)) continue;
    const int64_t ir = i + r;
    const uint32_t jr = j[r >> 2][r & 3];
    const int32_t a = m.map1 ? m.map1[ir] : static_cast<int32_t>(m.i0 + ir);
    const int32_t bj = m.map2 ? m.map2[jr] : static_cast<int32_t>(jr);
    sp[local] = make_int2(a, bj);
    if (out_score) ss[local] = sv[r >> 2][r & 3];
    ++local;
  }
  __syncthreads();
  const int64_t base = block_off[blockIdx.x];
  const int n = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(total), cap - base)));
  const bool pair8 = (reinterpret_cast<uintptr_t>(out_pairs) & 7) == 0;
  for (int k = threadIdx.x; k < n; k += kMutThreads) {
    const int2 v = sp[k];
    if (pair8) {
      *reinterpret_cast<int2*>(out_pairs + (base + k) * 2) = v;
    } else {
      out_pairs[(base + k) * 2] = v.x;
      out_pairs[(base + k) * 2 + 1] = v.y;
    }
    if (out_score) static_cast<uint32_t*>(out_score)[base + k] = ss[k];
  }
}

// ------------------------------------------------------- chunk boxes ---
__global__ void __launch_bounds__(256) chunk_box_kernel(const float4* __restrict__ rows,
                                                        int64_t N, int nchunk,
                                                        const int32_t* __restrict__ count,
                                                        float4* __restrict__ box) {
  const int b = blockIdx.x / nchunk, c = blockIdx.x % nchunk;
  const int64_t n = count ? min(static_cast<int64_t>(count[b]), N) : N;
  const int64_t r0 = static_cast<int64_t>(c) * kL2Chunk;
  const int64_t r1 = min(r0 + kL2Chunk, n);
  float lo[3] = {INFINITY, INFINITY, INFINITY}, hi[3] = {-INFINITY, -INFINITY, -INFINITY};
  for (int64_t r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    const float4 p = __ldg(rows + b * N + r);
    lo[0] = fminf(lo[0], p.x);
    lo[1] = fminf(lo[1], p.y);
    lo[2] = fminf(lo[2], p.z);
    hi[0] = fmaxf(hi[0], p.x);
    hi[1] = fmaxf(hi[1], p.y);
    hi[2] = fmaxf(hi[2], p.z);
  }
  __shared__ float sm[6][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo[k] = fminf(lo[k], __shfl_xor_sync(0xffffffffu, lo[k], o));
      hi[k] = fmaxf(hi[k], __shfl_xor_sync(0xffffffffu, hi[k], o));
    }
    if (lane == 0) {
      sm[k][warp] = lo[k];
      sm[3 + k][warp] = hi[k];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float l[3], h[3];
    for (int k = 0; k < 3; ++k) {
      l[k] = sm[k][0];
      h[k] = sm[3 + k][0];
      for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) {
        l[k] = fminf(l[k], sm[k][w]);
        h[k] = fmaxf(h[k], sm[3 + k][w]);
      }
    }
    box[2 * static_cast<int64_t>(blockIdx.x)] = make_float4(l[0], l[1], l[2], 0.f);
    box[2 * static_cast<int64_t>(blockIdx.x) + 1] = make_float4(h[0], h[1], h[2], 0.f);
  }
}

// ------------------------------------------------- image of the matching ---
// Rows of image 2 that are some image-1 row's forward match: only they can
// be in a mutual pair, so the backward pass runs on them alone.
// The best forward score among the rows matched to j is a score NN21(j)
// reaches (the same dot product, or distance, with the roles swapped).
__global__ void image_mark_kernel(const uint64_t* __restrict__ k12, int64_t n1, int64_t n2,
                                  uint32_t* __restrict__ first, uint32_t* __restrict__ best) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n1;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t key = k12[i];
    const uint32_t j = key_index(key);
    if (j < static_cast<uint64_t>(n2)) {
      atomicMin(first + j, static_cast<uint32_t>(i));
      atomicMax(best + j, key_score_bits(key));
    }
  }
}

// Row i of image 1 introduces j = NN12(i) when it is the first row matched to j.
__device__ __forceinline__ bool image_first(const uint64_t* k12, const uint32_t* first, int64_t n1,
                                            int64_t n2, int64_t i, uint32_t& j) {
  if (i >= n1) return false;
  j = key_index(k12[i]);
  return j < static_cast<uint64_t>(n2) && first[j] == static_cast<uint32_t>(i);
}

__global__ void __launch_bounds__(1024) image_count_kernel(const uint64_t* __restrict__ k12,
                                                           const uint32_t* __restrict__ first,
                                                           int64_t n1, int64_t n2,
                                                           int32_t* __restrict__ block_cnt) {
  __shared__ int sm[64];
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t j;
  const Scan2 sc = block_scan2(image_first(k12, first, n1, n2, i, j), false, sm);
  if (threadIdx.x == 0) block_cnt[blockIdx.x] = sc.tot0;
}

__global__ void __launch_bounds__(1024) image_emit_kernel(const uint64_t* __restrict__ k12,
                                                          const uint32_t* __restrict__ first,
                                                          const uint32_t* __restrict__ best,
                                                          int64_t n1, int64_t n2,
                                                          const int32_t* __restrict__ block_off,
                                                          int32_t* __restrict__ pos,
                                                          int32_t* __restrict__ list,
                                                          uint32_t* __restrict__ list_bound) {
  __shared__ int sm[64];
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t j = 0;
  const bool f = image_first(k12, first, n1, n2, i, j);
  const Scan2 sc = block_scan2(f, false, sm);
  if (f) {
    const int32_t slot = block_off[blockIdx.x] + sc.ex0;
    list[slot] = static_cast<int32_t>(j);
    list_bound[slot] = best[j];
    pos[j] = slot;
  }
}

// ---------------------------------------------- image rows of an NN12 ---
// The ascending list of image-2 rows j in [0, n2) that some nn12[i] names:
// byte flags, per-block counts, the shared scan, an ordered emit. A block of
// kImgThreads threads covers kMutBlockRows rows (the scan's block count is
// the dense mutual test's); thread t takes the 32 consecutive flags
// 32t .. 32t + 31, two 16-byte loads in flight together.
constexpr int kImgFlagsPerThread = 32;
constexpr int kImgThreads = kMutBlockRows / kImgFlagsPerThread;

__global__ void image_flag_kernel(const int32_t* __restrict__ nn12, int64_t n1, int64_t n2,
                                  uint8_t* __restrict__ flag) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(nn12) & 15) == 0) {
    const int64_t n4 = n1 >> 2;
    for (int64_t q = t; q < n4; q += stride) {
      // Streamed with the evict-first hint, so that the flag array (one byte
      // per image-2 row) rather than NN12 stays in L2 for the passes after.
      const int4 v = __ldcs(reinterpret_cast<const int4*>(nn12 + 4 * q));
      if (v.x >= 0 && v.x < n2) flag[v.x] = 1;
      if (v.y >= 0 && v.y < n2) flag[v.y] = 1;
      if (v.z >= 0 && v.z < n2) flag[v.z] = 1;
      if (v.w >= 0 && v.w < n2) flag[v.w] = 1;
    }
    for (int64_t i = 4 * n4 + t; i < n1; i += stride) {
      const int32_t j = nn12[i];
      if (j >= 0 && j < n2) flag[j] = 1;
    }
  } else {
    for (int64_t i = t; i < n1; i += stride) {
      const int32_t j = nn12[i];
      if (j >= 0 && j < n2) flag[j] = 1;
    }
  }
}

// Bit r of the result: flag[j + r] is set (r < 32; rows at or past n2 read 0).
__device__ __forceinline__ uint32_t image_flags32(const uint8_t* flag, int64_t n2, int64_t j) {
  uint32_t bits = 0;
  if (j + 31 < n2) {
    // j is a multiple of 32 and the flag array starts 16-byte aligned.
    const uint4 v0 = *reinterpret_cast<const uint4*>(flag + j);
    const uint4 v1 = *reinterpret_cast<const uint4*>(flag + j + 16);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int b = 0; b < 4; ++b)
        bits |= (((w[q] >> (8 * b)) & 0xFFu) != 0u ? 1u : 0u) << (4 * q + b);
  } else {
    for (int r = 0; r < 32; ++r)
      if (j + r < n2 && flag[j + r]) bits |= 1u << r;
  }
  return bits;
}

__global__ void __launch_bounds__(kImgThreads) image_rows_count_kernel(
    const uint8_t* __restrict__ flag, int64_t n2, int32_t* __restrict__ block_cnt) {
  __shared__ int sm[32];
  const int64_t j =
      blockIdx.x * static_cast<int64_t>(kMutBlockRows) + kImgFlagsPerThread * threadIdx.x;
  int c = __popc(image_flags32(flag, n2, j));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kImgThreads / 32; ++w) t += sm[w];
    block_cnt[blockIdx.x] = t;
  }
}

// The block's rows are staged in shared memory in order and stored with
// consecutive threads writing consecutive words.
__global__ void __launch_bounds__(kImgThreads) image_rows_emit_kernel(
    const uint8_t* __restrict__ flag, int64_t n2, const int32_t* __restrict__ off,
    int32_t* __restrict__ rows) {
  __shared__ int sm[32];
  __shared__ int32_t stage[kMutBlockRows];
  const int64_t j0 = blockIdx.x * static_cast<int64_t>(kMutBlockRows);
  const int64_t j = j0 + kImgFlagsPerThread * threadIdx.x;
  uint32_t bits = image_flags32(flag, n2, j);
  int p = block_exclusive_scan(__popc(bits), sm);
  while (bits) {
    const int r = __ffs(bits) - 1;
    bits &= bits - 1;
    stage[p++] = static_cast<int32_t>(j + r);
  }
  int total = 0;
  for (int w = 0; w < kImgThreads / 32; ++w) total += sm[w];
  __syncthreads();
  int32_t* dst = rows + off[blockIdx.x];
  for (int k = threadIdx.x; k < total; k += kImgThreads) dst[k] = stage[k];
}

// ------------------------------------------------------------ decode nn ---
template <int DT>
__global__ void decode_kernel(const uint64_t* __restrict__ key, int64_t n,
                              int32_t* __restrict__ out_idx, void* __restrict__ out_score) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t k = key[i];
    out_idx[i] = static_cast<int32_t>(key_index(k));
    if (out_score) {
      if (DT == FASTNN_I8)
        static_cast<int32_t*>(out_score)[i] = unord_i32(key_score_bits(k));
      else if (DT == FASTNN_F32_L2)
        static_cast<float*>(out_score)[i] = k ? -unord_f32(key_score_bits(k)) : INFINITY;
      else
        static_cast<float*>(out_score)[i] = unord_f32(key_score_bits(k));
    }
  }
}

// Pointmap rows: float32 [rows][d] (d <= 3) -> float4 (x, y, z, -|p|^2),
// missing coordinates zero; pad_rows zero rows follow. The norm is computed
// in fp32 as fma(z, z, fma(y, y, x * x)); its maximum over the map goes to
// *max_p2 (fp32 bits; non-negative floats order like their bits).
__global__ void repack_l2_kernel(const float* __restrict__ src, int64_t rows, int d,
                                 float4* __restrict__ dst, int64_t pad_rows, int* max_p2) {
  float mx = 0.f;
  for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       row < rows + pad_rows; row += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < rows) {
      const float* s = src + row * d;
      p.x = __ldg(s);
      if (d > 1) p.y = __ldg(s + 1);
      if (d > 2) p.z = __ldg(s + 2);
      const float n2 = __fmaf_rn(p.z, p.z, __fmaf_rn(p.y, p.y, p.x * p.x));
      p.w = -n2;
      mx = fmaxf(mx, n2);
    }
    dst[row] = p;
  }
  if (max_p2) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0 && mx > 0.f) atomicMax(max_p2, __float_as_int(mx));
  }
}

int grid_for(int64_t n, int threads, int max_blocks = 148 * 16) {
  int64_t g = (n + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > max_blocks) g = max_blocks;
  return static_cast<int>(g);
}

// ------------------------------------------------------- confidence masks ---
// A pixel takes part iff its confidence is at least the threshold (no map:
// every pixel). Each map is compacted, in pixel order, to its kept rows:
// per-block counts, a per-pair scan of the counts, then an ordered scatter
// that repacks each kept row into slot (pair b, position) and records the
// slot's pixel (c2p) and the pixel's slot (p2c, -1 when dropped). Order is
// kept, so the lowest compacted index among equal scores is the lowest pixel.
__device__ __forceinline__ bool mask_kept(const MaskArgs& m, int64_t g) {
  return !m.conf || __ldg(m.conf + g) >= m.threshold;
}

// Kept pixels of each 1024-pixel block: 256 threads, four consecutive
// pixels each (one 16-byte load of confidences where aligned).
__global__ void __launch_bounds__(256) mask_count_kernel(MaskArgs m) {
  __shared__ int sm[8];
  const int b = blockIdx.x / m.bpp, blk = blockIdx.x % m.bpp;
  const int64_t p = static_cast<int64_t>(blk) * 1024 + 4 * threadIdx.x;
  const int64_t g = b * m.N + p;
  uint32_t bits = 0;
  if (m.conf && p + 3 < m.N && (reinterpret_cast<uintptr_t>(m.conf + g) & 15) == 0) {
    const float4 c4 = __ldg(reinterpret_cast<const float4*>(m.conf + g));
    bits = (c4.x >= m.threshold ? 1u : 0u) | (c4.y >= m.threshold ? 2u : 0u) |
           (c4.z >= m.threshold ? 4u : 0u) | (c4.w >= m.threshold ? 8u : 0u);
  } else {
#pragma unroll
    for (int r = 0; r < 4; ++r) bits |= (p + r < m.N && mask_kept(m, g + r)) ? (1u << r) : 0u;
  }
  int c = __popc(bits);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += sm[w];
    m.blocks[blockIdx.x] = t;
  }
}

// Descriptor row (ESIZE-byte elements) into an RB-byte slot; returns max
// |element| for int8 rows, 0 otherwise.
template <int ESIZE, int RB>
__device__ __forceinline__ int repack_row(const uint8_t* __restrict__ s, int d,
                                          uint8_t* __restrict__ o) {
  constexpr int NW = RB / 4;
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0;
  const int nbytes = d * ESIZE;
#pragma unroll
  for (int i = 0; i < RB; ++i)
    if (i < nbytes) w[i / 4] |= static_cast<uint32_t>(__ldg(s + i)) << (8 * (i % 4));
  int amax = 0;
  if (ESIZE == 1) {
#pragma unroll
    for (int i = 0; i < NW; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        amax = max(amax, abs(static_cast<int>(static_cast<int8_t>(w[i] >> (8 * k)))));
  }
  uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
  for (int i = 0; i < RB / 16; ++i) o4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  return amax;
}

// Pointmap row into a float4 (x, y, z, -|p|^2); returns the fp32 bits of |p|^2.
__device__ __forceinline__ int repack_point(const float* __restrict__ s, int d, float4* o) {
  float4 p = make_float4(__ldg(s), d > 1 ? __ldg(s + 1) : 0.f, d > 2 ? __ldg(s + 2) : 0.f, 0.f);
  const float n2 = __fmaf_rn(p.z, p.z, __fmaf_rn(p.y, p.y, p.x * p.x));
  p.w = -n2;
  *o = p;
  return __float_as_int(n2);
}

// KIND 0: descriptor rows (ESIZE, RB); KIND 1: pointmap rows.
template <int KIND, int ESIZE, int RB>
__global__ void __launch_bounds__(1024) mask_emit_kernel(MaskArgs m) {
  __shared__ int sm[64];
  const int b = blockIdx.x / m.bpp, blk = blockIdx.x % m.bpp;
  const int64_t p = static_cast<int64_t>(blk) * 1024 + threadIdx.x;
  const int64_t g = b * m.N + p;
  const bool f = p < m.N && mask_kept(m, g);
  const Scan2 sc = block_scan2(f, false, sm);
  int mag = 0;
  if (p < m.N) {
    const int64_t slot = b * m.N + m.blocks[blockIdx.x] + sc.ex0;
    if (m.p2c) m.p2c[g] = f ? static_cast<int32_t>(slot - b * m.N) : -1;
    if (f) {
      m.c2p[slot] = static_cast<int32_t>(p);
      if (KIND == 1)
        mag = repack_point(reinterpret_cast<const float*>(m.src) + g * m.d, m.d,
                           reinterpret_cast<float4*>(m.dst) + slot);
      else
        mag = repack_row<ESIZE, RB>(m.src + g * m.d * ESIZE, m.d, m.dst + slot * RB);
    }
  }
  if (m.absmax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
    if ((threadIdx.x & 31) == 0 && mag > 0) atomicMax(m.absmax, mag);
  }
}

// Staged form of the ordered scatter, for descriptor rows of a whole number
// of 8-byte words in a 16-byte aligned map whose pairs start 16-byte aligned.
// Block blk of pair b covers the same 1024 pixels as mask_count_kernel's: it
// loads their rows with coalesced 16-byte loads into shared memory
// (1024 * nbytes bytes of dynamic shared memory), then places and writes the
// kept rows in four rounds of 256 pixels.
constexpr int kMaskEmitThreads = 256;

template <int RB, bool I8>
__global__ void __launch_bounds__(kMaskEmitThreads) mask_emit_staged_kernel(MaskArgs m,
                                                                            int nbytes) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ int sm[64];
  const int b = blockIdx.x / m.bpp, blk = blockIdx.x % m.bpp;
  const int tid = static_cast<int>(threadIdx.x);
  const int64_t p0 = static_cast<int64_t>(blk) * 1024;
  const int rows = static_cast<int>(min(static_cast<int64_t>(1024), m.N - p0));
  const uint8_t* src = m.src + (b * m.N + p0) * nbytes;
  const int bytes = rows * nbytes;  // a multiple of 8
  for (int c = tid; c < bytes / 16; c += kMaskEmitThreads)
    reinterpret_cast<uint4*>(stage)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  if (tid == 0 && (bytes & 15))
    *reinterpret_cast<uint2*>(stage + bytes - 8) =
        __ldg(reinterpret_cast<const uint2*>(src + bytes - 8));
  // Four rounds of 256 pixels; in round r thread t takes pixel p0 + 256 r + t,
  // so a round's kept rows go to consecutive slots from consecutive threads.
  // The first scan's barriers also publish the staged rows. The four rounds'
  // keep flags are read up front, with the staging loads.
  constexpr int kRounds = 1024 / kMaskEmitThreads;
  bool keep[kRounds];
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int lr = r * kMaskEmitThreads + tid;
    keep[r] = lr < rows && mask_kept(m, b * m.N + p0 + lr);
  }
  int64_t base = b * m.N + m.blocks[blockIdx.x];
  uint32_t amax = 0;  // per-byte maxima of |x| (int8)
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int lr = r * kMaskEmitThreads + tid;  // row within the block
    const int64_t p = p0 + lr;
    const int64_t g = b * m.N + p;
    const bool f = keep[r];
    const Scan2 sc = block_scan2(f, false, sm);
    const int64_t slot = base + sc.ex0;
    base += sc.tot0;
    if (lr < rows && m.p2c) m.p2c[g] = f ? static_cast<int32_t>(slot - b * m.N) : -1;
    if (!f) continue;
    m.c2p[slot] = static_cast<int32_t>(p);
    const uint8_t* srow = stage + lr * nbytes;  // 8-byte aligned
    uint4* o = reinterpret_cast<uint4*>(m.dst + slot * RB);
#pragma unroll
    for (int c = 0; c < RB / 16; ++c) {
      uint2 lo = make_uint2(0, 0), hi = make_uint2(0, 0);
      if (16 * c < nbytes) lo = *reinterpret_cast<const uint2*>(srow + 16 * c);
      if (16 * c + 8 < nbytes) hi = *reinterpret_cast<const uint2*>(srow + 16 * c + 8);
      o[c] = make_uint4(lo.x, lo.y, hi.x, hi.y);
      if (I8)
        amax = __vmaxu4(__vmaxu4(amax, __vabs4(lo.x)),
                        __vmaxu4(__vmaxu4(__vabs4(lo.y), __vabs4(hi.x)), __vabs4(hi.y)));
    }
  }
  if (I8 && m.absmax) {
    int mag = static_cast<int>(max(max(amax & 0xFFu, (amax >> 8) & 0xFFu),
                                   max((amax >> 16) & 0xFFu, amax >> 24)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
    if ((threadIdx.x & 31) == 0 && mag > 0) atomicMax(m.absmax, mag);
  }
}

// Launch of the staged scatter for rows of RB repacked bytes.
template <int RB, bool I8>
int launch_mask_emit_staged(const MaskArgs& m, int nb, int nbytes, cudaStream_t st) {
  const int smem = 1024 * nbytes;
  // Above 48 KB of shared memory in all (static included) a kernel must opt in.
  FASTNN_CUDA_TRY(cudaFuncSetAttribute(mask_emit_staged_kernel<RB, I8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  mask_emit_staged_kernel<RB, I8><<<nb, kMaskEmitThreads, smem, st>>>(m, nbytes);
  return FASTNN_OK;
}

// Seeds of the masked fast scheme: the kept grid pixels of each pair in grid
// order, as compacted indices (p2c), and their count. One CTA per pair; each
// thread takes a run of up to kSeedRun consecutive seeds per pass, all of
// whose lookups are in flight together, and one block scan of the runs'
// counts places them.
constexpr int kSeedRun = 8;

__global__ void __launch_bounds__(1024) masked_seeds_kernel(const int32_t* __restrict__ p2c,
                                                            int64_t N1, int W1, int sub,
                                                            int64_t S, int32_t* __restrict__ F0,
                                                            int32_t* __restrict__ seed_cnt) {
  __shared__ int sm[32];
  const int b = blockIdx.x;
  const int gx = (W1 + sub - 1) / sub;
  const int64_t per_pass = static_cast<int64_t>(blockDim.x) * kSeedRun;
  const int64_t run = (min(S, per_pass) + blockDim.x - 1) / blockDim.x;  // seeds per thread
  int base = 0;
  for (int64_t s0 = 0; s0 < S; s0 += run * blockDim.x) {
    const int64_t k0 = s0 + threadIdx.x * run;
    int32_t pos[kSeedRun];
    int c = 0;
#pragma unroll
    for (int i = 0; i < kSeedRun; ++i) {
      const int64_t k = k0 + i;
      pos[i] = -1;
      if (i < run && k < S) {
        const int64_t u = (k / gx) * sub * static_cast<int64_t>(W1) + (k % gx) * sub;
        pos[i] = __ldg(p2c + b * N1 + u);
      }
    }
#pragma unroll
    for (int i = 0; i < kSeedRun; ++i) c += pos[i] >= 0 ? 1 : 0;
    int slot = base + block_exclusive_scan(c, sm);
#pragma unroll
    for (int i = 0; i < kSeedRun; ++i)
      if (pos[i] >= 0) F0[b * S + slot++] = pos[i];
    int total = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += sm[w];
    base += total;
    __syncthreads();  // sm is reused by the next pass
  }
  if (threadIdx.x == 0) seed_cnt[b] = base;
}

}  // namespace

int mask_blocks(int64_t N) { return static_cast<int>((N + 1023) / 1024); }

static int launch_mask_compact_impl(const MaskArgs& m0, int dtype, cudaStream_t st) {
  MaskArgs m = m0;
  m.bpp = mask_blocks(m.N);
  const int nb = m.batch * m.bpp;
  if (nb <= 0) return FASTNN_OK;
  mask_count_kernel<<<nb, 256, 0, st>>>(m);
  mutual_scan_kernel<<<m.batch, 1024, 0, st>>>(m.blocks, m.bpp, m.count);
  const int nbytes = m.d * elem_bytes(dtype);
  if (dtype != FASTNN_F32_L2 && nbytes % 8 == 0 && reinterpret_cast<uintptr_t>(m.src) % 16 == 0 &&
      (m.batch == 1 || (m.N * nbytes) % 16 == 0)) {
    const bool i8 = dtype == FASTNN_I8;
    int rc = FASTNN_OK;
    switch (row_bytes(dtype, m.d)) {
      case 32:
        rc = i8 ? launch_mask_emit_staged<32, true>(m, nb, nbytes, st)
                : launch_mask_emit_staged<32, false>(m, nb, nbytes, st);
        break;
      case 64:
        rc = i8 ? launch_mask_emit_staged<64, true>(m, nb, nbytes, st)
                : launch_mask_emit_staged<64, false>(m, nb, nbytes, st);
        break;
      case 128:
        rc = launch_mask_emit_staged<128, false>(m, nb, nbytes, st);
        break;
      default:
        return FASTNN_ERR_UNSUPPORTED;
    }
    if (rc != FASTNN_OK) return rc;
    FASTNN_CUDA_TRY(cudaGetLastError());
    return FASTNN_OK;
  }
  switch (dtype == FASTNN_F32_L2 ? 0 : row_bytes(dtype, m.d) * (dtype == FASTNN_I8 ? 1 : -1)) {
    case 0: mask_emit_kernel<1, 4, 16><<<nb, 1024, 0, st>>>(m); break;
    case 32: mask_emit_kernel<0, 1, 32><<<nb, 1024, 0, st>>>(m); break;
    case 64: mask_emit_kernel<0, 1, 64><<<nb, 1024, 0, st>>>(m); break;
    case -64: mask_emit_kernel<0, 2, 64><<<nb, 1024, 0, st>>>(m); break;
    case -128: mask_emit_kernel<0, 2, 128><<<nb, 1024, 0, st>>>(m); break;
    default: return FASTNN_ERR_UNSUPPORTED;
  }
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_mask_compact(const MaskArgs& m0, int dtype, cudaStream_t st) {
  const int slot = kernel_timer_begin(st, kTimeMask);
  if (slot == -2) return FASTNN_ERR_CUDA;
  const int rc = launch_mask_compact_impl(m0, dtype, st);
  if (rc != FASTNN_OK) return rc;
  return kernel_timer_end(slot, st);
}

int launch_masked_seeds(const int32_t* p2c, int batch, int64_t N1, int W1, int sub, int64_t S,
                        int32_t* F0, int32_t* seed_cnt, cudaStream_t st) {
  masked_seeds_kernel<<<batch, 1024, 0, st>>>(p2c, N1, W1, sub, S, F0, seed_cnt);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

static int launch_repack_impl(const void* src, int64_t rows, int d, int dtype, void* dst,
                              int64_t pad_rows, int* absmax, cudaStream_t st) {
  const int64_t total = rows + pad_rows;
  if (total <= 0) return FASTNN_OK;
  const uint8_t* s8 = static_cast<const uint8_t*>(src);
  uint8_t* d8 = static_cast<uint8_t*>(dst);
  const int g = grid_for(total, 256);
  if (dtype == FASTNN_F32_L2) {
    repack_l2_kernel<<<g, 256, 0, st>>>(static_cast<const float*>(src), rows, d,
                                        static_cast<float4*>(dst), pad_rows, absmax);
    FASTNN_CUDA_TRY(cudaGetLastError());
    return FASTNN_OK;
  }
  const int nbytes = d * elem_bytes(dtype);
  if (nbytes % 8 == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0) {
    // Staged stream copy; the grid covers the runs up to 148 SMs x 8 blocks.
    const int64_t runs = (total + kRepackRows - 1) / kRepackRows;
    const int gs = static_cast<int>(min(runs, static_cast<int64_t>(148 * 8)));
    int* am = dtype == FASTNN_I8 ? absmax : nullptr;
    switch (row_bytes(dtype, d)) {
      case 32:
        repack_staged_kernel<32><<<gs, kRepackThreads, 0, st>>>(s8, rows, nbytes, d8, pad_rows, am);
        break;
      case 64:
        repack_staged_kernel<64><<<gs, kRepackThreads, 0, st>>>(s8, rows, nbytes, d8, pad_rows, am);
        break;
      case 128:
        repack_staged_kernel<128><<<gs, kRepackThreads, 0, st>>>(s8, rows, nbytes, d8, pad_rows, am);
        break;
      default:
        return FASTNN_ERR_UNSUPPORTED;
    }
    FASTNN_CUDA_TRY(cudaGetLastError());
    return FASTNN_OK;
  }
  switch (row_bytes(dtype, d)) {
    case 32:
      repack_kernel<1, 32><<<g, 256, 0, st>>>(s8, rows, d, d8, pad_rows, absmax);
      break;
    case 64:
      if (dtype == FASTNN_I8)
        repack_kernel<1, 64><<<g, 256, 0, st>>>(s8, rows, d, d8, pad_rows, absmax);
      else
        repack_kernel<2, 64><<<g, 256, 0, st>>>(s8, rows, d, d8, pad_rows, nullptr);
      break;
    case 128:
      repack_kernel<2, 128><<<g, 256, 0, st>>>(s8, rows, d, d8, pad_rows, nullptr);
      break;
    default:
      return FASTNN_ERR_UNSUPPORTED;
  }
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_repack(const void* src, int64_t rows, int d, int dtype, void* dst, int64_t pad_rows,
                  int* absmax, cudaStream_t st) {
  const int slot = kernel_timer_begin(st, kTimeRepack);
  if (slot == -2) return FASTNN_ERR_CUDA;
  const int rc = launch_repack_impl(src, rows, d, dtype, dst, pad_rows, absmax, st);
  if (rc != FASTNN_OK) return rc;
  return kernel_timer_end(slot, st);
}

int mutual_blocks(int64_t n1) {
  return static_cast<int>((n1 + kMutBlockRows - 1) / kMutBlockRows);
}
int mutual_scratch_ints(int64_t n1) {
  const int nb = mutual_blocks(n1);
  return nb + nb * (kMutThreads / 4);  // block counts, then one keep byte per thread
}
int image_blocks(int64_t n1) { return static_cast<int>((n1 + 1023) / 1024); }

static int launch_mutual_impl(const MutualSrc& m, int32_t* block_scratch, int dtype,
                              int32_t* out_pairs, void* out_score, int64_t cap,
                              int32_t* out_count, cudaStream_t st) {
  const int nb = mutual_blocks(m.n1);
  uint8_t* keep = reinterpret_cast<uint8_t*>(block_scratch + nb);
  mutual_count_kernel<<<nb, kMutThreads, 0, st>>>(m, block_scratch, keep);
  mutual_scan_kernel<<<1, 1024, 0, st>>>(block_scratch, nb, out_count);
  if (dtype == FASTNN_I8) {
    FASTNN_CUDA_TRY(cudaFuncSetAttribute(mutual_emit_kernel<FASTNN_I8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMutEmitSmem));
    mutual_emit_kernel<FASTNN_I8><<<nb, kMutThreads, kMutEmitSmem, st>>>(
        m, block_scratch, keep, out_pairs, out_score, cap);
  } else if (dtype == FASTNN_F32_L2) {
    FASTNN_CUDA_TRY(cudaFuncSetAttribute(mutual_emit_kernel<FASTNN_F32_L2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMutEmitSmem));
    mutual_emit_kernel<FASTNN_F32_L2><<<nb, kMutThreads, kMutEmitSmem, st>>>(
        m, block_scratch, keep, out_pairs, out_score, cap);
  } else {
    FASTNN_CUDA_TRY(cudaFuncSetAttribute(mutual_emit_kernel<FASTNN_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMutEmitSmem));
    mutual_emit_kernel<FASTNN_BF16><<<nb, kMutThreads, kMutEmitSmem, st>>>(
        m, block_scratch, keep, out_pairs, out_score, cap);
  }
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_mutual(const MutualSrc& m, int32_t* block_scratch, int dtype, int32_t* out_pairs,
                  void* out_score, int64_t cap, int32_t* out_count, cudaStream_t st) {
  const int slot = kernel_timer_begin(st, kTimeMutual);
  if (slot == -2) return FASTNN_ERR_CUDA;
  const int rc =
      launch_mutual_impl(m, block_scratch, dtype, out_pairs, out_score, cap, out_count, st);
  if (rc != FASTNN_OK) return rc;
  return kernel_timer_end(slot, st);
}

int launch_chunk_boxes(const float4* rows, int64_t N, int batch, const int32_t* count,
                       float4* box, cudaStream_t st) {
  const int nchunk = static_cast<int>((N + kL2Chunk - 1) / kL2Chunk);
  if (batch < 1 || nchunk < 1) return FASTNN_OK;
  chunk_box_kernel<<<batch * nchunk, 256, 0, st>>>(rows, N, nchunk, count, box);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

static int launch_image_list_impl(const uint64_t* k12, int64_t n1, int64_t n2,
                                  uint32_t* first, uint32_t* best, int32_t* pos, int32_t* list,
                                  uint32_t* list_bound, int32_t* count, int32_t* block_scratch,
                                  cudaStream_t st) {
  const int nb = image_blocks(n1);
  image_mark_kernel<<<grid_for(n1, 256), 256, 0, st>>>(k12, n1, n2, first, best);
  image_count_kernel<<<nb, 1024, 0, st>>>(k12, first, n1, n2, block_scratch);
  mutual_scan_kernel<<<1, 1024, 0, st>>>(block_scratch, nb, count);
  image_emit_kernel<<<nb, 1024, 0, st>>>(k12, first, best, n1, n2, block_scratch, pos, list,
                                         list_bound);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_image_list(const uint64_t* k12, int64_t n1, int64_t n2, uint32_t* first,
                      uint32_t* best, int32_t* pos, int32_t* list, uint32_t* list_bound,
                      int32_t* count, int32_t* block_scratch, cudaStream_t st) {
  const int slot = kernel_timer_begin(st, kTimeMutual);
  if (slot == -2) return FASTNN_ERR_CUDA;
  const int rc = launch_image_list_impl(k12, n1, n2, first, best, pos, list, list_bound, count,
                                        block_scratch, st);
  if (rc != FASTNN_OK) return rc;
  return kernel_timer_end(slot, st);
}

int launch_image_rows(const int32_t* nn12, int64_t n1, int64_t n2, uint8_t* flag,
                      int32_t* block_scratch, int32_t* rows, int32_t* count, cudaStream_t st) {
  const int slot = kernel_timer_begin(st, kTimeMutual);
  if (slot == -2) return FASTNN_ERR_CUDA;
  const int nb = mutual_blocks(n2);
  FASTNN_CUDA_TRY(cudaMemsetAsync(flag, 0, static_cast<size_t>(n2), st));
  if (n1 > 0) image_flag_kernel<<<grid_for(n1, 256), 256, 0, st>>>(nn12, n1, n2, flag);
  image_rows_count_kernel<<<nb, kImgThreads, 0, st>>>(flag, n2, block_scratch);
  mutual_scan_kernel<<<1, 1024, 0, st>>>(block_scratch, nb, count);
  image_rows_emit_kernel<<<nb, kImgThreads, 0, st>>>(flag, n2, block_scratch, rows);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return kernel_timer_end(slot, st);
}

int launch_decode(const uint64_t* key, int64_t n, int dtype, int32_t* out_idx, void* out_score,
                  cudaStream_t st) {
  if (n <= 0) return FASTNN_OK;
  const int g = grid_for(n, 256);
  if (dtype == FASTNN_I8)
    decode_kernel<FASTNN_I8><<<g, 256, 0, st>>>(key, n, out_idx, out_score);
  else if (dtype == FASTNN_F32_L2)
    decode_kernel<FASTNN_F32_L2><<<g, 256, 0, st>>>(key, n, out_idx, out_score);
  else
    decode_kernel<FASTNN_BF16><<<g, 256, 0, st>>>(key, n, out_idx, out_score);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

}  // namespace fastnn
