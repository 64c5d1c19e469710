// Memory-bound kernels around the nearest-neighbour passes:
//   repack          descriptor rows [rows][d] -> zero-padded [rows][32 elems]
//   seed_grid       sparse seed grid of image 1 -> round-1 frontier
//   check_compact   reciprocal test of one round + next-frontier compaction
//   mutual_*        dense mutual-pair test and ordered emission
//   decode_nn       packed keys -> (index, score)
#include "common.cuh"
#include "frontier.cuh"

namespace fastnn {

namespace {

// ---------------------------------------------------------------- repack ---
// One thread per output row. Source rows of d elements (esize bytes each) are
// copied into 32-element rows (32 B int8 / 64 B bf16) with zero padding, so
// every row is 16-byte aligned for TMA and the MMA's K extent is exactly 32.
// For int8 maps, `absmax` (if given) receives max |element| over the map
// (atomicMax), which tells the nearest-neighbour kernel whether every score
// fits in 16 bits.
template <int ESIZE>
__global__ void repack_kernel(const uint8_t* __restrict__ src, int64_t rows, int d,
                              uint8_t* __restrict__ dst, int64_t pad_rows, int* absmax) {
  constexpr int RB = 32 * ESIZE;
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

// ------------------------------------------------------------- seed grid ---
// Seeds of pair b: pixels (x, y) with x = sub * (k mod gx), y = sub * (k div gx).
// Each seed claims its pixel with stamp 0 (round 0, slot k).
__global__ void seed_kernel(int32_t* __restrict__ F0, int64_t S_cap, uint32_t* __restrict__ claim,
                            int64_t N1, int32_t* __restrict__ cnt0, int H1, int W1, int sub,
                            int S) {
  const int b = blockIdx.y;
  const int gx = (W1 + sub - 1) / sub;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < S; k += gridDim.x * blockDim.x) {
    const int y = (k / gx) * sub;
    const int x = (k % gx) * sub;
    const int u = y * W1 + x;
    F0[b * S_cap + k] = u;
    claim[b * N1 + u] = static_cast<uint32_t>(k);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) cnt0[b] = S;
}

// Block-wide exclusive scan of two 0/1 flags (warp ballots + one smem pass).
// Returns the exclusive prefix of each flag and writes the block totals.
struct Scan2 {
  int ex0, ex1, tot0, tot1;
};

__device__ __forceinline__ Scan2 block_scan2(bool f0, bool f1, int* sm /* 2 * 32 ints */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned b0 = __ballot_sync(0xffffffffu, f0);
  const unsigned b1 = __ballot_sync(0xffffffffu, f1);
  const unsigned lt = (1u << lane) - 1u;
  if (lane == 0) {
    sm[warp] = __popc(b0);
    sm[32 + warp] = __popc(b1);
  }
  __syncthreads();
  int off0 = 0, off1 = 0, t0 = 0, t1 = 0;
  for (int w = 0; w < nw; ++w) {
    const int c0 = sm[w], c1 = sm[32 + w];
    if (w < warp) {
      off0 += c0;
      off1 += c1;
    }
    t0 += c0;
    t1 += c1;
  }
  __syncthreads();
  return Scan2{off0 + __popc(b0 & lt), off1 + __popc(b1 & lt), t0, t1};
}

// --------------------------------------------------------- check+compact ---
// One CTA per pair. Round t (1-based) of the fast scheme: slot k holds seed
// u = F[k], its forward match v and the backward match u'. u' == u keeps
// (u, v); otherwise u' is pushed to the next frontier if no frontier of this
// call has held it yet: phase 1 claims u' with atomicMin on a (round, slot)
// stamp, phase 2 lets only the claiming slot push, so duplicates within the
// round and pixels seen in earlier rounds are dropped, deterministically.
// Kept pairs and pushes are compacted in slot order. The round's key slots
// are reset to 0 for the next round's atomicMax merges.
template <int DT>
__global__ void __launch_bounds__(1024) check_compact_kernel(CompactArgs c, int t, int last_round) {
  __shared__ int sm[64];
  __shared__ int base_out;
  const int b = blockIdx.x;
  const int cnt = c.cnt_cur[b];
  if (cnt == 0) {
    if (threadIdx.x == 0) c.cnt_next[b] = 0;
    return;
  }
  const int32_t* F = c.F_cur + b * c.S_cap;
  uint64_t* fwd = c.fwd_key + b * c.S_cap;
  uint64_t* bwd = c.bwd_key + b * c.S_cap;
  uint32_t* claim = c.claim + b * c.N1;
  const uint32_t stamp_hi = static_cast<uint32_t>(t) << 24;

  if (!last_round) {
    for (int k = threadIdx.x; k < cnt; k += blockDim.x) {
      const uint32_t u2 = key_index(bwd[k]);
      if (u2 != static_cast<uint32_t>(F[k]) && u2 < static_cast<uint32_t>(c.N1))
        atomicMin(&claim[u2], stamp_hi | static_cast<uint32_t>(k));
    }
  }
  if (threadIdx.x == 0) base_out = c.out_count[b];
  __syncthreads();
  int out0 = base_out, next0 = 0;
  for (int s = 0; s < cnt; s += blockDim.x) {
    const int k = s + threadIdx.x;
    bool conv = false, push = false;
    uint32_t u = 0, v = 0, u2 = 0;
    uint64_t fk = 0;
    if (k < cnt) {
      u = static_cast<uint32_t>(F[k]);
      fk = fwd[k];
      v = key_index(fk);
      u2 = key_index(bwd[k]);
      conv = (u2 == u);
      push = !conv && !last_round && u2 < static_cast<uint32_t>(c.N1) &&
             claim[u2] == (stamp_hi | static_cast<uint32_t>(k));
      fwd[k] = 0;
      bwd[k] = 0;
    }
    const Scan2 sc = block_scan2(conv, push, sm);
    if (conv) {
      const int64_t pos = out0 + sc.ex0;
      if (pos < c.cap) {
        int32_t* op = c.out_pairs + (b * c.cap + pos) * 2;
        op[0] = static_cast<int32_t>(u);
        op[1] = static_cast<int32_t>(v);
        if (c.out_score) {
          if (DT == FASTNN_I8)
            static_cast<int32_t*>(c.out_score)[b * c.cap + pos] = unord_i32(key_score_bits(fk));
          else
            static_cast<float*>(c.out_score)[b * c.cap + pos] = unord_f32(key_score_bits(fk));
        }
      }
    }
    if (push) c.F_next[b * c.S_cap + next0 + sc.ex1] = static_cast<int32_t>(u2);
    out0 += sc.tot0;
    next0 += sc.tot1;
  }
  if (threadIdx.x == 0) {
    c.out_count[b] = out0;
    c.cnt_next[b] = next0;
    if (c.out_iters) c.out_iters[b] = t;
    if (c.out_frontier) c.out_frontier[b * c.max_iter + (t - 1)] = cnt;
  }
}

// ---------------------------------------------------------- dense mutual ---
// flag(i) = NN21(NN12(i)) == i. Three passes keep the output in ascending i
// without inter-CTA waiting: per-block counts, one scan block, ordered emit.
__device__ __forceinline__ bool mutual_flag(const uint64_t* k12, const uint64_t* k21, int64_t n1,
                                            int64_t n2, int64_t i, uint32_t& j) {
  if (i >= n1) return false;
  j = key_index(k12[i]);
  if (j >= static_cast<uint64_t>(n2)) return false;
  return key_index(k21[j]) == static_cast<uint32_t>(i);
}

__global__ void __launch_bounds__(1024) mutual_count_kernel(const uint64_t* __restrict__ k12,
                                                            const uint64_t* __restrict__ k21,
                                                            int64_t n1, int64_t n2,
                                                            int32_t* __restrict__ block_cnt) {
  __shared__ int sm[64];
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t j;
  const bool f = mutual_flag(k12, k21, n1, n2, i, j);
  const Scan2 sc = block_scan2(f, false, sm);
  if (threadIdx.x == 0) block_cnt[blockIdx.x] = sc.tot0;
}

__global__ void __launch_bounds__(1024) mutual_scan_kernel(int32_t* __restrict__ block_cnt,
                                                           int nblocks,
                                                           int32_t* __restrict__ out_count) {
  __shared__ int sm[64];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int s = 0; s < nblocks; s += blockDim.x) {
    const int k = s + threadIdx.x;
    const int v = k < nblocks ? block_cnt[k] : 0;
    // exclusive scan of counts via per-thread value: warp shuffles + smem
    int x = v;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    int woff = 0, tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      if (w < warp) woff += sm[w];
      tot += sm[w];
    }
    const int c0 = carry;
    if (k < nblocks) block_cnt[k] = c0 + woff + x - v;
    __syncthreads();
    if (threadIdx.x == 0) carry = c0 + tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) *out_count = carry;
}

template <int DT>
__global__ void __launch_bounds__(1024) mutual_emit_kernel(const uint64_t* __restrict__ k12,
                                                           const uint64_t* __restrict__ k21,
                                                           int64_t n1, int64_t n2,
                                                           const int32_t* __restrict__ block_off,
                                                           int32_t* __restrict__ out_pairs,
                                                           void* __restrict__ out_score,
                                                           int64_t cap) {
  __shared__ int sm[64];
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t j = 0;
  const bool f = mutual_flag(k12, k21, n1, n2, i, j);
  const Scan2 sc = block_scan2(f, false, sm);
  if (f) {
    const int64_t pos = block_off[blockIdx.x] + sc.ex0;
    if (pos < cap) {
      out_pairs[pos * 2] = static_cast<int32_t>(i);
      out_pairs[pos * 2 + 1] = static_cast<int32_t>(j);
      if (out_score) {
        const uint32_t h = key_score_bits(k12[i]);
        if (DT == FASTNN_I8)
          static_cast<int32_t*>(out_score)[pos] = unord_i32(h);
        else
          static_cast<float*>(out_score)[pos] = unord_f32(h);
      }
    }
  }
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
      else
        static_cast<float*>(out_score)[i] = unord_f32(key_score_bits(k));
    }
  }
}

int grid_for(int64_t n, int threads, int max_blocks = 148 * 16) {
  int64_t g = (n + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > max_blocks) g = max_blocks;
  return static_cast<int>(g);
}

}  // namespace

int launch_repack(const void* src, int64_t rows, int d, int dtype, void* dst, int64_t pad_rows,
                  int* absmax, cudaStream_t st) {
  const int64_t total = rows + pad_rows;
  if (total <= 0) return FASTNN_OK;
  if (dtype == FASTNN_I8)
    repack_kernel<1><<<grid_for(total, 256), 256, 0, st>>>(static_cast<const uint8_t*>(src), rows,
                                                            d, static_cast<uint8_t*>(dst), pad_rows, absmax);
  else
    repack_kernel<2><<<grid_for(total, 256), 256, 0, st>>>(static_cast<const uint8_t*>(src), rows,
                                                            d, static_cast<uint8_t*>(dst), pad_rows,
                                                            nullptr);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_seed(int32_t* F0, int64_t S_cap, uint32_t* claim, int64_t N1, int32_t* cnt0, int H1,
                int W1, int sub, int S, int batch, cudaStream_t st) {
  dim3 grid(grid_for(S, 256, 64), batch);
  seed_kernel<<<grid, 256, 0, st>>>(F0, S_cap, claim, N1, cnt0, H1, W1, sub, S);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_check_compact(const CompactArgs& c, int dtype, int t, bool last_round, int batch,
                         cudaStream_t st) {
  if (dtype == FASTNN_I8)
    check_compact_kernel<FASTNN_I8><<<batch, 1024, 0, st>>>(c, t, last_round ? 1 : 0);
  else
    check_compact_kernel<FASTNN_BF16><<<batch, 1024, 0, st>>>(c, t, last_round ? 1 : 0);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int mutual_blocks(int64_t n1) { return static_cast<int>((n1 + 1023) / 1024); }

int launch_mutual(const uint64_t* k12, const uint64_t* k21, int64_t n1, int64_t n2,
                  int32_t* block_scratch, int dtype, int32_t* out_pairs, void* out_score,
                  int64_t cap, int32_t* out_count, cudaStream_t st) {
  const int nb = mutual_blocks(n1);
  mutual_count_kernel<<<nb, 1024, 0, st>>>(k12, k21, n1, n2, block_scratch);
  mutual_scan_kernel<<<1, 1024, 0, st>>>(block_scratch, nb, out_count);
  if (dtype == FASTNN_I8)
    mutual_emit_kernel<FASTNN_I8><<<nb, 1024, 0, st>>>(k12, k21, n1, n2, block_scratch, out_pairs,
                                                       out_score, cap);
  else
    mutual_emit_kernel<FASTNN_BF16><<<nb, 1024, 0, st>>>(k12, k21, n1, n2, block_scratch,
                                                         out_pairs, out_score, cap);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

int launch_decode(const uint64_t* key, int64_t n, int dtype, int32_t* out_idx, void* out_score,
                  cudaStream_t st) {
  if (n <= 0) return FASTNN_OK;
  if (dtype == FASTNN_I8)
    decode_kernel<FASTNN_I8><<<grid_for(n, 256), 256, 0, st>>>(key, n, out_idx, out_score);
  else
    decode_kernel<FASTNN_BF16><<<grid_for(n, 256), 256, 0, st>>>(key, n, out_idx, out_score);
  FASTNN_CUDA_TRY(cudaGetLastError());
  return FASTNN_OK;
}

}  // namespace fastnn
