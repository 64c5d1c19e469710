// Device-side pieces of the fast scheme's frontier handling, shared by the
// persistent matching kernel (nn_tc.cu) and the dense-path kernels
// (frontier.cu). Everything other CTAs may have written during the same
// kernel is read with ld.global.cg (L2, never a stale L1 line).
#pragma once

#include "common.cuh"
#include "frontier.cuh"
#include "ptx.cuh"

namespace fastnn {

// Grid-wide barrier over the co-resident CTAs of a cooperative launch: a
// monotonic arrival counter (zero before the launch); each CTA waits, bounded
// by limit_ns, until the counter reaches its next multiple of the grid size.
// Thread 0 arrives with a release add and leaves with an acquire load of the
// counter, so the CTA's writes before the barrier are visible to every CTA
// after it, without separate fences. A CTA that arrives with cta_ok == false,
// or whose wait runs out, sets the counter's top bit (and the shared abort
// word, for the record): every waiter leaves at once and the barrier fails
// for all of them. `flag` is a shared int that carries thread 0's verdict to
// the CTA. Returns the CTA-uniform verdict.
constexpr uint32_t kBarrierAbortBit = 0x80000000u;

__device__ __forceinline__ bool grid_barrier(uint32_t* count, int* abort_word, int* status,
                                             uint32_t& target, bool cta_ok, int* flag,
                                             uint64_t limit_ns) {
  __syncthreads();
  if (threadIdx.x == 0) {
    target += gridDim.x;
    bool ok = cta_ok;
    if (!ok) {
      atomicExch(abort_word, 1);
      atomicOr(count, kBarrierAbortBit);
    }
    ptx::red_add_release_gpu(count, 1u);
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
      const uint32_t c = ptx::ld_relaxed_gpu(count);
      if ((c & kBarrierAbortBit) || c >= target) break;
      if ((n & 63) == 0 && ptx::globaltimer_ns() - t0 > limit_ns) {
        atomicOr(status, kStatusTimeout);
        atomicExch(abort_word, 1);
        atomicOr(count, kBarrierAbortBit);
        break;
      }
    }
    if (ptx::ld_acquire_gpu(count) & kBarrierAbortBit) ok = false;
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *reinterpret_cast<volatile int*>(flag) != 0;
}

// Block-wide exclusive scan of two 0/1 flags (warp ballots + one smem pass).
// Returns the exclusive prefix of each flag and the block totals. `sm` holds
// 64 ints; every thread of the block must call it.
struct Scan2 {
  int ex0, ex1, tot0, tot1;
};

__device__ __forceinline__ Scan2 block_scan2(bool f0, bool f1, int* sm) {
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

// Block-wide exclusive scan of two small per-thread counts (each block total
// below 2^16), packed in one word: a warp shuffle scan, then one pass over
// the warp totals. `sm` holds 32 ints; every thread of the block must call it.
__device__ __forceinline__ Scan2 block_scan_counts(int c0, int c1, int* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int x = c0 | (c1 << 16);
  int inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sm[warp] = inc;
  __syncthreads();
  int off = 0, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const int cw = sm[w];
    if (w < warp) off += cw;
    tot += cw;
  }
  __syncthreads();
  const int ex = off + inc - x;
  return Scan2{ex & 0xFFFF, ex >> 16, tot & 0xFFFF, tot >> 16};
}

// Repack inside a persistent kernel: rows [rows][nbytes] (nbytes a multiple
// of 8, 8-byte aligned source) into RB-byte rows zero-padded, plus pad_rows
// zero rows; one 16-byte output chunk per thread and step of a grid-stride
// loop (two 8-byte loads), so a warp's loads and stores cover consecutive
// bytes. absmax (int8, optional) receives max |element| by atomicMax. The
// stores are then ordered before the async proxy (the tensor-map loads that
// read the rows after the next grid barrier).
__device__ __forceinline__ void repack_in_kernel(const uint8_t* __restrict__ src, int64_t rows,
                                                 int nbytes, int RB, uint8_t* __restrict__ dst,
                                                 int64_t pad_rows, int* absmax, int64_t gtid,
                                                 int64_t gsize) {
  const int cpr = RB / 16;  // output chunks per row
  const int64_t total = (rows + pad_rows) * cpr;
  uint32_t amax = 0;
  for (int64_t k = gtid; k < total; k += gsize) {
    const int64_t row = k / cpr;
    const int off = 16 * static_cast<int>(k - row * cpr);
    uint2 lo = make_uint2(0, 0), hi = make_uint2(0, 0);
    if (row < rows) {
      const uint8_t* sr = src + row * nbytes;
      if (off < nbytes) lo = __ldg(reinterpret_cast<const uint2*>(sr + off));
      if (off + 8 < nbytes) hi = __ldg(reinterpret_cast<const uint2*>(sr + off + 8));
      if (absmax)
        amax = __vmaxu4(__vmaxu4(amax, __vabs4(lo.x)),
                        __vmaxu4(__vmaxu4(__vabs4(lo.y), __vabs4(hi.x)), __vabs4(hi.y)));
    }
    reinterpret_cast<uint4*>(dst + row * RB)[off / 16] = make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
  if (absmax) {
    int m = static_cast<int>(max(max(amax & 0xFFu, (amax >> 8) & 0xFFu),
                                 max((amax >> 16) & 0xFFu, amax >> 24)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0) atomicMax(absmax, m);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// The round's frontier buffers (the rest of CompactArgs is fixed per call).
struct FrontierBufs {
  const int32_t* F_cur;
  int32_t* F_next;
  const int32_t* cnt_cur;
  int32_t* cnt_next;
  uint32_t* B_next;  // score bound of each pushed pixel (see fast_rounds)
};

// Slots per thread and pass of the per-pair compaction: each thread loads
// its run of kCE consecutive slots at once, so that one pass costs a few
// dependent L2 round trips rather than a few per slot.
constexpr int kCE = 6;

// Round t (1-based) of the fast scheme for pair b, run by one whole CTA.
// Slot k holds pixel u = F[k] of image 1, its forward match v = NN(D1[u], D2)
// and the backward match u' = NN(D2[v], D1). u' == u keeps (u, v); otherwise
// u' is pushed to the next frontier if no frontier of this call has held it
// yet: every slot claims its u' with atomicMin on a (round, slot) stamp and
// only the claiming slot pushes, so duplicates within the round and pixels
// seen in earlier rounds are dropped, deterministically. A pass checks a
// slot's claim once the claims of that pass and of all earlier passes have
// landed: a later slot's stamp is larger and cannot undercut it. Kept pairs
// and pushes are compacted in slot order. The round's key slots are reset to
// 0 for the next round's atomicMax merges. `cnt` is the pair's frontier
// count (the planner's cached copy); `sm` holds 66 ints.
template <int DT>
__device__ void compact_pair(const CompactArgs& c, const FrontierBufs& fb, int b, int t,
                             bool last_round, int* sm, int cnt) {
  if (cnt == 0) {
    if (threadIdx.x == 0) fb.cnt_next[b] = 0;
    return;
  }
  const int32_t* F = fb.F_cur + b * c.S_cap;
  uint64_t* fwd = c.fwd_key + b * c.S_cap;
  uint64_t* bwd = c.bwd_key + b * c.S_cap;
  uint32_t* claim = c.claim + b * c.N1;
  const uint32_t stamp_hi = static_cast<uint32_t>(t) << 24;
  const uint32_t N1 = static_cast<uint32_t>(c.N1), N2 = static_cast<uint32_t>(c.N2);

  // Every thread reads the output count itself: the load overlaps the first
  // pass's loads instead of costing a round trip and a barrier of its own.
  int out0 = __ldcg(c.out_count + b), next0 = 0;
  const int per_pass = static_cast<int>(blockDim.x) * kCE;
  for (int s = 0; s < cnt; s += per_pass) {
    const int k0 = s + static_cast<int>(threadIdx.x) * kCE;
    uint32_t u[kCE], u2[kCE], s2[kCE];
    uint64_t fk[kCE];
#pragma unroll
    for (int j = 0; j < kCE; ++j) {
      const bool in = k0 + j < cnt;
      u[j] = in ? static_cast<uint32_t>(__ldcg(F + k0 + j)) : 0u;
      fk[j] = in ? __ldcg(fwd + k0 + j) : 0ull;
      const uint64_t bk = in ? __ldcg(bwd + k0 + j) : 0ull;
      u2[j] = key_index(bk);
      s2[j] = key_score_bits(bk);
    }
    if (!last_round) {
#pragma unroll
      for (int j = 0; j < kCE; ++j)
        if (k0 + j < cnt && u2[j] != u[j] && u2[j] < N1)
          atomicMin(&claim[u2[j]], stamp_hi | static_cast<uint32_t>(k0 + j));
      __syncthreads();
    }
    unsigned conv_m = 0, push_m = 0;
#pragma unroll
    for (int j = 0; j < kCE; ++j) {
      const int k = k0 + j;
      if (k < cnt) {
        // A forward pass that found no candidate leaves v = 0xFFFFFFFF: the
        // walk ends there.
        const uint32_t v = key_index(fk[j]);
        if (u2[j] == u[j] && v < N2) {
          conv_m |= 1u << j;
        } else if (!last_round && v < N2 && u2[j] < N1 &&
                   __ldcg(claim + u2[j]) == (stamp_hi | static_cast<uint32_t>(k))) {
          push_m |= 1u << j;
        }
        fwd[k] = 0;
        bwd[k] = 0;
      }
    }
    const Scan2 sc = block_scan_counts(__popc(conv_m), __popc(push_m), sm);
    int pos = out0 + sc.ex0, nxt = next0 + sc.ex1;
#pragma unroll
    for (int j = 0; j < kCE; ++j) {
      if ((conv_m >> j) & 1u) {
        if (pos < c.cap) {
          const uint32_t v = key_index(fk[j]);
          int32_t* op = c.out_pairs + (b * c.cap + pos) * 2;
          op[0] = c.map1 ? c.map1[b * c.N1 + u[j]] : static_cast<int32_t>(u[j]);
          op[1] = c.map2 ? c.map2[b * c.N2 + v] : static_cast<int32_t>(v);
          if (c.out_score) {
            if (DT == FASTNN_I8)
              static_cast<int32_t*>(c.out_score)[b * c.cap + pos] = unord_i32(key_score_bits(fk[j]));
            else if (DT == FASTNN_F32_L2)
              static_cast<float*>(c.out_score)[b * c.cap + pos] = -unord_f32(key_score_bits(fk[j]));
            else
              static_cast<float*>(c.out_score)[b * c.cap + pos] = unord_f32(key_score_bits(fk[j]));
          }
        }
        ++pos;
      }
      if ((push_m >> j) & 1u) {
        fb.F_next[b * c.S_cap + nxt] = static_cast<int32_t>(u2[j]);
        fb.B_next[b * c.S_cap + nxt] = s2[j];
        ++nxt;
      }
    }
    out0 += sc.tot0;
    next0 += sc.tot1;
  }
  if (threadIdx.x == 0) {
    c.out_count[b] = out0;
    fb.cnt_next[b] = next0;
    if (c.out_iters) c.out_iters[b] = t;
    if (c.out_frontier) c.out_frontier[b * c.max_iter + (t - 1)] = cnt;
  }
  __syncthreads();
}

// The fast scheme's round loop, shared by the persistent matching kernels:
// clear the per-call state, seed the grid, then per round a forward pass
// (image 1 -> 2), a backward pass (matches -> image 1) and the per-pair
// check/compaction, separated by grid barriers; stops when every pair's
// frontier is empty or after max_iter rounds. `nn(dir, q)` runs one
// nearest-neighbour pass over the whole grid (dir 0: r.fwd, 1: r.bwd) and
// ends with a CTA barrier. `cta_abort` is the CTA's own abort flag (shared
// memory); `flag` and `scan` (66 ints) are shared scratch, and
// `cnt_cache` (one int per pair) the planner's count cache: the backward pass
// plans from the forward pass's counts, and each later forward pass from the
// counts the check after the compaction read.
// `prologue()` runs in every CTA beside the clearing of the per-call state,
// before the first grid barrier.
template <int DT, class NNPass, class Prologue>
__device__ void fast_rounds(const RecArgs& r, NNPass&& nn, Prologue&& prologue,
                            volatile int* cta_abort, int* flag, int* scan, int* cnt_cache) {
  uint32_t target = 0;
  const int batch = r.batch;
  const int64_t S = r.S;
  const int64_t gtid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t gsize = static_cast<int64_t>(gridDim.x) * blockDim.x;
  auto sync = [&]() {
    return grid_barrier(r.grid_count, r.grid_abort, r.status, target, !*cta_abort, flag,
                        wait_limit(r.fwd.wait_ns));
  };

  // Clear per-call state: keys, first-visit claims, outputs.
  for (int64_t i = gtid; i < batch * S; i += gsize) {
    r.cmp.fwd_key[i] = 0;
    r.cmp.bwd_key[i] = 0;
  }
  if (r.seed_cnt) {
    for (int64_t i = gtid; i < batch * r.N1; i += gsize) r.cmp.claim[i] = 0xFFFFFFFFu;
  } else {
    // Unmasked: the grid seeds are known, so the clearing pass writes each
    // seed pixel's stamp (round 0, slot k) directly, with the round-1
    // frontier, and seeding needs no pass (nor barrier) of its own.
    const int gx = (r.W1 + r.sub - 1) / r.sub;
    for (int64_t i = gtid; i < batch * r.N1; i += gsize) {
      const int u = static_cast<int>(i % r.N1);
      const int y = u / r.W1, x = u % r.W1;
      r.cmp.claim[i] = (x % r.sub == 0 && y % r.sub == 0)
                           ? static_cast<uint32_t>((y / r.sub) * gx + x / r.sub)
                           : 0xFFFFFFFFu;
    }
    for (int64_t i = gtid; i < batch * S; i += gsize) {
      const int k = static_cast<int>(i % S);
      r.F[0][i] = (k / gx) * r.sub * r.W1 + (k % gx) * r.sub;
    }
    for (int64_t i = gtid; i < batch; i += gsize) r.cnt[0][i] = static_cast<int>(S);
  }
  for (int64_t i = gtid; i < batch; i += gsize) {
    r.cmp.out_count[i] = 0;
    if (r.cmp.out_iters) r.cmp.out_iters[i] = 0;
  }
  if (r.cmp.out_frontier)
    for (int64_t i = gtid; i < batch * r.max_iter; i += gsize) r.cmp.out_frontier[i] = 0;
  prologue();
  bool ok = sync();
  if (ok && r.seed_cnt) {
    // Masked: the kept grid pixels are already in F[0]; each claims its pixel
    // with stamp (round 0, slot k) once the claims are cleared.
    for (int64_t i = gtid; i < batch * S; i += gsize) {
      const int b = static_cast<int>(i / S), k = static_cast<int>(i % S);
      if (k < __ldcg(r.seed_cnt + b))
        r.cmp.claim[b * r.N1 + __ldcg(r.F[0] + i)] = static_cast<uint32_t>(k);
    }
    for (int64_t i = gtid; i < batch; i += gsize) r.cnt[0][i] = __ldcg(r.seed_cnt + i);
    ok = sync();
  }
  for (int t = 1; ok && t <= r.max_iter; ++t) {
    const int cur = (t - 1) & 1, nxt = t & 1;
    // Score bounds: a pushed pixel u' reaches at least its backward score
    // <D2[v], D1[u']> in the forward pass, and a match v reaches at least its
    // forward score <D1[u], D2[v]> in the backward pass (the same dot
    // product). The seeds of round 1 have none.
    nn(0, PhaseQ{r.F[cur], r.cnt[cur], t > 1 ? r.Bd[cur] : nullptr, 1, t > 1 ? 1 : 0});
    if (!sync()) break;
    nn(1, PhaseQ{nullptr, r.cnt[cur], reinterpret_cast<const uint32_t*>(r.cmp.fwd_key) + 1, 2, 1});
    if (!sync()) break;
    const FrontierBufs fb{r.F[cur], r.F[nxt], r.cnt[cur], r.cnt[nxt], r.Bd[nxt]};
    for (int b = blockIdx.x; b < batch; b += gridDim.x)
      compact_pair<DT>(r.cmp, fb, b, t, t == r.max_iter, scan, cnt_cache[b]);
    if (!sync()) break;
    // Every CTA reads the same counts after the barrier: a uniform exit. The
    // pairs' counts are read by as many threads, all loads in flight at once.
    int any = 0;
    for (int b = threadIdx.x; b < batch; b += blockDim.x) {
      const int c = __ldcg(r.cnt[nxt] + b);
      cnt_cache[b] = c;
      any |= c;
    }
    if (!__syncthreads_or(any != 0)) break;
  }
}

}  // namespace fastnn
