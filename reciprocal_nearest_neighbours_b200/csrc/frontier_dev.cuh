// Device-side pieces of the fast scheme's frontier handling, shared by the
// persistent matching kernel (nn_tc.cu) and the dense-path kernels
// (frontier.cu). Everything other CTAs may have written during the same
// kernel is read with ld.global.cg (L2, never a stale L1 line).
#pragma once

#include "common.cuh"
#include "frontier.cuh"

namespace fastnn {

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

// Seeds of pair b: pixels (x, y) with x = sub * (k mod gx), y = sub * (k div gx)
// for k < S, written to the round-1 frontier; each seed claims its pixel with
// stamp 0 (round 0, slot k).
__device__ __forceinline__ void seed_one(int32_t* F0, int64_t S_cap, uint32_t* claim, int64_t N1,
                                         int W1, int sub, int b, int k) {
  const int gx = (W1 + sub - 1) / sub;
  const int y = (k / gx) * sub;
  const int x = (k % gx) * sub;
  const int u = y * W1 + x;
  F0[b * S_cap + k] = u;
  claim[b * N1 + u] = static_cast<uint32_t>(k);
}

// The round's frontier buffers (the rest of CompactArgs is fixed per call).
struct FrontierBufs {
  const int32_t* F_cur;
  int32_t* F_next;
  const int32_t* cnt_cur;
  int32_t* cnt_next;
};

// Round t (1-based) of the fast scheme for pair b, run by one whole CTA.
// Slot k holds pixel u = F[k] of image 1, its forward match v = NN(D1[u], D2)
// and the backward match u' = NN(D2[v], D1). u' == u keeps (u, v); otherwise
// u' is pushed to the next frontier if no frontier of this call has held it
// yet: phase 1 claims u' with atomicMin on a (round, slot) stamp, phase 2 lets
// only the claiming slot push, so duplicates within the round and pixels seen
// in earlier rounds are dropped, deterministically. Kept pairs and pushes are
// compacted in slot order. The round's key slots are reset to 0 for the next
// round's atomicMax merges. `sm` holds 66 ints.
template <int DT>
__device__ void compact_pair(const CompactArgs& c, const FrontierBufs& fb, int b, int t,
                             bool last_round, int* sm) {
  // Each thread handles up to kPer slots per batch, all of whose loads are
  // issued together, so a round costs a few L2 round trips instead of a few
  // per block-sized chunk.
  constexpr int kPer = 8;
  const int cnt = __ldcg(fb.cnt_cur + b);
  if (cnt == 0) {
    if (threadIdx.x == 0) fb.cnt_next[b] = 0;
    return;
  }
  const int32_t* F = fb.F_cur + b * c.S_cap;
  uint64_t* fwd = c.fwd_key + b * c.S_cap;
  uint64_t* bwd = c.bwd_key + b * c.S_cap;
  uint32_t* claim = c.claim + b * c.N1;
  const uint32_t stamp_hi = static_cast<uint32_t>(t) << 24;
  const int step = blockDim.x * kPer;

  // Phase 1: claim every pushed pixel with the smallest (round, slot) stamp.
  if (!last_round) {
    for (int base = 0; base < cnt; base += step) {
      uint32_t u[kPer], u2[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int k = base + threadIdx.x + i * blockDim.x;
        u[i] = k < cnt ? static_cast<uint32_t>(__ldcg(F + k)) : 0u;
        u2[i] = k < cnt ? key_index(__ldcg(bwd + k)) : 0u;
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int k = base + threadIdx.x + i * blockDim.x;
        if (k < cnt && u2[i] != u[i] && u2[i] < static_cast<uint32_t>(c.N1))
          atomicMin(&claim[u2[i]], stamp_hi | static_cast<uint32_t>(k));
      }
    }
  }
  if (threadIdx.x == 0) sm[64] = __ldcg(c.out_count + b);
  __syncthreads();

  // Phase 2: kept pairs and pushes, compacted in slot order.
  int out0 = sm[64], next0 = 0;
  for (int base = 0; base < cnt; base += step) {
    uint32_t u[kPer], u2[kPer], cl[kPer];
    uint64_t fk[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int k = base + threadIdx.x + i * blockDim.x;
      const bool in = k < cnt;
      u[i] = in ? static_cast<uint32_t>(__ldcg(F + k)) : 0u;
      fk[i] = in ? __ldcg(fwd + k) : 0ull;
      u2[i] = in ? key_index(__ldcg(bwd + k)) : 0u;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int k = base + threadIdx.x + i * blockDim.x;
      cl[i] = (k < cnt && !last_round && u2[i] != u[i] && u2[i] < static_cast<uint32_t>(c.N1))
                  ? __ldcg(claim + u2[i])
                  : 0xFFFFFFFFu;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int k = base + threadIdx.x + i * blockDim.x;
      if (base + i * blockDim.x >= cnt) break;  // uniform over the block
      const bool in = k < cnt;
      const bool conv = in && u2[i] == u[i];
      const bool push = in && !conv && cl[i] == (stamp_hi | static_cast<uint32_t>(k));
      if (in) {
        fwd[k] = 0;
        bwd[k] = 0;
      }
      const Scan2 sc = block_scan2(conv, push, sm);
      if (conv) {
        const int64_t pos = out0 + sc.ex0;
        if (pos < c.cap) {
          int32_t* op = c.out_pairs + (b * c.cap + pos) * 2;
          op[0] = static_cast<int32_t>(u[i]);
          op[1] = static_cast<int32_t>(key_index(fk[i]));
          if (c.out_score) {
            if (DT == FASTNN_I8)
              static_cast<int32_t*>(c.out_score)[b * c.cap + pos] =
                  unord_i32(key_score_bits(fk[i]));
            else
              static_cast<float*>(c.out_score)[b * c.cap + pos] = unord_f32(key_score_bits(fk[i]));
          }
        }
      }
      if (push) fb.F_next[b * c.S_cap + next0 + sc.ex1] = static_cast<int32_t>(u2[i]);
      out0 += sc.tot0;
      next0 += sc.tot1;
    }
  }
  if (threadIdx.x == 0) {
    c.out_count[b] = out0;
    fb.cnt_next[b] = next0;
    if (c.out_iters) c.out_iters[b] = t;
    if (c.out_frontier) c.out_frontier[b * c.max_iter + (t - 1)] = cnt;
  }
  __syncthreads();
}

}  // namespace fastnn
