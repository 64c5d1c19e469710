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

  if (!last_round) {
    for (int k = threadIdx.x; k < cnt; k += blockDim.x) {
      const uint32_t u2 = key_index(__ldcg(bwd + k));
      if (u2 != static_cast<uint32_t>(__ldcg(F + k)) && u2 < static_cast<uint32_t>(c.N1))
        atomicMin(&claim[u2], stamp_hi | static_cast<uint32_t>(k));
    }
  }
  if (threadIdx.x == 0) sm[64] = __ldcg(c.out_count + b);
  __syncthreads();
  int out0 = sm[64], next0 = 0;
  for (int s = 0; s < cnt; s += blockDim.x) {
    const int k = s + threadIdx.x;
    bool conv = false, push = false;
    uint32_t u = 0, v = 0, u2 = 0;
    uint64_t fk = 0;
    if (k < cnt) {
      u = static_cast<uint32_t>(__ldcg(F + k));
      fk = __ldcg(fwd + k);
      v = key_index(fk);
      u2 = key_index(__ldcg(bwd + k));
      conv = (u2 == u);
      push = !conv && !last_round && u2 < static_cast<uint32_t>(c.N1) &&
             __ldcg(claim + u2) == (stamp_hi | static_cast<uint32_t>(k));
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
    if (push) fb.F_next[b * c.S_cap + next0 + sc.ex1] = static_cast<int32_t>(u2);
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

}  // namespace fastnn
