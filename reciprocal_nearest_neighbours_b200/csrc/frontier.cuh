// Launchers of the memory-bound kernels (frontier.cu).
#pragma once

#include "common.cuh"

namespace fastnn {

// Per-round state of the fast scheme, all device pointers.
struct CompactArgs {
  const int32_t* F_cur;   // [batch][S_cap] frontier of this round
  int32_t* F_next;        // [batch][S_cap] frontier of the next round
  int64_t S_cap;
  const int32_t* cnt_cur; // [batch]
  int32_t* cnt_next;      // [batch]
  uint64_t* fwd_key;      // [batch][S_cap] NN12 of the frontier (reset to 0 here)
  uint64_t* bwd_key;      // [batch][S_cap] NN21 of those matches (reset to 0 here)
  uint32_t* claim;        // [batch][N1] first-visit stamps (round << 24 | slot)
  int64_t N1;
  int64_t N2;
  const int32_t* map1;    // optional [batch][N1]: pixel of compacted image-1 index (masks)
  const int32_t* map2;    // optional [batch][N2]: pixel of compacted image-2 index
  int32_t* out_pairs;     // [batch][cap][2]
  void* out_score;        // [batch][cap] or nullptr
  int64_t cap;
  int32_t* out_count;     // [batch]
  int32_t* out_iters;     // [batch] or nullptr
  int32_t* out_frontier;  // [batch][max_iter] or nullptr
  int max_iter;
};

// Everything a persistent fast-matching kernel needs (device pointers).
struct RecArgs {
  NNArgs fwd;        // forward pass template: queries = image-1 rows, database = image 2
  NNArgs bwd;        // backward pass template: queries = image-2 rows of the forward keys
  CompactArgs cmp;   // per-round check/compaction template
  int32_t* F[2];     // frontier ping-pong [batch][S]
  uint32_t* Bd[2];   // score bounds of the frontier entries (ordered bits) [batch][S]
  int32_t* cnt[2];   // frontier sizes ping-pong [batch]
  int64_t N1;        // pixels of image 1
  int64_t S;         // seeds per pair
  int W1, sub, max_iter, batch;
  uint32_t* grid_count;  // grid-barrier arrival counter (zero before the launch)
  int* grid_abort;       // set when any CTA gives up (zero before the launch)
  int* status;
  const int32_t* seed_cnt;  // optional [batch]: F[0] already holds this many seeds per pair
  // Repack inside the kernel (src_nbytes > 0): the raw maps [batch * N][d]
  // (rows of src_nbytes bytes, a multiple of 8, 8-byte aligned) are written
  // to r.bwd.db_rows / r.fwd.db_rows (plus 256 zero rows each) by the
  // clearing pass, before the first grid barrier.
  const uint8_t* src1;
  const uint8_t* src2;
  int src_nbytes;
  int64_t N2;
};

// Confidence-mask compaction of one map (all pairs of a batch).
struct MaskArgs {
  const uint8_t* src;   // [batch][N][d] rows of the map (dtype's element size)
  const float* conf;    // [batch][N] confidences, or nullptr (every pixel kept)
  float threshold;      // kept iff conf >= threshold
  int64_t N;            // pixels per pair
  int batch;
  int d;
  uint8_t* dst;         // [batch][N] repacked rows; the first count[b] of pair b are kept
  int32_t* c2p;         // [batch][N]: pixel of compacted slot
  int32_t* p2c;         // [batch][N]: slot of pixel, -1 when dropped (or nullptr)
  int32_t* count;       // [batch] kept pixels
  int* absmax;          // int8: max |element|; pointmaps: bits of max |p|^2 (or nullptr)
  int32_t* blocks;      // [batch][mask_blocks(N)] scratch
  int bpp;              // set by the launcher
};

int mask_blocks(int64_t N);
int launch_mask_compact(const MaskArgs& m, int dtype, cudaStream_t st);
// Kept grid seeds per pair (compacted indices, grid order) into F0, counts
// into seed_cnt.
int launch_masked_seeds(const int32_t* p2c, int batch, int64_t N1, int W1, int sub, int64_t S,
                        int32_t* F0, int32_t* seed_cnt, cudaStream_t st);

// Repack `rows` rows (plus pad_rows zero rows) into the kernels' layout.
// absmax (optional) receives, by atomicMax, the largest |element| (int8) or
// the fp32 bits of the largest |p|^2 (pointmaps).
int launch_repack(const void* src, int64_t rows, int d, int dtype, void* dst, int64_t pad_rows,
                  int* absmax, cudaStream_t st);
// Nearest-neighbour results for the mutual test: packed keys (k12/k21) or
// index arrays (nn12/nn21, with scores score12). Local image-1 row i is
// global row i0 + i; nn21 / k21 index global image-1 rows.
struct MutualSrc {
  const uint64_t* k12;
  const uint64_t* k21;
  const int32_t* nn12;
  const int32_t* nn21;
  const void* score12;
  const int32_t* map1;  // optional: pixel of compacted image-1 row i (masked maps)
  const int32_t* map2;  // optional: pixel of compacted image-2 row j
  const int32_t* pos21; // optional: slot of row j in k21 when the backward pass ran on a list
  int64_t n1;  // local image-1 rows
  int64_t n2;  // image-2 rows
  int64_t i0;  // global index of local row 0
};

// Scan scratch (ints) of the mutual test over n1 rows, and of the image list.
int mutual_blocks(int64_t n1);
// Scratch (ints) the mutual test takes: its block counts and one keep-flag
// byte per eight rows.
int mutual_scratch_ints(int64_t n1);
int image_blocks(int64_t n1);
// Bounding box (lo, hi; xyz) of every kL2Chunk-row chunk of each pair's
// repacked pointmap rows [batch][N]: box[(b * nchunk + c) * 2 + {0, 1}],
// nchunk = ceil(N / kL2Chunk). With `count`, pair b has count[b] rows;
// chunks past them get an empty box (lo = +inf, hi = -inf).
int launch_chunk_boxes(const float4* rows, int64_t N, int batch, const int32_t* count,
                       float4* box, cudaStream_t st);
// The image of NN12 (the rows j that are some row's forward match) as a
// list in the order of the first image-1 row matched to each j (queries next
// to each other in the list then lie near each other, whatever the order of
// image 2): on entry first[j] = 0xFFFFFFFF and best[j] = 0 for every j; on
// exit list[0..*count) holds the matched rows, pos[j] their slot (only for
// matched j) and list_bound[slot] the best forward score bits among the rows
// matched to j (a score NN21(j) reaches). block_scratch holds
// image_blocks(n1) ints.
int launch_image_list(const uint64_t* k12, int64_t n1, int64_t n2, uint32_t* first,
                      uint32_t* best, int32_t* pos, int32_t* list, uint32_t* list_bound,
                      int32_t* count, int32_t* block_scratch, cudaStream_t st);
// Ascending list of the distinct nn12[i] in [0, n2) into rows[0 .. *count).
// flag holds n2 bytes, block_scratch mutual_blocks(n2) ints.
int launch_image_rows(const int32_t* nn12, int64_t n1, int64_t n2, uint8_t* flag,
                      int32_t* block_scratch, int32_t* rows, int32_t* count, cudaStream_t st);
int launch_mutual(const MutualSrc& m, int32_t* block_scratch, int dtype, int32_t* out_pairs,
                  void* out_score, int64_t cap, int32_t* out_count, cudaStream_t st);
// Keys -> (index, score); pointmap scores are the squared distances the keys
// carry (negated).
int launch_decode(const uint64_t* key, int64_t n, int dtype, int32_t* out_idx, void* out_score,
                  cudaStream_t st);

}  // namespace fastnn
