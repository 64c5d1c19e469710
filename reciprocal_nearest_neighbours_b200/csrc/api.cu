// C ABI entry points (declared in include/fastnn.h): argument checks,
// workspace carving and the launch sequence of each operation. No memory is
// allocated here; every launch goes on the caller's stream.
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "frontier.cuh"
#include "l2_nn.cuh"
#include "nn_tc.cuh"

using namespace fastnn;

namespace fastnn {
namespace {
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
}
void note_cuda_error(cudaError_t e) { g_last_cuda_error = e; }
}  // namespace fastnn

namespace {

// Limit of the kernels' bounded pipeline waits for subsequent calls (0: the
// kernels' default of two seconds); see fastnn_set_wait_timeout_ns.
std::atomic<uint64_t> g_wait_ns{0};

constexpr size_t kAlign = 256;
constexpr int kPadRows = 256;  // zero rows after each repacked database (one TMA box)
constexpr int kMaxIter = 255;
// Status block at the head of every workspace: [0] device status word,
// [1] / [2] max |element| of the first / second int8 map, [4] / [5] grid-
// barrier arrival counter and abort word of the persistent matching kernel.
constexpr size_t kStatusBytes = 64 * sizeof(int);
constexpr int64_t kMaxSeeds = (int64_t{1} << 24) - 1;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Bump allocator over the caller's workspace (or a size-only dry run).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

bool dtype_ok(int dtype) {
  return dtype == FASTNN_I8 || dtype == FASTNN_BF16 || dtype == FASTNN_F16 ||
         dtype == FASTNN_F32_L2;
}
bool d_ok(int d, int dtype) { return d >= 1 && d <= (dtype == FASTNN_F32_L2 ? 3 : 64); }

struct NNLayout {
  int* status;
  uint8_t* qrep;
  uint8_t* dbrep;
  uint64_t* keys;
};
NNLayout carve_nn(Carver& c, int64_t nq, int64_t ndb, int d, int dtype) {
  NNLayout L;
  const int rb = row_bytes(dtype, d);
  L.status = c.take<int>(64);
  L.qrep = c.take<uint8_t>(static_cast<size_t>(nq) * rb);
  L.dbrep = c.take<uint8_t>(static_cast<size_t>(ndb + kPadRows) * rb);
  L.keys = c.take<uint64_t>(static_cast<size_t>(nq));
  return L;
}

struct RecLayout {
  int* status;
  uint8_t* d1rep;
  uint8_t* d2rep;
  int32_t* F[2];
  uint32_t* Bd[2];
  float4* box1;  // pointmaps: chunk boxes of image 1 (database of the backward pass)
  float4* box2;  // pointmaps: chunk boxes of image 2
  uint64_t* fwd;
  uint64_t* bwd;
  uint32_t* claim;
  int32_t* cnt[2];
};
RecLayout carve_rec(Carver& c, int64_t N1, int64_t N2, int d, int dtype, int batch, int64_t S) {
  RecLayout L;
  const int rb = row_bytes(dtype, d);
  L.status = c.take<int>(64);
  L.d1rep = c.take<uint8_t>(static_cast<size_t>(batch * N1 + kPadRows) * rb);
  L.d2rep = c.take<uint8_t>(static_cast<size_t>(batch * N2 + kPadRows) * rb);
  L.F[0] = c.take<int32_t>(static_cast<size_t>(batch) * S);
  L.F[1] = c.take<int32_t>(static_cast<size_t>(batch) * S);
  L.Bd[0] = c.take<uint32_t>(static_cast<size_t>(batch) * S);
  L.Bd[1] = c.take<uint32_t>(static_cast<size_t>(batch) * S);
  L.box1 = L.box2 = nullptr;
  if (dtype == FASTNN_F32_L2) {
    L.box1 = c.take<float4>(static_cast<size_t>(batch) * 2 * ((N1 + kL2Chunk - 1) / kL2Chunk));
    L.box2 = c.take<float4>(static_cast<size_t>(batch) * 2 * ((N2 + kL2Chunk - 1) / kL2Chunk));
  }
  L.fwd = c.take<uint64_t>(static_cast<size_t>(batch) * S);
  L.bwd = c.take<uint64_t>(static_cast<size_t>(batch) * S);
  L.claim = c.take<uint32_t>(static_cast<size_t>(batch) * N1);
  L.cnt[0] = c.take<int32_t>(static_cast<size_t>(batch));
  L.cnt[1] = c.take<int32_t>(static_cast<size_t>(batch));
  return L;
}

struct MutLayout {
  int* status;
  uint8_t* d1rep;
  uint8_t* d2rep;
  uint64_t* k12;
  uint64_t* k21;
  int32_t* blocks;
  int32_t* pos21;    // [n2] slot of image-2 row j in the backward list (matched rows only)
  uint32_t* first21; // [n2] first image-1 row matched to j
  int32_t* list21;   // [n2] image-2 rows of the backward pass (the image of NN12)
  int32_t* cnt21;    // [1] their number
  int32_t* blocks2;  // image-list scan scratch
  uint32_t* best21;  // [n2] best forward score bits among the rows matched to j
  uint32_t* bnd21;   // [n2] the same, per list slot: the backward pass's score bounds
  float4* box1;      // pointmaps: chunk boxes of image 1 (database of the backward pass)
};
MutLayout carve_mut(Carver& c, int64_t n1, int64_t n2, int d, int dtype) {
  MutLayout L;
  const int rb = row_bytes(dtype, d);
  L.status = c.take<int>(64);
  L.d1rep = c.take<uint8_t>(static_cast<size_t>(n1 + kPadRows) * rb);
  L.d2rep = c.take<uint8_t>(static_cast<size_t>(n2 + kPadRows) * rb);
  L.k12 = c.take<uint64_t>(static_cast<size_t>(n1));
  L.k21 = c.take<uint64_t>(static_cast<size_t>(n2));
  L.blocks = c.take<int32_t>(static_cast<size_t>(mutual_scratch_ints(n1)));
  L.pos21 = c.take<int32_t>(static_cast<size_t>(n2));
  L.list21 = c.take<int32_t>(static_cast<size_t>(n2));
  L.cnt21 = c.take<int32_t>(1);
  L.blocks2 = c.take<int32_t>(static_cast<size_t>(image_blocks(n1)));
  L.first21 = c.take<uint32_t>(static_cast<size_t>(n2));
  L.best21 = c.take<uint32_t>(static_cast<size_t>(n2));
  L.bnd21 = c.take<uint32_t>(static_cast<size_t>(n2));
  L.box1 = dtype == FASTNN_F32_L2
               ? c.take<float4>(static_cast<size_t>(2 * ((n1 + kL2Chunk - 1) / kL2Chunk)))
               : nullptr;
  return L;
}

// Compaction state of the confidence-masked calls.
struct MaskLayout {
  int32_t* c2p1;     // [batch][N1] pixel of compacted image-1 slot
  int32_t* p2c1;     // [batch][N1] slot of image-1 pixel (-1: dropped); fast scheme only
  int32_t* c2p2;     // [batch][N2]
  int32_t* cnt1;     // [batch] kept pixels of image 1
  int32_t* cnt2;     // [batch]
  int32_t* seedcnt;  // [batch] kept seeds
  int32_t* blocks;   // per-block scan scratch, reused by both maps
};
MaskLayout carve_mask(Carver& c, int64_t N1, int64_t N2, int batch, bool seeds) {
  MaskLayout L;
  L.c2p1 = c.take<int32_t>(static_cast<size_t>(batch) * N1);
  L.p2c1 = seeds ? c.take<int32_t>(static_cast<size_t>(batch) * N1) : nullptr;
  L.c2p2 = c.take<int32_t>(static_cast<size_t>(batch) * N2);
  L.cnt1 = c.take<int32_t>(static_cast<size_t>(batch));
  L.cnt2 = c.take<int32_t>(static_cast<size_t>(batch));
  L.seedcnt = c.take<int32_t>(static_cast<size_t>(batch));
  const int bpp = mask_blocks(N1) > mask_blocks(N2) ? mask_blocks(N1) : mask_blocks(N2);
  L.blocks = c.take<int32_t>(static_cast<size_t>(batch) * bpp);
  return L;
}

int64_t seed_count(int H, int W, int sub) {
  return static_cast<int64_t>((H + sub - 1) / sub) * ((W + sub - 1) / sub);
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define FASTNN_TRY(expr)              \
  do {                                \
    int rc_ = (expr);                 \
    if (rc_ != FASTNN_OK) return rc_; \
  } while (0)

}  // namespace

extern "C" {

size_t fastnn_workspace_size(int op, int64_t n1, int64_t n2, int d, int dtype, int batch,
                             int64_t max_queries) {
  if (!dtype_ok(dtype) || !d_ok(d, dtype) || n1 < 0 || n2 < 1) return 0;
  Carver c{nullptr};
  switch (op) {
    case FASTNN_OP_NN:
      carve_nn(c, n1, n2, d, dtype);
      break;
    case FASTNN_OP_RECIPROCAL:
      if (batch < 1 || max_queries < 1 || n1 < 1) return 0;
      carve_rec(c, n1, n2, d, dtype, batch, max_queries);
      break;
    case FASTNN_OP_MUTUAL_DENSE:
      if (n1 < 1) return 0;
      carve_mut(c, n1, n2, d, dtype);
      break;
    case FASTNN_OP_MUTUAL_FROM_NN:
      c.take<int32_t>(static_cast<size_t>(mutual_scratch_ints(n1 > 0 ? n1 : 1)));
      break;
    case FASTNN_OP_IMAGE_ROWS:
      c.take<uint8_t>(static_cast<size_t>(n2));
      c.take<int32_t>(static_cast<size_t>(mutual_blocks(n2)));
      break;
    case FASTNN_OP_RECIPROCAL_MASKED:
      if (batch < 1 || max_queries < 1 || n1 < 1) return 0;
      carve_rec(c, n1, n2, d, dtype, batch, max_queries);
      carve_mask(c, n1, n2, batch, true);
      break;
    case FASTNN_OP_MUTUAL_DENSE_MASKED:
      if (n1 < 1) return 0;
      carve_mut(c, n1, n2, d, dtype);
      carve_mask(c, n1, n2, 1, false);
      break;
    default:
      return 0;
  }
  return c.off;
}

int fastnn_nn(const void* q, int64_t nq, const void* db, int64_t ndb, int d, int dtype,
              int32_t* out_idx, void* out_score, void* workspace, size_t workspace_bytes,
              fastnn_stream_t stream) {
  if (!dtype_ok(dtype) || !d_ok(d, dtype)) return FASTNN_ERR_UNSUPPORTED;
  if (nq < 0 || ndb < 1 || nq > INT32_MAX || ndb > INT32_MAX - kPadRows) return FASTNN_ERR_INVALID;
  if (nq == 0) return FASTNN_OK;
  if (!q || !db || !out_idx || !workspace || !aligned(workspace, kAlign)) return FASTNN_ERR_INVALID;
  if (workspace_bytes < fastnn_workspace_size(FASTNN_OP_NN, nq, ndb, d, dtype, 1, 0))
    return FASTNN_ERR_CAPACITY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Carver c{static_cast<uint8_t*>(workspace)};
  NNLayout L = carve_nn(c, nq, ndb, d, dtype);
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.status, 0, kStatusBytes, st));
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.keys, 0, static_cast<size_t>(nq) * sizeof(uint64_t), st));
  FASTNN_TRY(launch_repack(q, nq, d, dtype, L.qrep, 0, L.status + 1, st));
  FASTNN_TRY(launch_repack(db, ndb, d, dtype, L.dbrep, kPadRows, L.status + 2, st));
  NNArgs a{};
  a.q_rows = L.qrep;
  a.q_rows_per_pair = nq;
  a.q_cap = nq;
  a.nq_static = nq;
  a.db_rows = L.dbrep;
  a.ndb = ndb;
  a.out_key = L.keys;
  a.batch = 1;
  a.status = L.status;
  a.d = d;
  a.q_absmax = L.status + 1;
  a.db_absmax = L.status + 2;
  a.wait_ns = g_wait_ns.load();
  if (dtype == FASTNN_F32_L2) {
    FASTNN_TRY(launch_nn_l2(a, st));
    return launch_decode(L.keys, nq, dtype, out_idx, out_score, st);
  }
  FASTNN_TRY(launch_nn_tc(a, dtype, ndb + kPadRows, st));
  return launch_decode(L.keys, nq, dtype, out_idx, out_score, st);
}

}  // extern "C"

namespace {

// The fast scheme, unmasked or (masked == true) among confident pixels.
int reciprocal_impl(const void* desc1, const float* conf1, int H1, int W1, const void* desc2,
                    const float* conf2, int H2, int W2, int d, int dtype, bool masked,
                    float threshold, int subsample, int max_iter, int batch, int32_t* out_pairs,
                    void* out_score, int64_t capacity, int32_t* out_count, int32_t* out_iters,
                    int32_t* out_frontier, void* workspace, size_t workspace_bytes,
                    fastnn_stream_t stream) {
  if (!dtype_ok(dtype) || !d_ok(d, dtype)) return FASTNN_ERR_UNSUPPORTED;
  if (H1 < 1 || W1 < 1 || H2 < 1 || W2 < 1 || subsample < 1 || max_iter < 1 ||
      max_iter > kMaxIter || batch < 1 || batch > nn_tc_max_batch())
    return FASTNN_ERR_INVALID;
  const int64_t N1 = static_cast<int64_t>(H1) * W1;
  const int64_t N2 = static_cast<int64_t>(H2) * W2;
  if (batch * N1 > INT32_MAX - kPadRows || batch * N2 > INT32_MAX - kPadRows)
    return FASTNN_ERR_INVALID;
  const int64_t S = seed_count(H1, W1, subsample);
  if (S > kMaxSeeds) return FASTNN_ERR_INVALID;
  if (!desc1 || !desc2 || !out_pairs || !out_count || !workspace || !aligned(workspace, kAlign))
    return FASTNN_ERR_INVALID;
  if (capacity < S) return FASTNN_ERR_CAPACITY;
  const int op = masked ? FASTNN_OP_RECIPROCAL_MASKED : FASTNN_OP_RECIPROCAL;
  if (workspace_bytes < fastnn_workspace_size(op, N1, N2, d, dtype, batch, S))
    return FASTNN_ERR_CAPACITY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Carver c{static_cast<uint8_t*>(workspace)};
  RecLayout L = carve_rec(c, N1, N2, d, dtype, batch, S);

  // Status block: status word, per-map max |element|, grid-barrier words.
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.status, 0, kStatusBytes, st));
  MaskLayout M{};
  if (masked) {
    // Kept pixels of each map, compacted in pixel order; kept grid seeds.
    M = carve_mask(c, N1, N2, batch, true);
    MaskArgs m1{static_cast<const uint8_t*>(desc1), conf1, threshold, N1, batch, d,
                L.d1rep, M.c2p1, M.p2c1, M.cnt1, L.status + 1, M.blocks, 0};
    FASTNN_TRY(launch_mask_compact(m1, dtype, st));
    MaskArgs m2{static_cast<const uint8_t*>(desc2), conf2, threshold, N2, batch, d,
                L.d2rep, M.c2p2, nullptr, M.cnt2, L.status + 2, M.blocks, 0};
    FASTNN_TRY(launch_mask_compact(m2, dtype, st));
    FASTNN_TRY(launch_masked_seeds(M.p2c1, batch, N1, W1, subsample, S, L.F[0], M.seedcnt, st));
  }
  // The tensor-core kernel repacks both maps itself (in its clearing pass)
  // when their rows are whole 8-byte words at 8-byte aligned addresses;
  // otherwise the repack kernels run first.
  const int nbytes = d * (dtype == FASTNN_I8 ? 1 : dtype == FASTNN_F32_L2 ? 4 : 2);
  const bool repack_in_kernel = !masked && dtype != FASTNN_F32_L2 && nbytes % 8 == 0 &&
                                aligned(desc1, 8) && aligned(desc2, 8);
  if (!masked && !repack_in_kernel) {
    FASTNN_TRY(launch_repack(desc1, batch * N1, d, dtype, L.d1rep, kPadRows, L.status + 1, st));
    FASTNN_TRY(launch_repack(desc2, batch * N2, d, dtype, L.d2rep, kPadRows, L.status + 2, st));
  }

  RecArgs r{};
  if (repack_in_kernel) {
    r.src1 = static_cast<const uint8_t*>(desc1);
    r.src2 = static_cast<const uint8_t*>(desc2);
    r.src_nbytes = nbytes;
  }
  r.N2 = N2;
  r.fwd.q_rows = L.d1rep;
  r.fwd.q_rows_per_pair = N1;
  r.fwd.q_cap = S;
  r.fwd.db_rows = L.d2rep;
  r.fwd.ndb = N2;
  r.fwd.out_key = L.fwd;
  r.fwd.batch = batch;
  r.fwd.status = L.status;
  r.fwd.d = d;
  r.fwd.q_absmax = L.status + 1;
  r.fwd.db_absmax = L.status + 2;
  r.fwd.wait_ns = g_wait_ns.load();
  r.bwd = r.fwd;
  r.bwd.q_rows = L.d2rep;
  r.bwd.q_rows_per_pair = N2;
  r.bwd.q_key = L.fwd;
  r.bwd.db_rows = L.d1rep;
  r.bwd.ndb = N1;
  r.bwd.out_key = L.bwd;
  r.bwd.q_absmax = L.status + 2;
  r.bwd.db_absmax = L.status + 1;
  r.fwd.db_box = L.box2;
  r.bwd.db_box = L.box1;
  if (masked) {
    r.fwd.ndb_dev = M.cnt2;
    r.bwd.ndb_dev = M.cnt1;
    r.seed_cnt = M.seedcnt;
    r.cmp.map1 = M.c2p1;
    r.cmp.map2 = M.c2p2;
  }
  r.cmp.S_cap = S;
  r.cmp.fwd_key = L.fwd;
  r.cmp.bwd_key = L.bwd;
  r.cmp.claim = L.claim;
  r.cmp.N1 = N1;
  r.cmp.N2 = N2;
  r.cmp.out_pairs = out_pairs;
  r.cmp.out_score = out_score;
  r.cmp.cap = capacity;
  r.cmp.out_count = out_count;
  r.cmp.out_iters = out_iters;
  r.cmp.out_frontier = out_frontier;
  r.cmp.max_iter = max_iter;
  r.F[0] = L.F[0];
  r.F[1] = L.F[1];
  r.Bd[0] = L.Bd[0];
  r.Bd[1] = L.Bd[1];
  r.cnt[0] = L.cnt[0];
  r.cnt[1] = L.cnt[1];
  r.N1 = N1;
  r.S = S;
  r.W1 = W1;
  r.sub = subsample;
  r.max_iter = max_iter;
  r.batch = batch;
  r.grid_count = reinterpret_cast<uint32_t*>(L.status + 4);
  r.grid_abort = L.status + 5;
  r.status = L.status;
  if (dtype == FASTNN_F32_L2) return launch_reciprocal_l2(r, st);
  return launch_reciprocal(r, dtype, batch * N1 + kPadRows, batch * N2 + kPadRows, st);
}

}  // namespace

extern "C" {

int fastnn_reciprocal(const void* desc1, int H1, int W1, const void* desc2, int H2, int W2, int d,
                      int dtype, int subsample, int max_iter, int batch, int32_t* out_pairs,
                      void* out_score, int64_t capacity, int32_t* out_count, int32_t* out_iters,
                      int32_t* out_frontier, void* workspace, size_t workspace_bytes,
                      fastnn_stream_t stream) {
  return reciprocal_impl(desc1, nullptr, H1, W1, desc2, nullptr, H2, W2, d, dtype, false, 0.f,
                         subsample, max_iter, batch, out_pairs, out_score, capacity, out_count,
                         out_iters, out_frontier, workspace, workspace_bytes, stream);
}

int fastnn_reciprocal_masked(const void* desc1, const float* conf1, int H1, int W1,
                             const void* desc2, const float* conf2, int H2, int W2, int d,
                             int dtype, float conf_threshold, int subsample, int max_iter,
                             int batch, int32_t* out_pairs, void* out_score, int64_t capacity,
                             int32_t* out_count, int32_t* out_iters, int32_t* out_frontier,
                             void* workspace, size_t workspace_bytes, fastnn_stream_t stream) {
  if (conf_threshold != conf_threshold) return FASTNN_ERR_INVALID;  // NaN threshold
  return reciprocal_impl(desc1, conf1, H1, W1, desc2, conf2, H2, W2, d, dtype, true,
                         conf_threshold, subsample, max_iter, batch, out_pairs, out_score,
                         capacity, out_count, out_iters, out_frontier, workspace,
                         workspace_bytes, stream);
}

}  // extern "C"

namespace {

int mutual_dense_impl(const void* desc1, const float* conf1, int64_t n1, const void* desc2,
                      const float* conf2, int64_t n2, int d, int dtype, bool masked,
                      float threshold, int32_t* out_pairs, void* out_score, int64_t capacity,
                      int32_t* out_count, void* workspace, size_t workspace_bytes,
                      fastnn_stream_t stream) {
  if (!dtype_ok(dtype) || !d_ok(d, dtype)) return FASTNN_ERR_UNSUPPORTED;
  if (n1 < 1 || n2 < 1 || n1 > INT32_MAX - kPadRows || n2 > INT32_MAX - kPadRows)
    return FASTNN_ERR_INVALID;
  if (!desc1 || !desc2 || !out_pairs || !out_count || !workspace || !aligned(workspace, kAlign))
    return FASTNN_ERR_INVALID;
  if (capacity < (n1 < n2 ? n1 : n2)) return FASTNN_ERR_CAPACITY;
  const int op = masked ? FASTNN_OP_MUTUAL_DENSE_MASKED : FASTNN_OP_MUTUAL_DENSE;
  if (workspace_bytes < fastnn_workspace_size(op, n1, n2, d, dtype, 1, 0))
    return FASTNN_ERR_CAPACITY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Carver c{static_cast<uint8_t*>(workspace)};
  MutLayout L = carve_mut(c, n1, n2, d, dtype);
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.status, 0, kStatusBytes, st));
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.k12, 0, static_cast<size_t>(n1) * 8, st));
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.k21, 0, static_cast<size_t>(n2) * 8, st));
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.first21, 0xFF, static_cast<size_t>(n2) * 4, st));
  FASTNN_CUDA_TRY(cudaMemsetAsync(L.best21, 0, static_cast<size_t>(n2) * 4, st));
  MaskLayout M{};
  if (masked) {
    M = carve_mask(c, n1, n2, 1, false);
    MaskArgs m1{static_cast<const uint8_t*>(desc1), conf1, threshold, n1, 1, d,
                L.d1rep, M.c2p1, nullptr, M.cnt1, L.status + 1, M.blocks, 0};
    FASTNN_TRY(launch_mask_compact(m1, dtype, st));
    MaskArgs m2{static_cast<const uint8_t*>(desc2), conf2, threshold, n2, 1, d,
                L.d2rep, M.c2p2, nullptr, M.cnt2, L.status + 2, M.blocks, 0};
    FASTNN_TRY(launch_mask_compact(m2, dtype, st));
  } else {
    FASTNN_TRY(launch_repack(desc1, n1, d, dtype, L.d1rep, kPadRows, L.status + 1, st));
    FASTNN_TRY(launch_repack(desc2, n2, d, dtype, L.d2rep, kPadRows, L.status + 2, st));
  }
  NNArgs a{};
  a.q_rows = L.d1rep;
  a.q_rows_per_pair = n1;
  a.q_cap = n1;
  a.nq_static = n1;
  a.db_rows = L.d2rep;
  a.ndb = n2;
  a.out_key = L.k12;
  a.batch = 1;
  a.status = L.status;
  a.d = d;
  a.q_absmax = L.status + 1;
  a.db_absmax = L.status + 2;
  a.wait_ns = g_wait_ns.load();
  if (masked) {
    a.q_count = M.cnt1;
    a.ndb_dev = M.cnt2;
  }
  if (dtype == FASTNN_F32_L2)
    FASTNN_TRY(launch_nn_l2(a, st));
  else
    FASTNN_TRY(launch_nn_tc(a, dtype, n2 + kPadRows, st));
  // A mutual pair (i, j) has j = NN12(i): the backward pass needs only the
  // rows in the image of NN12, listed in the order of the first image-1 row
  // matched to each; its keys are indexed by list slot.
  FASTNN_TRY(launch_image_list(L.k12, n1, n2, L.first21, L.best21, L.pos21, L.list21, L.bnd21,
                               L.cnt21, L.blocks2, st));
  NNArgs r{};
  r.q_rows = L.d2rep;
  r.q_rows_per_pair = n2;
  r.q_cap = n2;
  r.nq_static = n2;
  r.q_index = L.list21;
  r.q_count = L.cnt21;
  r.q_bound = L.bnd21;
  if (dtype == FASTNN_F32_L2) {
    FASTNN_TRY(launch_chunk_boxes(reinterpret_cast<const float4*>(L.d1rep), n1, 1,
                                  masked ? M.cnt1 : nullptr, L.box1, st));
    r.db_box = L.box1;
  }
  r.db_rows = L.d1rep;
  r.ndb = n1;
  r.out_key = L.k21;
  r.batch = 1;
  r.status = L.status;
  r.d = d;
  r.q_absmax = L.status + 2;
  r.db_absmax = L.status + 1;
  r.wait_ns = g_wait_ns.load();
  if (masked) r.ndb_dev = M.cnt1;
  if (dtype == FASTNN_F32_L2)
    FASTNN_TRY(launch_nn_l2(r, st));
  else
    FASTNN_TRY(launch_nn_tc(r, dtype, n1 + kPadRows, st));
  MutualSrc m{};
  m.k12 = L.k12;
  m.k21 = L.k21;

  m.n1 = n1;
  m.n2 = n2;
  m.map1 = M.c2p1;
  m.map2 = M.c2p2;
  m.pos21 = L.pos21;
  return launch_mutual(m, L.blocks, dtype, out_pairs, out_score, capacity, out_count, st);
}

}  // namespace

extern "C" {

int fastnn_mutual_dense(const void* desc1, int64_t n1, const void* desc2, int64_t n2, int d,
                        int dtype, int32_t* out_pairs, void* out_score, int64_t capacity,
                        int32_t* out_count, void* workspace, size_t workspace_bytes,
                        fastnn_stream_t stream) {
  return mutual_dense_impl(desc1, nullptr, n1, desc2, nullptr, n2, d, dtype, false, 0.f,
                           out_pairs, out_score, capacity, out_count, workspace,
                           workspace_bytes, stream);
}

int fastnn_mutual_dense_masked(const void* desc1, const float* conf1, int64_t n1,
                               const void* desc2, const float* conf2, int64_t n2, int d,
                               int dtype, float conf_threshold, int32_t* out_pairs,
                               void* out_score, int64_t capacity, int32_t* out_count,
                               void* workspace, size_t workspace_bytes, fastnn_stream_t stream) {
  if (conf_threshold != conf_threshold) return FASTNN_ERR_INVALID;  // NaN threshold
  return mutual_dense_impl(desc1, conf1, n1, desc2, conf2, n2, d, dtype, true, conf_threshold,
                           out_pairs, out_score, capacity, out_count, workspace,
                           workspace_bytes, stream);
}

int fastnn_mutual_from_nn(const int32_t* nn12, const void* score12, int64_t n1, int64_t i0,
                          const int32_t* nn21, int64_t n2, int64_t n1_total, int dtype,
                          int32_t* out_pairs, void* out_score, int64_t capacity,
                          int32_t* out_count, void* workspace, size_t workspace_bytes,
                          fastnn_stream_t stream) {
  if (!dtype_ok(dtype)) return FASTNN_ERR_UNSUPPORTED;
  if (n1 < 0 || n2 < 1 || i0 < 0 || n1_total < i0 + n1 || n1_total > INT32_MAX ||
      n2 > INT32_MAX)
    return FASTNN_ERR_INVALID;
  if (!out_count) return FASTNN_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n1 == 0) {
    FASTNN_CUDA_TRY(cudaMemsetAsync(out_count, 0, sizeof(int32_t), st));
    return FASTNN_OK;
  }
  if (!nn12 || !nn21 || !out_pairs || !workspace || !aligned(workspace, kAlign))
    return FASTNN_ERR_INVALID;
  if (capacity < (n1 < n2 ? n1 : n2)) return FASTNN_ERR_CAPACITY;
  if (workspace_bytes < fastnn_workspace_size(FASTNN_OP_MUTUAL_FROM_NN, n1, n2, 1, dtype, 1, 0))
    return FASTNN_ERR_CAPACITY;
  Carver c{static_cast<uint8_t*>(workspace)};
  int32_t* blocks = c.take<int32_t>(static_cast<size_t>(mutual_scratch_ints(n1)));
  MutualSrc m{};
  m.nn12 = nn12;
  m.nn21 = nn21;
  m.score12 = score12;
  m.n1 = n1;
  m.n2 = n2;
  m.i0 = i0;
  return launch_mutual(m, blocks, dtype, out_pairs, out_score, capacity, out_count, st);
}

int fastnn_image_rows(const int32_t* nn12, int64_t n1, int64_t n2, int32_t* out_rows,
                      int32_t* out_count, void* workspace, size_t workspace_bytes,
                      fastnn_stream_t stream) {
  if (n1 < 0 || n2 < 1 || n2 > INT32_MAX) return FASTNN_ERR_INVALID;
  if ((n1 > 0 && !nn12) || !out_rows || !out_count || !workspace || !aligned(workspace, kAlign))
    return FASTNN_ERR_INVALID;
  if (workspace_bytes <
      fastnn_workspace_size(FASTNN_OP_IMAGE_ROWS, n1, n2, 1, FASTNN_I8, 1, 0))
    return FASTNN_ERR_CAPACITY;
  Carver c{static_cast<uint8_t*>(workspace)};
  uint8_t* flag = c.take<uint8_t>(static_cast<size_t>(n2));
  int32_t* blocks = c.take<int32_t>(static_cast<size_t>(mutual_blocks(n2)));
  return launch_image_rows(nn12, n1, n2, flag, blocks, out_rows, out_count,
                           reinterpret_cast<cudaStream_t>(stream));
}

int fastnn_device_status(const void* workspace, fastnn_stream_t stream) {
  if (!workspace) return FASTNN_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int h = 0;
  FASTNN_CUDA_TRY(cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, st));
  FASTNN_CUDA_TRY(cudaStreamSynchronize(st));
  return (h & kStatusTimeout) ? FASTNN_ERR_TIMEOUT : FASTNN_OK;
}

int fastnn_kernel_timer_enable(int capacity) { return kernel_timer_enable(capacity); }

int fastnn_kernel_timer_select(int kinds) { return kernel_timer_select(kinds); }

void fastnn_set_wait_timeout_ns(uint64_t ns) { g_wait_ns.store(ns); }

int fastnn_kernel_timer_read(int* launches, double* total_ms) {
  return kernel_timer_read(launches, total_ms);
}

const char* fastnn_last_cuda_error(void) {
  return cudaGetErrorString(fastnn::g_last_cuda_error);
}

const char* fastnn_status_str(int status) {
  switch (status) {
    case FASTNN_OK: return "FASTNN_OK";
    case FASTNN_ERR_INVALID: return "FASTNN_ERR_INVALID";
    case FASTNN_ERR_UNSUPPORTED: return "FASTNN_ERR_UNSUPPORTED";
    case FASTNN_ERR_CAPACITY: return "FASTNN_ERR_CAPACITY";
    case FASTNN_ERR_CUDA: return "FASTNN_ERR_CUDA";
    case FASTNN_ERR_TIMEOUT: return "FASTNN_ERR_TIMEOUT";
    default: return "FASTNN_UNKNOWN_STATUS";
  }
}

}  // extern "C"
