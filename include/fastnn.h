/*
 * fastnn.h -- C ABI of the B200 (sm_100a) reciprocal nearest-neighbour
 * matcher for dense per-pixel descriptor maps (MASt3R's matching step).
 *
 * What is computed
 *   Similarity of two descriptors is their dot product; the nearest
 *   neighbour of a query in a database is argmax_k <q, db_k>, the LOWEST k
 *   among equal scores ("MASt3R dissection", section 3 Napkin Formula: the
 *   inference-time reciprocal set is written with argmax of dot products).
 *   A reciprocal match is a pair (i, j) with NN(D1[i], D2) = j and
 *   NN(D2[j], D1) = i ("MASt3R dissection", section 1 architecture diagram
 *   and section 3).
 *   Pointmaps (dtype FASTNN_F32_L2): rows are 3D points and the nearest
 *   neighbour is the nearest point, argmin_k |q - db_k|^2, lowest k on ties
 *   ("DUSt3R / MASt3R explained", the paragraph on recovering the cameras:
 *   pixels match when their predicted 3D points are nearest neighbours in
 *   the shared frame). The same reciprocal and fast schemes apply.
 *
 * Conventions shared by every entry point
 *   - Every data pointer is a DEVICE pointer owned by the caller. The library
 *     allocates no memory: scratch lives in a caller-provided workspace whose
 *     size comes from fastnn_workspace_size(). Workspace and descriptor
 *     pointers must be 256-byte aligned.
 *   - Descriptor maps are row-major [rows][d] (an image is [H][W][d], pixel
 *     index p = y * W + x); batches are [batch][rows][d].
 *   - dtype FASTNN_I8: int8 descriptors, int32 scores (exact).
 *     dtype FASTNN_BF16 / FASTNN_F16: bfloat16 / IEEE half descriptors (raw
 *     16-bit patterns), float32 scores (fp32 accumulation of exact products).
 *     1 <= d <= 64 for all three (d <= 32 runs one 32-element K step).
 *     dtype FASTNN_F32_L2: float32 points, 1 <= d <= 3 (DUSt3R pointmaps
 *     have d = 3); scores are float32 SQUARED DISTANCES (lower is nearer).
 *     Inputs must be finite. The squared distance of a point is computed in
 *     fp64 from the coordinate differences, (dx^2 + dy^2) + dz^2 with one
 *     rounding per operation, and rounded to fp32; the nearest point is the
 *     lowest index among those whose fp32 value is the smallest. (The
 *     kernels scan with fp32 scores 2<q, p> - |p|^2 and re-rank every point
 *     their rounding error could place first.)
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream). The host blocks only in fastnn_device_status().
 *   - Return value: FASTNN_OK, or a negative fastnn_status describing an
 *     argument or launch error detected on the host; nothing has been
 *     enqueued when an argument error is returned. Errors found on the
 *     device (a bounded wait that ran out) are recorded in the workspace and
 *     read with fastnn_device_status().
 *   - Calls that share a workspace must be ordered (same stream or events);
 *     overlapping calls on one workspace race.
 */
#ifndef FASTNN_H_
#define FASTNN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fastnn_stream_t; /* same type as cudaStream_t */

typedef enum {
    FASTNN_OK = 0,
    FASTNN_ERR_INVALID = -1,     /* bad pointer, size, alignment or argument */
    FASTNN_ERR_UNSUPPORTED = -2, /* d (1..64; 1..3 for pointmaps) or dtype not taken */
    FASTNN_ERR_CAPACITY = -3,    /* output capacity or workspace too small */
    FASTNN_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed */
    FASTNN_ERR_TIMEOUT = -5      /* a device-side bounded wait ran out */
} fastnn_status;

typedef enum {
    FASTNN_I8 = 0,     /* int8 descriptors, dot product, int32 scores */
    FASTNN_BF16 = 1,   /* bfloat16 descriptors, dot product, float32 scores */
    FASTNN_F16 = 2,    /* IEEE half descriptors, dot product, float32 scores */
    FASTNN_F32_L2 = 3  /* float32 3D points, Euclidean distance, float32 squared distances */
} fastnn_dtype;

typedef enum {
    FASTNN_OP_NN = 0,
    FASTNN_OP_RECIPROCAL = 1,
    FASTNN_OP_MUTUAL_DENSE = 2,
    FASTNN_OP_MUTUAL_FROM_NN = 3,
    FASTNN_OP_RECIPROCAL_MASKED = 4,
    FASTNN_OP_MUTUAL_DENSE_MASKED = 5,
    FASTNN_OP_IMAGE_ROWS = 6
} fastnn_op;

/*
 * Workspace bytes one call needs.
 *   FASTNN_OP_NN:           n1 = nq, n2 = ndb (batch and max_queries unused)
 *   FASTNN_OP_RECIPROCAL:   n1 = H1*W1, n2 = H2*W2, max_queries = number of
 *                           grid seeds per pair, batch = pairs
 *   FASTNN_OP_MUTUAL_DENSE: n1, n2 = pixel counts (batch, max_queries unused)
 *   FASTNN_OP_MUTUAL_FROM_NN: n1 = local image-1 rows, n2 = image-2 rows
 *                           (d must still be valid for dtype; unused)
 *   FASTNN_OP_RECIPROCAL_MASKED, FASTNN_OP_MUTUAL_DENSE_MASKED: as the
 *                           unmasked ops
 *   FASTNN_OP_IMAGE_ROWS:   n1 = entries of nn12, n2 = image-2 rows (d must
 *                           still be valid for dtype; unused)
 * Returns 0 for arguments no call would accept.
 */
size_t fastnn_workspace_size(int op, int64_t n1, int64_t n2, int d, int dtype,
                             int batch, int64_t max_queries);

/*
 * fastnn_nn -- nearest neighbour of every query row in a database.
 *   For i < nq: out_idx[i] = argmax_k <q[i], db[k]> (lowest k on ties),
 *   out_score[i] = that score (int32 for FASTNN_I8, float for the float
 *   types; out_score may be NULL). For FASTNN_F32_L2, out_idx[i] is the
 *   nearest point and out_score[i] its squared distance. This is the primitive of both matching schemes
 *   ("MASt3R dissection", section 3, argmax of dot products).
 *   q: [nq][d], db: [ndb][d]; nq >= 0, ndb >= 1; nq == 0 is a no-op.
 */
int fastnn_nn(const void *q, int64_t nq, const void *db, int64_t ndb, int d,
              int dtype, int32_t *out_idx, void *out_score, void *workspace,
              size_t workspace_bytes, fastnn_stream_t stream);

/*
 * fastnn_reciprocal -- MASt3R fast reciprocal matching ("DUSt3R / MASt3R
 * explained", the paragraph on fast reciprocal matching: seeds on a sparse
 * grid of image 1 are mapped to their best match in image 2 and back; pixels
 * that map onto themselves are kept; the others walk on).
 *   Seeds: pixels (x, y) of image 1 with x, y multiples of `subsample`
 *   (origin 0), S = ceil(H1/subsample) * ceil(W1/subsample) per pair.
 *   Round t = 1..max_iter while the frontier is non-empty: for u in the
 *   frontier, v = NN(D1[u], D2), u' = NN(D2[v], D1); u' == u keeps (u, v);
 *   otherwise u' joins the next frontier unless it was already in any
 *   frontier of this call (a pruning that leaves the kept set unchanged: the
 *   walk from a pixel is deterministic, and its first visit is the furthest
 *   ahead). Walks still open after max_iter rounds are dropped.
 *   desc1: [batch][H1][W1][d], desc2: [batch][H2][W2][d]; pairs independent.
 *   out_pairs: [batch][capacity][2] int32 (u, v) pixel indices in order of
 *   discovery (round, then frontier position); out_score: [batch][capacity]
 *   (int32 or float) or NULL; out_count: [batch] int32 pairs written per
 *   pair; out_iters: [batch] int32 rounds run with a non-empty frontier, or
 *   NULL; out_frontier: [batch][max_iter] int32 frontier size of each round
 *   (0 for rounds not run), or NULL. capacity must be >= S (at most one pair
 *   per seed), else
 *   FASTNN_ERR_CAPACITY. 1 <= subsample, 1 <= max_iter <= 255, S < 2^24.
 */
int fastnn_reciprocal(const void *desc1, int H1, int W1, const void *desc2,
                      int H2, int W2, int d, int dtype, int subsample,
                      int max_iter, int batch, int32_t *out_pairs,
                      void *out_score, int64_t capacity, int32_t *out_count,
                      int32_t *out_iters, int32_t *out_frontier,
                      void *workspace, size_t workspace_bytes,
                      fastnn_stream_t stream);

/*
 * fastnn_mutual_dense -- every mutual nearest-neighbour pair of two maps,
 * the brute-force reciprocal set ("MASt3R dissection", section 1 and section
 * 3; "DUSt3R / MASt3R explained" calls it the naive every-pixel-against-
 * every-pixel comparison that the fast scheme avoids).
 *   desc1: [n1][d], desc2: [n2][d]. Output pairs (i, j) in ascending i into
 *   out_pairs [capacity][2] int32 and out_score [capacity] (or NULL);
 *   *out_count (device int32) = number of pairs. capacity must be
 *   >= min(n1, n2), else FASTNN_ERR_CAPACITY.
 *   Work: NN12 for every row of desc1, then NN21 only for the rows of desc2
 *   that are some row's NN12 (no other row can be in a mutual pair).
 */
int fastnn_mutual_dense(const void *desc1, int64_t n1, const void *desc2,
                        int64_t n2, int d, int dtype, int32_t *out_pairs,
                        void *out_score, int64_t capacity, int32_t *out_count,
                        void *workspace, size_t workspace_bytes,
                        fastnn_stream_t stream);

/*
 * fastnn_mutual_from_nn -- the mutual test of the reciprocal set ("MASt3R
 * dissection", section 1 and section 3) applied to nearest-neighbour indices
 * that were computed elsewhere, for a row shard of image 1: local row i (global
 * row i0 + i) with partner j = nn12[i] is kept iff nn21[j] == i0 + i. This is
 * the last step of the dense mutual set when image 1's rows are split across
 * GPUs and nn21 (all n2 image-2 rows, global image-1 indices) was gathered.
 *   nn12: [n1] int32 in [0, n2); score12: [n1] int32/float or NULL;
 *   nn21: [n2] int32 in [0, n1_total), or -1 for a row with no partner (a row
 *   outside the image of NN12, see fastnn_image_rows). Output (i0 + i, j) in
 *   ascending i into
 *   out_pairs [capacity][2], scores into out_score (or NULL), *out_count =
 *   pairs. capacity >= min(n1, n2). n1 == 0 writes *out_count = 0.
 */
int fastnn_mutual_from_nn(const int32_t *nn12, const void *score12, int64_t n1,
                          int64_t i0, const int32_t *nn21, int64_t n2,
                          int64_t n1_total, int dtype, int32_t *out_pairs,
                          void *out_score, int64_t capacity, int32_t *out_count,
                          void *workspace, size_t workspace_bytes,
                          fastnn_stream_t stream);

/*
 * fastnn_image_rows -- the image-2 rows that can be in a mutual pair: a pair
 * (i, j) of the reciprocal set ("MASt3R dissection", section 1 and section 3)
 * has j = NN12(i), so only the rows some image-1 row matches need their own
 * nearest neighbour in image 1. Writes the distinct values of nn12 that lie
 * in [0, n2), in ascending order, to out_rows[0 .. *out_count) (device int32);
 * out_rows must hold min(n1, n2) entries. When image 1's rows are split
 * across GPUs, the gathered NN12 of all of them gives every rank the same
 * list, whose rows are then split for the backward pass.
 *   nn12: [n1] int32 (may be NULL when n1 == 0; values outside [0, n2) are
 *   ignored). Workspace: FASTNN_OP_IMAGE_ROWS.
 */
int fastnn_image_rows(const int32_t *nn12, int64_t n1, int64_t n2,
                      int32_t *out_rows, int32_t *out_count, void *workspace,
                      size_t workspace_bytes, fastnn_stream_t stream);

/*
 * fastnn_set_wait_timeout_ns -- limit of the kernels' bounded waits for the
 * calls that follow (process-wide; 0 restores the default of 2 s). Every wait
 * inside the kernels (a pipeline stage, an accumulator, a grid barrier) gives
 * up after this long: the kernel then stops issuing work, drains what it has
 * in flight (those waits always use the 2 s default), frees its tensor
 * memory and returns, and fastnn_device_status() reports FASTNN_ERR_TIMEOUT;
 * the outputs of that call are undefined, the context stays usable. Meant
 * for supervision and for testing that failure path (a limit far below a
 * call's duration makes its waits run out); the pages have no counterpart.
 */
void fastnn_set_wait_timeout_ns(uint64_t ns);

/*
 * Confidence-masked matching. The network predicts a confidence beside every
 * per-pixel output ("DUSt3R / MASt3R explained", the pointmap paragraph), and
 * the remedy for pixels whose geometry cannot be trusted is to mask them or
 * reject their low-confidence matches ("MASt3R dissection", section 5).
 * Here a pixel takes part iff conf >= conf_threshold: it is a candidate in
 * its image's database and, if on the seed grid, a seed; other pixels are
 * neither. Without a confidence map (NULL) every pixel of that image takes
 * part. Reported indices are pixel indices of the full maps; everything else
 * (tie rule, order of the output, scores, capacities, errors) is that of the
 * unmasked call. The kept pixels are compacted on the device, in pixel order,
 * before matching; confidences must not be NaN for pixels meant to be kept.
 *   conf1: [batch][H1][W1] float32 or NULL; conf2: [batch][H2][W2] or NULL.
 *   Workspace: FASTNN_OP_RECIPROCAL_MASKED (or _MUTUAL_DENSE_MASKED) sizes.
 *   capacity >= S (fast) / min(n1, n2) (dense) as for the unmasked calls;
 *   out_frontier counts kept seeds in round 1. A pair whose image 2 keeps no
 *   pixel runs one round and keeps nothing.
 */
int fastnn_reciprocal_masked(const void *desc1, const float *conf1, int H1,
                             int W1, const void *desc2, const float *conf2,
                             int H2, int W2, int d, int dtype,
                             float conf_threshold, int subsample, int max_iter,
                             int batch, int32_t *out_pairs, void *out_score,
                             int64_t capacity, int32_t *out_count,
                             int32_t *out_iters, int32_t *out_frontier,
                             void *workspace, size_t workspace_bytes,
                             fastnn_stream_t stream);

int fastnn_mutual_dense_masked(const void *desc1, const float *conf1, int64_t n1,
                               const void *desc2, const float *conf2,
                               int64_t n2, int d, int dtype,
                               float conf_threshold, int32_t *out_pairs,
                               void *out_score, int64_t capacity,
                               int32_t *out_count, void *workspace,
                               size_t workspace_bytes, fastnn_stream_t stream);

/*
 * fastnn_reciprocal_noalloc -- fastnn_reciprocal for callers that cannot
 * allocate device memory (a plugin inside an application that owns every
 * allocation, a real-time loop that must not take cudaMalloc's implicit
 * synchronisation, a fixed pre-reserved memory budget). The pages describe no
 * such entry point: it is a property of this library, with no counterpart in
 * the method.
 *   Arguments and results are those of fastnn_reciprocal without the
 *   workspace: the scratch is a static device array of
 *   FASTNN_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU loading this library
 *   holds until the process exits. Calls whose workspace would exceed it
 *   (fastnn_workspace_size) return FASTNN_ERR_CAPACITY and enqueue nothing;
 *   one 512x384 pair with int8 or bf16 descriptors fits.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture. The call allocates nothing.
 *   All calls share the one array and it keeps the last call's contents (the
 *   call clears what must start at zero). Calls that overlap on the GPU (on
 *   different streams, or from several host threads without ordering) race on
 *   it. Argument errors are returned before anything is enqueued, with the
 *   statuses fastnn_reciprocal gives; a device-side bounded wait that ran out
 *   is read with fastnn_noalloc_device_status().
 */
#define FASTNN_NOALLOC_SCRATCH_BYTES (32u << 20)

int fastnn_reciprocal_noalloc(const void *desc1, int H1, int W1, const void *desc2,
                              int H2, int W2, int d, int dtype, int subsample,
                              int max_iter, int batch, int32_t *out_pairs,
                              void *out_score, int64_t capacity,
                              int32_t *out_count, int32_t *out_iters,
                              int32_t *out_frontier, fastnn_stream_t stream);

/*
 * fastnn_noalloc_device_status -- synchronise `stream` and read the device
 * status word that the last fastnn_reciprocal_noalloc call on the CURRENT
 * device left in the static scratch array: FASTNN_OK, or FASTNN_ERR_TIMEOUT
 * when one of that call's bounded waits ran out (its outputs are then
 * invalid). Blocks the host. If no allocation-free call has run on this
 * device yet, the first use looks up the array's address (as the first
 * allocation-free call does). Like the array itself, this has no counterpart
 * in the pages.
 */
int fastnn_noalloc_device_status(fastnn_stream_t stream);

/*
 * fastnn_device_status -- synchronise `stream` and read the device status
 * word of the last call that used `workspace`: FASTNN_OK, or
 * FASTNN_ERR_TIMEOUT when a kernel's bounded wait ran out (its outputs are
 * then invalid). Blocks the host.
 */
int fastnn_device_status(const void *workspace, fastnn_stream_t stream);

/*
 * Benchmark instrumentation (not needed for matching). After
 * fastnn_kernel_timer_enable(capacity > 0), each of the next `capacity`
 * launches of the selected kinds (fastnn_kernel_timer_select below; by
 * default the nearest-neighbour and matching kernels) is bracketed by two
 * CUDA events recorded on the launching stream (events are created here, once,
 * not per call). fastnn_kernel_timer_read() waits for the recorded events,
 * returns the number of timed launches and their summed device time in
 * milliseconds, and starts a new count. fastnn_kernel_timer_enable(0)
 * destroys the events. Process-wide state: not for concurrent use from
 * several host threads.
 */
int fastnn_kernel_timer_enable(int capacity);
int fastnn_kernel_timer_read(int *launches, double *total_ms);

/*
 * fastnn_kernel_timer_select -- which launches the timer above brackets, as a
 * bit mask (each bracket covers the kernels one call of that kind launches):
 *   FASTNN_TIME_MATCHING (1, the default): the tensor-core and pointmap
 *     nearest-neighbour kernels and the persistent matching kernels;
 *   FASTNN_TIME_REPACK (2): the repack of each descriptor map;
 *   FASTNN_TIME_MUTUAL (4): the dense mutual test and ordered emit (count,
 *     scan, emit), and the list of image-2 rows the dense backward pass runs on;
 *   FASTNN_TIME_MASK (8): the confidence-mask compaction of each map.
 * kinds <= 0 leaves the selection as it is. Returns the previous selection.
 * Benchmark instrumentation: process-wide, like the timer itself.
 */
#define FASTNN_TIME_MATCHING 1
#define FASTNN_TIME_REPACK 2
#define FASTNN_TIME_MUTUAL 4
#define FASTNN_TIME_MASK 8
int fastnn_kernel_timer_select(int kinds);

/* Text of the last CUDA runtime error this library saw on the calling host
 * thread (the cause behind a FASTNN_ERR_CUDA return); a static string. */
const char *fastnn_last_cuda_error(void);

/* Human-readable name of a fastnn_status value (static string). */
const char *fastnn_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* FASTNN_H_ */
