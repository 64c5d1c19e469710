/*
 * CPU oracle for reciprocal nearest-neighbour matching: the nearest-neighbour
 * scan. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library; the product path
 * never does, and this file includes nothing from the GPU path.
 *
 * What it computes ("MASt3R dissection", section 3 Napkin Formula, the
 * inference-time reciprocal matching set): for every query descriptor q_i,
 *
 *     NN(q_i, DB) = argmax_k <q_i, DB_k>
 *
 * by a plain linear scan k = 0, 1, ..., n-1 that replaces the running best
 * only on a STRICTLY greater score, so among equal scores the lowest index
 * wins (the tie rule this build fixes; the pages are silent on ties).
 *
 * Precision: int8 descriptors are multiplied and summed exactly in int64.
 * bfloat16 and IEEE half descriptors are widened exactly to double; each
 * product of two 8- or 11-bit significands is exact in double and the sum of
 * d <= 64 such terms carries an error far below any score gap the tests look
 * at.
 *
 * The float scans also return the runner-up score (the best score over every
 * k other than the chosen one; equal to the best when the best is tied),
 * which the float tolerance rule needs.
 *
 * Pointmaps ("DUSt3R / MASt3R explained", the paragraph on recovering the
 * cameras: two pixels match when their predicted 3D points are nearest
 * neighbours in the shared frame): oracle_nn_l2 returns, for every query
 * point a, argmin_k |a - DB_k|^2 over float32 points of d <= 3 coordinates,
 * again by a linear scan that replaces the running best only on a STRICTLY
 * smaller distance (lowest index on ties). Each coordinate difference of two
 * float32 values is exact in double for the magnitudes pointmaps hold, and
 * the squared distance is summed in double.
 *
 * Queries are independent, so the outer loop may run on several threads; the
 * per-query scan is the plain sequential loop above either way.
 */
#include <stdint.h>
#include <math.h>
#include <string.h>

static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16 to double, exactly: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 holds subnormals (fraction * 2^-24). Inputs
 * are finite. */
static double f16_to_double(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1F;
    const int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else
        v = ldexp((double)(f | 0x400), e - 25);
    return sign ? -v : v;
}

typedef double (*to_double_fn)(uint16_t);

int oracle_nn_i8(const int8_t *q, int64_t nq, const int8_t *db, int64_t ndb,
                 int d, int32_t *out_idx, int64_t *out_score, int nthreads)
{
    if (nq < 0 || ndb <= 0 || d <= 0)
        return -1;
    (void)nthreads;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < nq; ++i) {
        const int8_t *qi = q + i * (int64_t)d;
        int64_t best = 0;
        int32_t best_k = -1;
        for (int64_t k = 0; k < ndb; ++k) {
            const int8_t *dk = db + k * (int64_t)d;
            int64_t s = 0;
            for (int c = 0; c < d; ++c)
                s += (int64_t)qi[c] * (int64_t)dk[c];
            if (best_k < 0 || s > best) {
                best = s;
                best_k = (int32_t)k;
            }
        }
        out_idx[i] = best_k;
        out_score[i] = best;
    }
    return 0;
}

/* 16-bit float descriptors; `cvt` widens bfloat16 or IEEE half exactly. */
static int nn_f16_like(const uint16_t *q, int64_t nq, const uint16_t *db,
                       int64_t ndb, int d, int32_t *out_idx, double *out_score,
                       double *out_second, int nthreads, to_double_fn cvt)
{
    if (nq < 0 || ndb <= 0 || d <= 0 || d > 64)
        return -1;
    (void)nthreads;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < nq; ++i) {
        double qi[64];
        for (int c = 0; c < d; ++c)
            qi[c] = cvt(q[i * (int64_t)d + c]);
        double best = 0.0, second = 0.0;
        int32_t best_k = -1;
        int have_second = 0;
        for (int64_t k = 0; k < ndb; ++k) {
            const uint16_t *dk = db + k * (int64_t)d;
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += qi[c] * cvt(dk[c]);
            if (best_k < 0) {
                best = s;
                best_k = (int32_t)k;
            } else if (s > best) {
                second = best;
                have_second = 1;
                best = s;
                best_k = (int32_t)k;
            } else if (!have_second || s > second) {
                second = s;
                have_second = 1;
            }
        }
        out_idx[i] = best_k;
        out_score[i] = best;
        out_second[i] = have_second ? second : -1.0e300;
    }
    return 0;
}

int oracle_nn_bf16(const uint16_t *q, int64_t nq, const uint16_t *db,
                   int64_t ndb, int d, int32_t *out_idx, double *out_score,
                   double *out_second, int nthreads)
{
    return nn_f16_like(q, nq, db, ndb, d, out_idx, out_score, out_second,
                       nthreads, bf16_to_double);
}

int oracle_nn_f16(const uint16_t *q, int64_t nq, const uint16_t *db,
                  int64_t ndb, int d, int32_t *out_idx, double *out_score,
                  double *out_second, int nthreads)
{
    return nn_f16_like(q, nq, db, ndb, d, out_idx, out_score, out_second,
                       nthreads, f16_to_double);
}

int oracle_nn_l2(const float *q, int64_t nq, const float *db, int64_t ndb,
                 int d, int32_t *out_idx, double *out_d2, double *out_second,
                 int nthreads)
{
    if (nq < 0 || ndb <= 0 || d <= 0 || d > 3)
        return -1;
    (void)nthreads;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < nq; ++i) {
        const float *qi = q + i * (int64_t)d;
        double best = 0.0, second = 0.0;
        int32_t best_k = -1;
        int have_second = 0;
        for (int64_t k = 0; k < ndb; ++k) {
            const float *dk = db + k * (int64_t)d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) {
                const double diff = (double)qi[c] - (double)dk[c];
                s += diff * diff;
            }
            if (best_k < 0) {
                best = s;
                best_k = (int32_t)k;
            } else if (s < best) {
                second = best;
                have_second = 1;
                best = s;
                best_k = (int32_t)k;
            } else if (!have_second || s < second) {
                second = s;
                have_second = 1;
            }
        }
        out_idx[i] = best_k;
        out_d2[i] = best;
        out_second[i] = have_second ? second : 1.0e300;
    }
    return 0;
}

/* Exposed for the oracle's own tests (exhaustive check of the conversion). */
double oracle_half_to_double(uint16_t h) { return f16_to_double(h); }
