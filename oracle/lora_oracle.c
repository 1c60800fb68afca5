/*
 * CPU oracle for the heterogeneous-batch LoRA delta -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load this
 * library.  The product path never calls it and shares no code with it.
 *
 * Everything is computed in fp64 from the already-rounded inputs (bf16 or fp32 values
 * widened exactly to double), one token at a time, in the plain order of the definition.
 *
 * Sources (multi-LoRA serving pages):
 *  - "TGI Multi-LoRA: Deploy Once, Serve 30 Models", section "Technical Foundation: LoRA":
 *    the base weight stays frozen and two small trained matrices A and B carry the
 *    adaptation, so a layer's output gains the low-rank term B A x.
 *  - Same page, "How Multi-LoRA Serving Works": every request names its own adapter, and
 *    requests for different adapters form one heterogeneous batch.
 *  - "Compress then Serve" review thread, authors' rebuttal on Punica:
 *    SGMV groups the requests that use the same LoRA model; the pseudocode of
 *    add_lora_slice_with_sigma applies A to x into an fp32 buffer of shape
 *    (tokens, R) with scale 1, then applies B to that buffer with the adapter scale and
 *    updates a column slice of y in place; the adapter of each token comes from a
 *    per-token index vector.
 *
 * Readings where the pages are silent:
 *  - an id of -1 means "no adapter": the token's output row is y0 unchanged;
 *    any other id outside [0, n) is an error (return -1);
 *  - the scale multiplies the B step only, as in the pseudocode; the delta is added to
 *    y0 without intermediate rounding (the fp64 result is returned unrounded);
 *  - segments are listed in ascending adapter id, a segment only for adapters with at
 *    least one token, and tokens keep their batch order inside a segment.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Exact widening of one stored element to double. */
static double widen(const void *base, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int ids_valid(int64_t T, const int32_t *ids, int32_t n_adapters)
{
    for (int64_t t = 0; t < T; ++t)
        if (ids[t] < -1 || ids[t] >= n_adapters)
            return 0;
    return 1;
}

static void set_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * y_ref[t, n] = y0[t, y_offset + n] + s_i * sum_k B_i[n, k] * v[k],
 * v[k]        = sum_j x[t, j] * A_i[k, j],      i = ids[t],  k < r_i,  n < o.
 *
 * x    : [T, ldx] elements, the first h columns are read.
 * y0   : [T, ldy] elements, columns [y_offset, y_offset + o) are read.
 * A[i] : [r_i, h] row-major,  B[i] : [o, r_i] row-major  (i < n_adapters).
 * y_ref: [T, o] doubles (output, written fully).
 * Returns 0, or -1 if an id is out of range (nothing is written then).
 */
int oracle_lora_delta(int dtype, int64_t T, int64_t h, int64_t o,
                      const void *x, int64_t ldx,
                      const void *y0, int64_t ldy, int64_t y_offset,
                      const int32_t *ids, int32_t n_adapters,
                      const void *const *A, const void *const *B,
                      const int32_t *ranks, const double *scales,
                      double *y_ref, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters))
        return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *xrow = (double *)malloc((size_t)h * sizeof(double));
        double *v = NULL;
        int32_t vcap = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *yr = y_ref + t * o;
            for (int64_t n = 0; n < o; ++n)
                yr[n] = widen(y0, dtype, t * ldy + y_offset + n);
            int32_t i = ids[t];
            if (i < 0)
                continue;
            int32_t r = ranks[i];
            if (r > vcap) {
                free(v);
                v = (double *)malloc((size_t)r * sizeof(double));
                vcap = r;
            }
            for (int64_t j = 0; j < h; ++j)
                xrow[j] = widen(x, dtype, t * ldx + j);
            /* shrink: v = A_i x  (scale 1) */
            for (int32_t k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int64_t j = 0; j < h; ++j)
                    acc += xrow[j] * widen(A[i], dtype, (int64_t)k * h + j);
                v[k] = acc;
            }
            /* expand: y += s_i * B_i v */
            for (int64_t n = 0; n < o; ++n) {
                double acc = 0.0;
                for (int32_t k = 0; k < r; ++k)
                    acc += widen(B[i], dtype, n * r + k) * v[k];
                yr[n] += scales[i] * acc;
            }
        }
        free(v);
        free(xrow);
    }
    return 0;
}

/*
 * Shrink step alone: v[t, k] = sum_j x[t, j] * A_i[k, j] for k < r_i; v is [T, ldv] doubles.
 * Rows of tokens without an adapter and columns k >= r_i are set to 0.
 */
int oracle_lora_shrink(int dtype, int64_t T, int64_t h,
                       const void *x, int64_t ldx,
                       const int32_t *ids, int32_t n_adapters,
                       const void *const *A, const int32_t *ranks,
                       double *v, int64_t ldv, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters))
        return -1;
    set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *vr = v + t * ldv;
        for (int64_t k = 0; k < ldv; ++k)
            vr[k] = 0.0;
        int32_t i = ids[t];
        if (i < 0)
            continue;
        for (int32_t k = 0; k < ranks[i]; ++k) {
            double acc = 0.0;
            for (int64_t j = 0; j < h; ++j)
                acc += widen(x, dtype, t * ldx + j) * widen(A[i], dtype, (int64_t)k * h + j);
            vr[k] = acc;
        }
    }
    return 0;
}

/*
 * Expand step alone, from a given fp32 intermediate v [T, ldv]:
 * y_ref[t, n] = y0[t, y_offset + n] + s_i * sum_{k < r_i} B_i[n, k] * v[t, k].
 */
int oracle_lora_expand(int dtype, int64_t T, int64_t o,
                       const float *v, int64_t ldv,
                       const void *y0, int64_t ldy, int64_t y_offset,
                       const int32_t *ids, int32_t n_adapters,
                       const void *const *B, const int32_t *ranks, const double *scales,
                       double *y_ref, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters))
        return -1;
    set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *yr = y_ref + t * o;
        for (int64_t n = 0; n < o; ++n)
            yr[n] = widen(y0, dtype, t * ldy + y_offset + n);
        int32_t i = ids[t];
        if (i < 0)
            continue;
        int32_t r = ranks[i];
        for (int64_t n = 0; n < o; ++n) {
            double acc = 0.0;
            for (int32_t k = 0; k < r; ++k)
                acc += widen(B[i], dtype, n * r + k) * (double)v[t * ldv + k];
            yr[n] += scales[i] * acc;
        }
    }
    return 0;
}

/*
 * Three-stage form of the "Compress then Serve" review thread (authors' rebuttal on Punica,
 * pseudocode of add_lora_slice_with_sigma): step 1 applies A_i to x with scale 1 into a
 * buffer of width R, step 2 applies the adapter's small matrix Sigma_i to that buffer with
 * scale 1, step 3 applies B_i with the adapter scale and updates the y slice:
 *
 *   u[k]        = sum_j x[t, j] * A_i[k, j]                       k < r_i
 *   w[k]        = sum_m Sigma_i[k, m] * u[m]        (sigma_kind 1: r_i x r_i, row-major)
 *               = Sigma_i[k] * u[k]                 (sigma_kind 2: diagonal, r_i values)
 *               = u[k]                              (sigma_kind 0: no Sigma)
 *   y_ref[t, n] = y0[t, y_offset + n] + s_i * sum_k B_i[n, k] * w[k]
 *
 * Sigma[i] points to fp32 values (widened exactly).  The pages name the two Sigma shapes
 * JD-Full and JD-Diag; where the adapters of one cluster share A and B, the caller passes
 * the same A / B pointer for each of them.  Other arguments as oracle_lora_delta.
 */
static void sigma_step(int sigma_kind, const float *S, int32_t r, const double *u, double *w)
{
    for (int32_t k = 0; k < r; ++k) {
        if (sigma_kind == 1) {
            double acc = 0.0;
            for (int32_t m = 0; m < r; ++m)
                acc += (double)S[(int64_t)k * r + m] * u[m];
            w[k] = acc;
        } else if (sigma_kind == 2) {
            w[k] = (double)S[k] * u[k];
        } else {
            w[k] = u[k];
        }
    }
}

int oracle_lora_delta_sigma(int dtype, int64_t T, int64_t h, int64_t o,
                            const void *x, int64_t ldx,
                            const void *y0, int64_t ldy, int64_t y_offset,
                            const int32_t *ids, int32_t n_adapters,
                            const void *const *A, const void *const *B,
                            const int32_t *ranks, const double *scales,
                            int sigma_kind, const float *const *Sigma,
                            double *y_ref, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters) || sigma_kind < 0 || sigma_kind > 2)
        return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *u = NULL, *w = NULL;
        int32_t cap = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *yr = y_ref + t * o;
            for (int64_t n = 0; n < o; ++n)
                yr[n] = widen(y0, dtype, t * ldy + y_offset + n);
            int32_t i = ids[t];
            if (i < 0)
                continue;
            int32_t r = ranks[i];
            if (r > cap) {
                free(u);
                free(w);
                u = (double *)malloc((size_t)r * sizeof(double));
                w = (double *)malloc((size_t)r * sizeof(double));
                cap = r;
            }
            /* step 1: u = A_i x, scale 1 */
            for (int32_t k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int64_t j = 0; j < h; ++j)
                    acc += widen(x, dtype, t * ldx + j) * widen(A[i], dtype, (int64_t)k * h + j);
                u[k] = acc;
            }
            /* step 2: w = Sigma_i u, scale 1 */
            sigma_step(sigma_kind, sigma_kind ? Sigma[i] : NULL, r, u, w);
            /* step 3: y += s_i * B_i w */
            for (int64_t n = 0; n < o; ++n) {
                double acc = 0.0;
                for (int32_t k = 0; k < r; ++k)
                    acc += widen(B[i], dtype, n * r + k) * w[k];
                yr[n] += scales[i] * acc;
            }
        }
        free(u);
        free(w);
    }
    return 0;
}

/*
 * Steps 1 and 2 of the three-stage form: v[t, k] = (Sigma_i (A_i x[t]))[k] for k < r_i;
 * v is [T, ldv] doubles, other entries 0.  Arguments as oracle_lora_shrink plus Sigma.
 */
int oracle_lora_shrink_sigma(int dtype, int64_t T, int64_t h,
                             const void *x, int64_t ldx,
                             const int32_t *ids, int32_t n_adapters,
                             const void *const *A, const int32_t *ranks,
                             int sigma_kind, const float *const *Sigma,
                             double *v, int64_t ldv, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters) || sigma_kind < 0 || sigma_kind > 2)
        return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *u = (double *)malloc((size_t)(ldv > 0 ? ldv : 1) * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *vr = v + t * ldv;
            for (int64_t k = 0; k < ldv; ++k)
                vr[k] = 0.0;
            int32_t i = ids[t];
            if (i < 0)
                continue;
            int32_t r = ranks[i];
            for (int32_t k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int64_t j = 0; j < h; ++j)
                    acc += widen(x, dtype, t * ldx + j) * widen(A[i], dtype, (int64_t)k * h + j);
                u[k] = acc;
            }
            sigma_step(sigma_kind, sigma_kind ? Sigma[i] : NULL, r, u, vr);
        }
        free(u);
    }
    return 0;
}

/*
 * Several adapters merged per token ("Lorax" pages: adapters merged per request into an
 * ensemble with weighted merge strategies).  Reading: the merge is the weighted sum of the
 * adapters' deltas,
 *
 *   y_ref[t, n] = y0[t, y_offset + n] + sum_{j < K, i = ids[t, j] >= 0} w[t, j] * s_i * (B_i (A_i x[t]))[n]
 *
 * ids and w are [T, K] row-major (K slots per token, id -1 = empty slot); w is fp32,
 * widened exactly.  Other arguments as oracle_lora_delta.  Returns -1 for an id outside
 * [-1, n_adapters).
 */
int oracle_lora_delta_merged(int dtype, int64_t T, int64_t h, int64_t o,
                             const void *x, int64_t ldx,
                             const void *y0, int64_t ldy, int64_t y_offset,
                             int32_t K, const int32_t *ids, const float *w, int32_t n_adapters,
                             const void *const *A, const void *const *B,
                             const int32_t *ranks, const double *scales,
                             double *y_ref, int n_threads)
{
    if (K < 1 || !ids_valid(T * K, ids, n_adapters))
        return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *v = NULL;
        int32_t cap = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *yr = y_ref + t * o;
            for (int64_t n = 0; n < o; ++n)
                yr[n] = widen(y0, dtype, t * ldy + y_offset + n);
            for (int32_t j = 0; j < K; ++j) {
                int32_t i = ids[t * K + j];
                if (i < 0)
                    continue;
                int32_t r = ranks[i];
                if (r > cap) {
                    free(v);
                    v = (double *)malloc((size_t)r * sizeof(double));
                    cap = r;
                }
                for (int32_t k = 0; k < r; ++k) {
                    double acc = 0.0;
                    for (int64_t jj = 0; jj < h; ++jj)
                        acc += widen(x, dtype, t * ldx + jj) * widen(A[i], dtype, (int64_t)k * h + jj);
                    v[k] = acc;
                }
                double wt = (double)w[t * K + j];
                for (int64_t n = 0; n < o; ++n) {
                    double acc = 0.0;
                    for (int32_t k = 0; k < r; ++k)
                        acc += widen(B[i], dtype, n * r + k) * v[k];
                    yr[n] += wt * (scales[i] * acc);
                }
            }
        }
        free(v);
    }
    return 0;
}

/*
 * Segment bookkeeping: a stable counting sort of the tokens by adapter id.
 *   perm[p]          token index at sorted position p (p < number of tokens with an adapter)
 *   seg_ptr[s]       first sorted position of segment s; seg_ptr[num_segs] = valid tokens
 *   seg_adapter[s]   adapter of segment s, strictly ascending
 * perm needs T entries, seg_ptr n_adapters + 1, seg_adapter n_adapters.
 * Returns the number of tokens with an adapter, or -1 for an out-of-range id.
 */
int64_t oracle_build_segments(int64_t T, const int32_t *ids, int32_t n_adapters,
                              int32_t *perm, int32_t *seg_ptr, int32_t *seg_adapter,
                              int32_t *num_segs)
{
    if (!ids_valid(T, ids, n_adapters))
        return -1;
    int64_t *count = (int64_t *)calloc((size_t)n_adapters + 1, sizeof(int64_t));
    int64_t *next = (int64_t *)calloc((size_t)n_adapters + 1, sizeof(int64_t));
    for (int64_t t = 0; t < T; ++t)
        if (ids[t] >= 0)
            count[ids[t]] += 1;
    int32_t S = 0;
    int64_t pos = 0;
    for (int32_t i = 0; i < n_adapters; ++i) {
        next[i] = pos;
        if (count[i] > 0) {
            seg_adapter[S] = i;
            seg_ptr[S] = (int32_t)pos;
            ++S;
        }
        pos += count[i];
    }
    seg_ptr[S] = (int32_t)pos;
    for (int64_t t = 0; t < T; ++t)
        if (ids[t] >= 0)
            perm[next[ids[t]]++] = (int32_t)t;
    *num_segs = S;
    free(count);
    free(next);
    return pos;
}

/*
 * Layer output with the frozen base weight: the "TGI Multi-LoRA" page ("Technical
 * Foundation: LoRA") keeps the pretrained weight W frozen and adds the adapter's low-rank
 * term, so one layer computes W x + s_i B_i A_i x; the "predibase/lorax" repository page
 * describes the adapter update as part of a single forward pass of the layer.
 *
 *   y_ref[t, n] = (accumulate ? y0[t, y_offset + n] : 0)
 *               + sum_j W[n, j] * x[t, j]                          (base product)
 *               + s_i * sum_k B_i[n, k] * v[k],  v[k] = sum_j x[t, j] * A_i[k, j]
 *
 * for i = ids[t]; a token with id -1 gets the first two terms only.  W is [o, ldw] row-major
 * (an output feature per row, the first h columns used), the orientation of a linear
 * layer's weight.  Terms are added in the order written, in fp64, unrounded.
 * Returns 0, or -1 if an id is out of range (nothing is written then).
 */
int oracle_lora_base_delta(int dtype, int64_t T, int64_t h, int64_t o,
                           const void *x, int64_t ldx,
                           const void *W, int64_t ldw,
                           const void *y0, int64_t ldy, int64_t y_offset, int accumulate,
                           const int32_t *ids, int32_t n_adapters,
                           const void *const *A, const void *const *B,
                           const int32_t *ranks, const double *scales,
                           double *y_ref, int n_threads)
{
    if (!ids_valid(T, ids, n_adapters))
        return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *xr = (double *)malloc((size_t)h * sizeof(double));
        double *u = NULL;
        int32_t ucap = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < T; ++t) {
            double *yr = y_ref + t * o;
            for (int64_t j = 0; j < h; ++j)
                xr[j] = widen(x, dtype, t * ldx + j);
            for (int64_t n = 0; n < o; ++n)
                yr[n] = accumulate ? widen(y0, dtype, t * ldy + y_offset + n) : 0.0;
            /* base product: y += W x */
            for (int64_t n = 0; n < o; ++n) {
                double acc = 0.0;
                for (int64_t j = 0; j < h; ++j)
                    acc += widen(W, dtype, n * ldw + j) * xr[j];
                yr[n] += acc;
            }
            int32_t i = ids[t];
            if (i < 0)
                continue;
            const int32_t ri = ranks[i];
            if (ri > ucap) {
                free(u);
                u = (double *)malloc((size_t)ri * sizeof(double));
                ucap = ri;
            }
            /* adapter shrink: u = A_i x  (scale 1) */
            for (int32_t m = 0; m < ri; ++m) {
                double su = 0.0;
                for (int64_t j = 0; j < h; ++j)
                    su += xr[j] * widen(A[i], dtype, (int64_t)m * h + j);
                u[m] = su;
            }
            /* adapter expand: y += s_i * B_i u */
            for (int64_t n = 0; n < o; ++n) {
                double sd = 0.0;
                for (int32_t m = 0; m < ri; ++m)
                    sd += widen(B[i], dtype, n * ri + m) * u[m];
                yr[n] += scales[i] * sd;
            }
        }
        free(u);
        free(xr);
    }
    return 0;
}
