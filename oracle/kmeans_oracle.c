/*
 * kmeans_oracle.c -- plain fp64 CPU oracle for one exact Lloyd k-means iteration.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file's library. It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes, and where the pages define it:
 *   - Lloyd's iteration is two stages: each point goes to its nearest centroid,
 *     then each centroid becomes the mean of its points (technologypulse.uk,
 *     "Flash-KMeans" article, section "Flash-KMeans: same maths, new dataflow";
 *     wispaper.ai "Flash-KMeans" blog, Background). Flash-KMeans states its
 *     output is mathematically identical to standard Lloyd, so the oracle is that
 *     plain definition, written out with no tiling, fusion or reordering.
 *   - Each cluster keeps a sum vector S_j and a count N_j whose quotient is the
 *     centroid (steinslab "e-means" daily, first section). With per-point
 *     weights (LeanQuant issue "1D k-means", the kmeans_fit sample_weight
 *     argument) S_j = sum w_i x_i and the divisor is W_j = sum w_i.
 *   - Uniform-grid init: linspace(row min, row max, K) (LeanQuant issue
 *     "1D k-means", the diff of lean_quantizer.py and the follow-up comment).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - ties between equal distances go to the lowest centroid index;
 *   - an empty cluster (count 0, or total weight 0) keeps its previous centroid;
 *   - distances use the direct form sum_j (x_j - c_j)^2 in fp64;
 *   - d2 is the second-smallest distance over distinct centroid indices (it
 *     equals d1 when two centroids are at the same distance);
 *   - inertia is sum_i w_i * d1_i, the objective of the assignment just made.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math, no
 * FMA contraction, so every operation rounds as written).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int kmo_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Squared Euclidean distance between two d-vectors, direct form, fp64. */
static double sqdist(const double *x, const double *c, int64_t d)
{
    double s = 0.0;
    for (int64_t j = 0; j < d; ++j) {
        double t = x[j] - c[j];
        s += t * t;
    }
    return s;
}

/*
 * Assignment stage. X[B,N,d], C[B,K,d] (row-major, fp64), w[B,N] or NULL.
 * ids[B,N] receives argmin_k ||x - c_k||^2 (lowest k on ties); d1/d2 (may be
 * NULL) the best and second-best distances; inertia[B] (may be NULL) the
 * weighted sum of best distances, summed in point order.
 */
void kmo_assign(const double *X, const double *C, const double *w,
                int64_t B, int64_t N, int64_t K, int64_t d,
                int32_t *ids, double *d1, double *d2, double *inertia)
{
    for (int64_t b = 0; b < B; ++b) {
        const double *Xb = X + b * N * d;
        const double *Cb = C + b * K * d;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < N; ++i) {
            double best = INFINITY, second = INFINITY;
            int32_t bk = 0;
            for (int64_t k = 0; k < K; ++k) {
                double dist = sqdist(Xb + i * d, Cb + k * d, d);
                if (dist < best) {
                    second = best;
                    best = dist;
                    bk = (int32_t)k;
                } else if (dist < second) {
                    second = dist;
                }
            }
            ids[b * N + i] = bk;
            if (d1) d1[b * N + i] = best;
            if (d2) d2[b * N + i] = second;
        }
        if (inertia) {
            double s = 0.0;
            for (int64_t i = 0; i < N; ++i) {
                double wi = w ? w[b * N + i] : 1.0;
                double di = d1 ? d1[b * N + i] : sqdist(Xb + i * d, Cb + (int64_t)ids[b * N + i] * d, d);
                s += wi * di;
            }
            inertia[b] = s;
        }
    }
}

/*
 * Update stage, fed a given assignment ids[B,N]. counts[B,K] (int64) get the
 * member counts, wsum[B,K] (may be NULL) the member weight totals, and
 * C_new[B,K,d] the weighted means; a cluster with no member or zero total
 * weight keeps C_prev.
 */
void kmo_update(const double *X, const int32_t *ids, const double *w, const double *C_prev,
                int64_t B, int64_t N, int64_t K, int64_t d,
                double *C_new, int64_t *counts, double *wsum)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b) {
        double *S = (double *)calloc((size_t)(K * d), sizeof(double));
        double *W = (double *)calloc((size_t)K, sizeof(double));
        int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
        const double *Xb = X + b * N * d;
        for (int64_t i = 0; i < N; ++i) {
            int64_t k = ids[b * N + i];
            double wi = w ? w[b * N + i] : 1.0;
            cnt[k] += 1;
            W[k] += wi;
            for (int64_t j = 0; j < d; ++j) S[k * d + j] += wi * Xb[i * d + j];
        }
        for (int64_t k = 0; k < K; ++k) {
            double *out = C_new + (b * K + k) * d;
            const double *prev = C_prev + (b * K + k) * d;
            if (cnt[k] > 0 && W[k] > 0.0) {
                for (int64_t j = 0; j < d; ++j) out[j] = S[k * d + j] / W[k];
            } else {
                for (int64_t j = 0; j < d; ++j) out[j] = prev[j];
            }
            counts[b * K + k] = cnt[k];
            if (wsum) wsum[b * K + k] = W[k];
        }
        free(S);
        free(W);
        free(cnt);
    }
}

/*
 * Uniform-grid init of one 1-D row per batch: the same values as numpy's
 * linspace(min, max, K): step = (max - min) / (K - 1), c_k = k * step + min,
 * and the last value set to max exactly; K == 1 gives [min]. X[B,N] (d = 1).
 */
void kmo_grid_init(const double *X, int64_t B, int64_t N, int64_t K, double *C)
{
    for (int64_t b = 0; b < B; ++b) {
        double lo = X[b * N], hi = X[b * N];
        for (int64_t i = 1; i < N; ++i) {
            double v = X[b * N + i];
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        if (K == 1) {
            C[b * K] = lo;
            continue;
        }
        double step = (hi - lo) / (double)(K - 1);
        for (int64_t k = 0; k < K; ++k) C[b * K + k] = (double)k * step + lo;
        C[b * K + K - 1] = hi;
    }
}
