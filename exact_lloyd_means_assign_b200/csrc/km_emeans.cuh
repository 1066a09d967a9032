// km_emeans.cuh -- the e-means moving-average update and proportional splitting of dead clusters.
//
// The steinslab daily on e-means ("Beating 25 Lloyd Iterations in 2 Epochs") keeps, per cluster,
// a sum vector S_j and a count N_j whose quotient is the centroid, and replaces Lloyd's reset of
// both on every pass by an exponential moving average over mini-batches, S_j <- (1 - a) S_j +
// a s_j (section "Breaking 70 Years of Full-Batch Inertia..."; the count gets the same average).
// Clusters left without points are revived by splitting large clusters, donors drawn in
// proportion to their size (section "Proportional Splitting Resurrects Thousands of Dead
// Centers"). The assignment and the per-batch statistics s_j, n_j come from the assignment
// kernels and the sort-inverse update; the kernels here only fold them into the state.
#pragma once

#include "km_common.cuh"

namespace km {
namespace em {

__global__ void fill_f32_kernel(float *__restrict__ p, float v, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) p[i] = v;
}

__global__ void i32_to_f32_kernel(const int32_t *__restrict__ src, float *__restrict__ dst, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = static_cast<float>(src[i]);
}

// One warp per cluster row (b, k). The batch's sums s and size n (point count, or weight sum
// when `wsum` is given) enter the moving averages
//     S <- (1 - a) S + a s,   Nc <- (1 - a) Nc + a n,   C = S / Nc  (C kept when Nc == 0),
// Cx / cn (the rounded centroids and their squared norms for the next assignment) are rewritten,
// and, when eS is given, the batch statistics are added to the epoch totals (eS, eCnt, eW).
template <typename T>
__global__ void ema_kernel(const float *__restrict__ s, const int32_t *__restrict__ cnt,
                           const float *__restrict__ wsum, float alpha, int64_t rows, int d,
                           float *__restrict__ S, float *__restrict__ Nc, float *__restrict__ C,
                           T *__restrict__ Cx, float *__restrict__ cn, float *__restrict__ eS,
                           int32_t *__restrict__ eCnt, float *__restrict__ eW) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float a1 = 1.f - alpha;
    const float n = wsum ? wsum[row] : static_cast<float>(cnt[row]);
    const float nn = a1 * Nc[row] + alpha * n;
    float sq = 0.f;
    for (int j = lane; j < d; j += 32) {
        const int64_t e = row * d + j;
        const float sv = s[e];
        const float Sv = a1 * S[e] + alpha * sv;
        S[e] = Sv;
        const float c = nn > 0.f ? Sv / nn : C[e];
        C[e] = c;
        const T t = Cvt<T>::from_f(c);
        Cx[e] = t;
        const float f = Cvt<T>::to_f(t);
        sq = fmaf(f, f, sq);
        if (eS) eS[e] += sv;
    }
    sq = warp_sum(sq);
    if (lane == 0) {
        Nc[row] = nn;
        cn[row] = sq;
        if (eS) {
            eCnt[row] += cnt[row];
            if (eW) eW[row] += wsum[row];
        }
    }
}

// Proportional splitting, one block per problem. The clusters whose size is 0 are revived in
// index order; dead cluster i takes as donor the first cluster j whose running size sum exceeds
// u[i] * (total size), evaluated in fp64. Then, per coordinate k with s_k = +1 for even k and -1
// for odd k, c_i = c_j (1 + eps s_k) and c_j <- c_j (1 - eps s_k); sizes and (when given) the
// moving-average counts Nc are halved between the two, and S (when given) is set to C * Nc on
// both rows. A dead cluster never becomes a donor (its size is 0) and a donor stays alive, so the
// dead set is fixed at entry. donors[i] receives j (or -1 for clusters that were alive).
constexpr int SPLIT_THREADS = 1024;

__global__ void __launch_bounds__(SPLIT_THREADS)
    split_kernel(float *__restrict__ sizes, const float *__restrict__ u, float eps, int K, int d,
                 float *__restrict__ C, float *__restrict__ Nc, float *__restrict__ S,
                 int32_t *__restrict__ donors) {
    constexpr int NW = SPLIT_THREADS / 32;
    __shared__ int dead_list[SPLIT_THREADS];
    __shared__ int ndead;
    __shared__ double wtot[NW];
    __shared__ int donor;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *sz = sizes + static_cast<int64_t>(b) * K;
    const float *ub = u + static_cast<int64_t>(b) * K;
    float *Cb = C + static_cast<int64_t>(b) * K * d;
    float *Nb = Nc ? Nc + static_cast<int64_t>(b) * K : nullptr;
    float *Sb = S ? S + static_cast<int64_t>(b) * K * d : nullptr;
    int32_t *db = donors ? donors + static_cast<int64_t>(b) * K : nullptr;
    const int per = (K + SPLIT_THREADS - 1) / SPLIT_THREADS;   // sizes owned per thread
    for (int base = 0; base < K; base += SPLIT_THREADS) {
        // the dead clusters of this range, in index order
        const int i0 = base + tid;
        const bool dead = i0 < K && sz[i0] == 0.f;
        if (db && i0 < K) db[i0] = -1;
        const unsigned m = __ballot_sync(0xffffffffu, dead);
        if (tid == 0) ndead = 0;
        __syncthreads();
        if (lane == 0) wtot[warp] = __popc(m);
        __syncthreads();
        int before = 0;
        for (int v = 0; v < warp; ++v) before += static_cast<int>(wtot[v]);
        if (dead) dead_list[before + __popc(m & ((1u << lane) - 1u))] = i0;
        if (tid == NW * 32 - 1) ndead = before + __popc(m);
        __syncthreads();
        const int nd = ndead;
        for (int q = 0; q < nd; ++q) {
            const int i = dead_list[q];
            // running sums of the sizes: thread t owns [t * per, t * per + per)
            const int k0 = min(K, tid * per), k1 = min(K, k0 + per);
            double loc = 0.0;
            for (int k = k0; k < k1; ++k) loc += sz[k];
            double inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double t = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += t;
            }
            __syncthreads();   // wtot reuse
            if (lane == 31) wtot[warp] = inc;
            if (tid == 0) donor = -1;
            __syncthreads();
            double total = 0.0, off = 0.0;
            for (int v = 0; v < NW; ++v) {
                if (v < warp) off += wtot[v];
                total += wtot[v];
            }
            if (total <= 0.0) break;   // block-uniform: nothing to split from
            const double target = static_cast<double>(ub[i]) * total;
            double run = off + inc - loc;   // exclusive prefix of this thread's range
            if (run <= target && run + loc > target) {
                for (int k = k0; k < k1; ++k) {
                    run += sz[k];
                    if (run > target) {
                        donor = k;
                        break;
                    }
                }
            }
            __syncthreads();
            int j = donor;
            if (j < 0) {   // rounding left the target at the total: the last cluster with mass
                if (tid == 0) {
                    for (int k = K - 1; k >= 0; --k)
                        if (sz[k] > 0.f) {
                            donor = k;
                            break;
                        }
                }
                __syncthreads();
                j = donor;
            }
            const float nj = Nb ? Nb[j] : 0.f;
            const float ni_new = 0.5f * nj, nj_new = nj - ni_new;
            for (int k = tid; k < d; k += SPLIT_THREADS) {
                const float c = Cb[static_cast<int64_t>(j) * d + k];
                const float sg = (k & 1) ? -eps : eps;
                const float ci = c * (1.f + sg), cj = c * (1.f - sg);
                Cb[static_cast<int64_t>(i) * d + k] = ci;
                Cb[static_cast<int64_t>(j) * d + k] = cj;
                if (Sb) {
                    Sb[static_cast<int64_t>(i) * d + k] = ci * ni_new;
                    Sb[static_cast<int64_t>(j) * d + k] = cj * nj_new;
                }
            }
            __syncthreads();   // every thread has read Nc[j] before it changes
            if (tid == 0) {
                const float si = 0.5f * sz[j];
                sz[i] = si;
                sz[j] -= si;
                if (Nb) {
                    Nb[i] = ni_new;
                    Nb[j] = nj_new;
                }
                if (db) db[i] = j;
            }
            __syncthreads();
        }
        __syncthreads();
    }
}

}  // namespace em
}  // namespace km
