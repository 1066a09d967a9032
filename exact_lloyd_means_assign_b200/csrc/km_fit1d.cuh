// km_fit1d.cuh -- weighted 1-D Lloyd for per-row codebooks, and the uniform-grid init.
//
// The LeanQuant issue "1D k-means" fits a small codebook (K = 8 or 16) to every row of a weight
// matrix with per-weight sample_weight, each row independently (a Pool over rows calling sklearn
// KMeans), with the initial centroids np.linspace(row.min(), row.max(), K). Here one CTA owns one
// row for all iterations and the row never leaves shared memory:
//
//   1. the row's values (exact fp32 copies of the stored values) are sorted once, carrying the
//      original index, and the weights are gathered into sorted order;
//   2. per iteration, the centroids (rounded to the row's dtype, like every assignment path) are
//      ranked by (value, index). In one dimension each cluster of the assignment is a contiguous
//      range of the sorted row, so the assignment is fully described by K boundaries: boundary q
//      is the number of points whose nearest centroid (exact argmin over all K of the fp32
//      (x - c)^2, lowest index on ties) has rank <= q, found by binary search over the sorted row;
//   3. the per-cluster weight sums, weighted value sums and the inertia are accumulated over
//      those ranges (fp64), and the centroids are updated (empty clusters keep theirs).
// The result is the same assignment a per-point argmin gives, except where two distances are
// within rounding of each other; cost per iteration is O(K log N + N) instead of O(N K).
#pragma once

#include "km_common.cuh"

namespace km {
namespace fit1d {

constexpr int THREADS = 256;
constexpr int KMAX = 64;
constexpr int NMAX = 8192;

// Grid init, one block per row: lo/hi reduction, then numpy linspace semantics in fp64.
template <typename T>
__global__ void __launch_bounds__(256)
    grid_init_kernel(const T *__restrict__ X, int N, int K, float *__restrict__ C) {
    __shared__ float smin[8], smax[8];
    const int b = blockIdx.x, tid = threadIdx.x;
    const T *xb = X + static_cast<int64_t>(b) * N;
    float lo = INFINITY, hi = -INFINITY;
    for (int i = tid; i < N; i += blockDim.x) {
        const float v = Cvt<T>::to_f(xb[i]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((tid & 31) == 0) {
        smin[tid >> 5] = lo;
        smax[tid >> 5] = hi;
    }
    __syncthreads();
    lo = smin[0];
    hi = smax[0];
    for (int wi = 1; wi < static_cast<int>(blockDim.x >> 5); ++wi) {
        lo = fminf(lo, smin[wi]);
        hi = fmaxf(hi, smax[wi]);
    }
    const double dlo = lo, dhi = hi;
    for (int k = tid; k < K; k += blockDim.x) {
        double v;
        if (K == 1) {
            v = dlo;
        } else if (k == K - 1) {
            v = dhi;
        } else {
            const double step = __ddiv_rn(__dsub_rn(dhi, dlo), static_cast<double>(K - 1));
            v = __dadd_rn(__dmul_rn(static_cast<double>(k), step), dlo);
        }
        C[static_cast<int64_t>(b) * K + k] = __double2float_rn(v);
    }
}

__device__ __forceinline__ int nearest(float x, const float *cx, int K) {
    float best = INFINITY;
    int bi = 0;
    for (int k = 0; k < K; ++k) {
        const float t = x - cx[k];
        const float dd = t * t;
        if (dd < best) {
            best = dd;
            bi = k;
        }
    }
    return bi;
}

// Shared memory: NP floats (sorted values), NP ints (original index), NP floats (weights).
template <typename T>
__global__ void __launch_bounds__(THREADS)
    fit1d_kernel(const T *__restrict__ X, const float *__restrict__ w, int B, int N, int NP, int K,
                 int iters, float *__restrict__ C, int32_t *__restrict__ ids,
                 double *__restrict__ inertia_hist, float *__restrict__ C_hist) {
    extern __shared__ uint8_t sm[];
    float *xs = reinterpret_cast<float *>(sm);
    int *is = reinterpret_cast<int *>(xs + NP);
    float *ws = reinterpret_cast<float *>(is + NP);
    __shared__ float cm[KMAX];      // fp32 master centroids
    __shared__ float cx[KMAX];      // rounded to T: what the assignment compares against
    __shared__ int rank_of[KMAX];   // rank of centroid k in (cx, k) order
    __shared__ int order[KMAX];     // centroid at each rank
    __shared__ int E[KMAX];         // E[q] = #points whose nearest centroid has rank <= q
    __shared__ double sw[KMAX], swx[KMAX];
    __shared__ double red[THREADS / 32];

    const int b = blockIdx.x, tid = threadIdx.x;
    const T *xb = X + static_cast<int64_t>(b) * N;
    for (int p = tid; p < NP; p += THREADS) {
        xs[p] = p < N ? Cvt<T>::to_f(xb[p]) : INFINITY;
        is[p] = p < N ? p : -1;
    }
    if (tid < K) {
        cm[tid] = C[static_cast<int64_t>(b) * K + tid];
        if (C_hist) C_hist[static_cast<int64_t>(b) * K + tid] = cm[tid];
    }
    __syncthreads();

    // bitonic sort of (value, index) pairs, ascending
    for (int k = 2; k <= NP; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = tid; t < (NP >> 1); t += THREADS) {
                const int i = 2 * j * (t / j) + (t % j);
                const int ixj = i + j;
                const bool asc = (i & k) == 0;
                const float a = xs[i], c = xs[ixj];
                if ((a > c) == asc) {
                    xs[i] = c;
                    xs[ixj] = a;
                    const int ti = is[i];
                    is[i] = is[ixj];
                    is[ixj] = ti;
                }
            }
            __syncthreads();
        }
    }
    for (int p = tid; p < N; p += THREADS)
        ws[p] = w ? w[static_cast<int64_t>(b) * N + is[p]] : 1.f;
    __syncthreads();

    for (int t = 0; t <= iters; ++t) {
        const bool final_pass = (t == iters);
        if (final_pass && !ids) break;
        if (tid < K) cx[tid] = round_through<T>(cm[tid]);
        __syncthreads();
        if (tid < K) {
            const float v = cx[tid];
            int r = 0;
            for (int j = 0; j < K; ++j) {
                const float u = cx[j];
                r += (u < v) || (u == v && j < tid);
            }
            rank_of[tid] = r;
            order[r] = tid;
            sw[tid] = 0.0;
            swx[tid] = 0.0;
        }
        __syncthreads();
        if (tid < K - 1) {
            int lo = 0, hi = N;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (rank_of[nearest(xs[mid], cx, K)] <= tid) lo = mid + 1; else hi = mid;
            }
            E[tid] = lo;
        } else if (tid == K - 1) {
            E[tid] = N;
        }
        __syncthreads();
        if (final_pass) {
            for (int p = tid; p < N; p += THREADS) {
                int qq = 0;
                while (E[qq] <= p) ++qq;
                ids[static_cast<int64_t>(b) * N + is[p]] = order[qq];
            }
            break;
        }
        // per-cluster sums over contiguous sorted ranges; each thread walks its own chunk
        double iner = 0.0;
        {
            const int per = (N + THREADS - 1) / THREADS;
            int p = tid * per;
            const int pend = min(N, p + per);
            if (p < pend) {
                int qq = 0;
                while (E[qq] <= p) ++qq;
                double aw = 0.0, awx = 0.0;
                for (; p < pend; ++p) {
                    while (E[qq] <= p) {
                        atomicAdd(&sw[qq], aw);
                        atomicAdd(&swx[qq], awx);
                        aw = 0.0;
                        awx = 0.0;
                        ++qq;
                    }
                    const float x = xs[p], wt = ws[p];
                    const float dx = x - cx[order[qq]];
                    aw += wt;
                    awx += static_cast<double>(wt) * x;
                    iner += static_cast<double>(wt) * static_cast<double>(dx * dx);
                }
                atomicAdd(&sw[qq], aw);
                atomicAdd(&swx[qq], awx);
            }
        }
        iner = warp_sum(iner);
        if ((tid & 31) == 0) red[tid >> 5] = iner;
        __syncthreads();
        if (tid == 0 && inertia_hist) {
            double s = 0.0;
            for (int i = 0; i < THREADS / 32; ++i) s += red[i];
            inertia_hist[static_cast<int64_t>(t) * B + b] = s;
        }
        if (tid < K) {
            const int qq = rank_of[tid];
            const int cnt = E[qq] - (qq ? E[qq - 1] : 0);
            const double W = sw[qq];
            if (cnt > 0 && W > 0.0) cm[tid] = __double2float_rn(__ddiv_rn(swx[qq], W));
            if (C_hist) C_hist[(static_cast<int64_t>(t + 1) * B + b) * K + tid] = cm[tid];
        }
        __syncthreads();
    }
    if (tid < K) C[static_cast<int64_t>(b) * K + tid] = cm[tid];
}

}  // namespace fit1d
}  // namespace km
