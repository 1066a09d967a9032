// km_codebook1d.cuh -- 1-D codebooks: encoding values to uint8 indices, and k-means++ seeding.
//
// Encoding: the weight-clustering proposal reposted on wpnews.pro ("Cache-Aware Weight
// Clustering ...", its compressed-representation and 100-million-weight examples) stores every
// weight as the 8-bit index of its cluster's shared value. Here the index is the exact nearest
// centroid (centroids rounded to the values' dtype, fp32 squared distance, lowest index on
// ties), the same decision as the assignment kernels with d = 1, found by binary search in the
// sorted codebook instead of a scan over all K: in one dimension the distance can only grow
// moving away from the value on either side (the rounded difference and its square are
// monotone), so the minimum sits on one of the two centroids bracketing the value, and only
// centroids with exactly the same rounded distance can tie with it; those are found by walking
// outwards while the distance stays equal.
//
// k-means++ seeding: the LeanQuant issue "1D k-means" seeds rows with more than 8 clusters by
// k-means++ (its KMeans(init=...) line): the first centre is drawn in proportion to the sample
// weights, every next one in proportion to weight x squared distance to the nearest centre so
// far. Each draw uses its own uniform u (an input) and takes the first point whose running mass
// exceeds u x (total mass); with no mass left it takes point 0.
#pragma once

#include "km_common.cuh"

namespace km {
namespace cb {

constexpr int ENC_THREADS = 256;
constexpr int ENC_VPT = 16;     // values per thread per block
constexpr int ENC_KMAX = 256;   // 8-bit indices

template <typename T>
__global__ void __launch_bounds__(ENC_THREADS)
    encode1d_kernel(const T *__restrict__ X, int64_t N, const float *__restrict__ C, int K,
                    uint8_t *__restrict__ codes) {
    __shared__ float sv[2 * ENC_KMAX];   // rounded centroids, ascending by (value, index), then +inf
    __shared__ int si[ENC_KMAX];         // their indices
    const int b = blockIdx.y, tid = threadIdx.x;
    const float *Cb = C + static_cast<int64_t>(b) * K;
    int P = 1;   // the search runs over P > K entries, a power of two (so lo can reach K)
    while (P <= K) P <<= 1;
    for (int t = K + tid; t < P; t += ENC_THREADS) sv[t] = INFINITY;
    if (tid < K) {
        const float v = round_through<T>(Cb[tid]);
        int r = 0;
        for (int j = 0; j < K; ++j) {
            const float u = round_through<T>(Cb[j]);
            r += (u < v) || (u == v && j < tid);
        }
        sv[r] = v;
        si[r] = tid;
    }
    __syncthreads();
    const T *xb = X + static_cast<int64_t>(b) * N;
    uint8_t *ob = codes + static_cast<int64_t>(b) * N;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * (ENC_THREADS * ENC_VPT);
    // all of this thread's values are requested before any is encoded (one memory latency)
    T xr[ENC_VPT];
#pragma unroll
    for (int v = 0; v < ENC_VPT; ++v) {
        const int64_t i = base + static_cast<int64_t>(v) * ENC_THREADS + tid;
        xr[v] = i < N ? xb[i] : Cvt<T>::from_f(0.f);
    }
#pragma unroll
    for (int v = 0; v < ENC_VPT; ++v) {
        const int64_t i = base + static_cast<int64_t>(v) * ENC_THREADS + tid;
        if (i >= N) break;
        const float x = Cvt<T>::to_f(xr[v]);
        int lo = 0;   // number of sorted entries <= x (branch-free, log2 P steps)
        for (int step = P >> 1; step > 0; step >>= 1)
            if (sv[lo + step - 1] <= x) lo += step;
        const float tl = lo > 0 ? x - sv[lo - 1] : INFINITY;
        const float tr = lo < K ? x - sv[lo] : INFINITY;
        const float dl = tl * tl, dr = tr * tr;
        const float best = fminf(dl, dr);
        int idx = min(dl == best ? si[max(lo - 1, 0)] : K, dr == best ? si[min(lo, K - 1)] : K);
        // a third centroid can tie only with exactly the same rounded distance (rare)
        float t2 = lo > 1 ? x - sv[lo - 2] : INFINITY;
        float t3 = lo + 1 < K ? x - sv[lo + 1] : INFINITY;
        if (t2 * t2 == best || t3 * t3 == best) {
            for (int q = lo - 2; q >= 0; --q) {   // distances grow leftwards
                const float t = x - sv[q];
                if (t * t != best) break;
                idx = min(idx, si[q]);
            }
            for (int q = lo + 1; q < K; ++q) {    // and rightwards
                const float t = x - sv[q];
                if (t * t != best) break;
                idx = min(idx, si[q]);
            }
        }
        ob[i] = static_cast<uint8_t>(idx);
    }
}

constexpr int PP_THREADS = 512;
constexpr int PP_PER = 16;      // points per thread: rows of up to PP_THREADS * PP_PER values
constexpr int PP_NMAX = PP_THREADS * PP_PER;

// One block per row; thread t owns the contiguous points [t * per, t * per + per), so a block scan
// of the per-thread masses gives running sums in point order.
template <typename T>
__global__ void __launch_bounds__(PP_THREADS)
    kmeanspp1d_kernel(const T *__restrict__ X, const float *__restrict__ w, int N, int K,
                      const float *__restrict__ u, float *__restrict__ C,
                      int32_t *__restrict__ chosen) {
    constexpr int NW = PP_THREADS / 32;
    __shared__ double wtot[NW];
    __shared__ int pick, last_mass;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (N + PP_THREADS - 1) / PP_THREADS;
    const int p0 = min(N, tid * per);
    const int np = min(N, p0 + per) - p0;
    const int64_t rb = static_cast<int64_t>(b) * N;
    float xv[PP_PER], wv[PP_PER];
    double d2[PP_PER];
#pragma unroll
    for (int e = 0; e < PP_PER; ++e) {
        const bool in = e < np;
        xv[e] = in ? Cvt<T>::to_f(X[rb + p0 + e]) : 0.f;
        wv[e] = in ? (w ? w[rb + p0 + e] : 1.f) : 0.f;
        d2[e] = 1.0;   // the first draw is proportional to the weights alone
    }
    for (int k = 0; k < K; ++k) {
        double loc = 0.0;
        int mylast = -1;   // this thread's last point with mass
#pragma unroll
        for (int e = 0; e < PP_PER; ++e) {
            const double m = static_cast<double>(wv[e]) * d2[e];
            loc += m;
            if (e < np && m > 0.0) mylast = p0 + e;
        }
        double inc = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (lane == 31) wtot[warp] = inc;
        if (tid == 0) {
            pick = -1;
            last_mass = -1;
        }
        __syncthreads();
        if (mylast >= 0) atomicMax(&last_mass, mylast);
        double total = 0.0, off = 0.0;
        for (int v = 0; v < NW; ++v) {
            if (v < warp) off += wtot[v];
            total += wtot[v];
        }
        if (total > 0.0) {
            const double target = static_cast<double>(u[static_cast<int64_t>(b) * K + k]) * total;
            double run = off + inc - loc;
            if (run <= target && run + loc > target) {
#pragma unroll
                for (int e = 0; e < PP_PER; ++e) {
                    const double m = static_cast<double>(wv[e]) * d2[e];
                    run += m;
                    if (e < np && m > 0.0 && run > target) {
                        pick = p0 + e;
                        break;
                    }
                }
            }
        }
        __syncthreads();
        // no mass left: point 0; rounding left the target at the total: the last point with mass
        if (tid == 0 && pick < 0) pick = last_mass >= 0 ? last_mass : 0;
        __syncthreads();
        const int i = pick;
        const float c = Cvt<T>::to_f(X[rb + i]);
        if (tid == 0) {
            C[static_cast<int64_t>(b) * K + k] = c;
            if (chosen) chosen[static_cast<int64_t>(b) * K + k] = i;
        }
#pragma unroll
        for (int e = 0; e < PP_PER; ++e) {
            const double t = static_cast<double>(xv[e]) - static_cast<double>(c);
            const double dd = t * t;
            d2[e] = (k == 0) ? dd : fmin(d2[e], dd);
        }
        __syncthreads();   // wtot and pick are rewritten by the next draw
    }
}

}  // namespace cb
}  // namespace km
