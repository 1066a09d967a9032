// km_fit_small.cuh -- a whole exact Lloyd fit in one cooperative launch, for small problems.
//
// Small problems (config 1's N = 4096 points, K = 32, d = 16) are launch-bound: the step-by-step
// fit spends its time starting seven small kernels per iteration. Here the CTAs of one launch
// (all resident: a cooperative launch) run every iteration themselves. Each CTA owns 64 points
// of one batch element, four threads per point, and keeps them in registers for the whole fit;
// every CTA also keeps its own copy of its problem's centroids in shared memory. Per iteration:
//   1. each point's four threads scan a quarter of the centroids each, rounded to the points'
//      dtype (what the assignment of the step-by-step fit sees), with the direct form
//      sum_j (x_j - c_j)^2 in fp32, and combine their (distance, index) pairs so that the lowest
//      index wins ties (the CUDA-core assignment's arithmetic and rule);
//   2. the CTA sorts its 64 labels by cluster in shared memory (counts, a scan, member lists),
//      then each thread owns a few (cluster, component) entries and sums the weighted
//      coordinates, weights and counts of that cluster's members, adding the nonzero entries into
//      the iteration's accumulator in global memory;
//   3. grid barrier; every CTA reads the problem's totals and computes the new centroids itself
//      (the mean where the cluster has members and positive weight, the previous centroid
//      otherwise: the Lloyd update of the Flash-KMeans article, "Bottleneck 2", with empty
//      clusters kept), so no second barrier is needed before the next assignment.
// Three accumulators rotate: iteration t adds into A[t % 3], reads it after the barrier and
// clears A[(t + 2) % 3], which every CTA finished reading before that barrier.
// The barrier is a counter and a generation word in global memory, ordered by acquire-release
// operations rather than full fences; waits are bounded (the library's wait limit,
// globaltimer), and a timeout sets the device error word and an abort word that every CTA
// checks, so no CTA waits forever (km_debug_inject(2) makes CTA 0 skip its first arrival so
// that a test can watch this happen).
#pragma once

#include "km_common.cuh"

namespace km {
namespace fs {

constexpr int kThreads = 256;
constexpr int kSplit = 4;                    // threads per point
constexpr int kPts = kThreads / kSplit;      // points per CTA

struct Params {
    int B, N, K, d, P;        // P = CTAs per batch element
    int iters;
    const float *w;           // [B, N] or null
    float *C;                 // [B, K, d] fp32: initial centroids in, final centroids out
    int32_t *ids;             // [B, N] labels of the final centroids, or null
    double *inertia_hist;     // [iters, B] or null
    float *C_hist;            // [iters + 1, B, K, d] or null
    float *acc;               // [3, B, K, d + 2]: sums, weights, counts (zero at launch)
    double *iacc;             // [3, B] inertia (zero at launch)
    unsigned int *bar;        // [0] arrival count, [1] generation, [2] abort (zero at launch)
};

__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int *p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned int *p, unsigned int v) {
    asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned int *p, unsigned int v) {
    asm volatile("st.relaxed.gpu.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded grid barrier (all CTAs resident). Returns false once any CTA has given up.
// Thread 0 of each CTA arrives with an acquire-release add (after the CTA barrier, so it
// publishes the whole CTA's writes); the last to arrive resets the count and publishes the next
// generation with a release store, which the others read with acquire loads.
__device__ __forceinline__ bool grid_sync(unsigned int *bar, unsigned int nblocks, unsigned int &gen) {
    __shared__ int ok_s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        // test-only fault switch (off by default): CTA 0 never arrives at the first barrier
        const bool skip = gen == 0 && blockIdx.x == 0 && *reinterpret_cast<volatile int *>(&g_km_inject) == 2;
        if (!skip && atom_add_acq_rel_gpu(bar, 1u) == nblocks - 1) {
            st_relaxed_gpu(bar, 0u);          // ordered before the release below
            st_release_gpu(bar + 1, gen + 1);   // release the others
        } else {
            const unsigned long long t0 = globaltimer_ns();
            const unsigned long long limit =
                *reinterpret_cast<volatile unsigned long long *>(&g_km_wait_limit_ns);
            while (ld_acquire_gpu(bar + 1) == gen) {
                if (*reinterpret_cast<volatile unsigned int *>(bar + 2)) { ok = 0; break; }
                if (globaltimer_ns() - t0 > limit) {
                    record_dev_error(kDevErrTimeout);
                    atomicExch(bar + 2, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        ok_s = ok && *reinterpret_cast<volatile unsigned int *>(bar + 2) == 0;
    }
    __syncthreads();
    ++gen;
    return ok_s != 0;
}

// DM = the largest d this instantiation takes (a point is held as DM registers per thread).
template <typename T, int DM>
__global__ void __launch_bounds__(kThreads) fit_small_kernel(const T *__restrict__ X, const Params p) {
    extern __shared__ float fsm[];
    const int K = p.K, d = p.d;
    const int KD = K * d, E = K * (d + 2);
    float *cm = fsm;               // [K, d] the centroids (fp32)
    float *cs = cm + KD;           // [K, d] the same, rounded to T
    float *xs = cs + KD;           // [kPts, d] this CTA's points
    float *wsm = xs + kPts * d;    // [kPts] their weights (0 past N)
    int *lab = reinterpret_cast<int *>(wsm + kPts);   // [kPts] their labels
    int *mem = lab + kPts;         // [kPts] the points sorted by cluster
    int *off = mem + kPts;         // [K + 1] the clusters' member counts, then their offsets
    __shared__ double red[kThreads / 32];
    const int b = blockIdx.x / p.P, q = blockIdx.x % p.P;
    const int tid = threadIdx.x, lane = tid & 31;
    const int pt = tid / kSplit, sub = tid % kSplit;
    const int i = q * kPts + pt;
    const bool valid = i < p.N;
    float x[DM];
#pragma unroll
    for (int j = 0; j < DM; ++j)
        x[j] = valid && j < d ? Cvt<T>::to_f(X[(static_cast<int64_t>(b) * p.N + i) * d + j]) : 0.f;
    const float wi = valid ? (p.w ? p.w[static_cast<int64_t>(b) * p.N + i] : 1.f) : 0.f;
    if (sub == 0) {
#pragma unroll
        for (int j = 0; j < DM; ++j)
            if (j < d) xs[pt * d + j] = x[j];
        wsm[pt] = wi;
    }
    float *Cb = p.C + static_cast<int64_t>(b) * KD;
    for (int e = tid; e < KD; e += kThreads) {
        const float c = Cb[e];
        cm[e] = c;
        cs[e] = Cvt<T>::to_f(Cvt<T>::from_f(c));
    }
    __syncthreads();
    const unsigned int nblocks = gridDim.x;
    unsigned int gen = 0;
    // the nearest centroid of this thread's point: each of the four threads takes every fourth
    // centroid, then the pairs (distance, index) combine with the lower index winning ties
    auto nearest = [&](float &best) -> int {
        best = INFINITY;
        int bi = 0x7fffffff;
        for (int k = sub; k < K; k += kSplit) {
            const float *c = cs + k * d;
            float a = 0.f;
#pragma unroll
            for (int j = 0; j < DM; ++j)
                if (j < d) {
                    const float t = x[j] - c[j];
                    a = fmaf(t, t, a);
                }
            if (a < best) {
                best = a;
                bi = k;
            }
        }
#pragma unroll
        for (int o = 1; o < kSplit; o <<= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ob < best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        return bi;
    };
    for (int t = 0; t < p.iters; ++t) {
        if (p.C_hist && q == 0)
            for (int e = tid; e < KD; e += kThreads) p.C_hist[(static_cast<int64_t>(t) * p.B + b) * KD + e] = cm[e];
        float best;
        const int bi = nearest(best);
        for (int k = tid; k <= K; k += kThreads) off[k] = 0;
        double contrib = (sub == 0 && valid) ? static_cast<double>(wi) * static_cast<double>(best) : 0.0;
        contrib = warp_sum(contrib);
        if (lane == 0) red[tid >> 5] = contrib;
        __syncthreads();
        // counting sort of the CTA's labels: rank within the cluster, member counts, offsets
        int rank = 0;
        if (sub == 0 && valid) rank = atomicAdd(&off[bi], 1);
        __syncthreads();
        if (tid < 32) {   // exclusive scan of the K counts by one warp
            int carry = 0;
            for (int k0 = 0; k0 < K; k0 += 32) {
                const int v = k0 + lane < K ? off[k0 + lane] : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (k0 + lane < K) off[k0 + lane] = carry + incl - v;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) off[K] = carry;
        }
        __syncthreads();
        if (sub == 0 && valid) mem[off[bi] + rank] = pt;
        __syncthreads();
        // this CTA's sums, weights and counts, entry (k, j) by entry, added to A[t % 3]
        float *A = p.acc + (static_cast<int64_t>(t % 3) * p.B + b) * E;
        for (int e = tid; e < E; e += kThreads) {
            const int k = e / (d + 2), j = e - k * (d + 2);
            const int m0 = off[k], m1 = off[k + 1];
            if (m0 == m1) continue;
            float s = 0.f;
            for (int m = m0; m < m1; ++m) {
                const int r = mem[m];
                s += j < d ? wsm[r] * xs[r * d + j] : (j == d ? wsm[r] : 1.f);
            }
            atomicAdd(A + e, s);
        }
        if (tid == 0) {
            double s = 0.0;
            for (int r = 0; r < kThreads / 32; ++r) s += red[r];
            atomicAdd(p.iacc + (t % 3) * p.B + b, s);
        }
        if (!grid_sync(p.bar, nblocks, gen)) return;
        // the new centroids, computed by every CTA of the problem from the totals
        for (int e = tid; e < KD; e += kThreads) {
            const int k = e / d, j = e - k * d;
            // read at L2 (__ldcg): this SM may hold the buffer's lines from three iterations ago
            const float wsum = __ldcg(A + k * (d + 2) + d), cnt = __ldcg(A + k * (d + 2) + d + 1);
            const float div = p.w ? wsum : cnt;
            if (cnt > 0.f && div > 0.f) cm[e] = __ldcg(A + k * (d + 2) + j) / div;
            cs[e] = Cvt<T>::to_f(Cvt<T>::from_f(cm[e]));
        }
        if (p.inertia_hist && q == 0 && tid == 0)
            p.inertia_hist[static_cast<int64_t>(t) * p.B + b] = __ldcg(p.iacc + (t % 3) * p.B + b);
        // clear the accumulator of iteration t + 2 (everyone read it before this barrier)
        float *Z = p.acc + (static_cast<int64_t>((t + 2) % 3) * p.B + b) * E;
        for (int e = q * kThreads + tid; e < E; e += p.P * kThreads) Z[e] = 0.f;
        if (q == 0 && tid == 0) p.iacc[((t + 2) % 3) * p.B + b] = 0.0;
        __syncthreads();
    }
    if (q == 0)
        for (int e = tid; e < KD; e += kThreads) {
            Cb[e] = cm[e];
            if (p.C_hist) p.C_hist[(static_cast<int64_t>(p.iters) * p.B + b) * KD + e] = cm[e];
        }
    if (p.ids) {
        float best;
        const int bi = nearest(best);
        if (sub == 0 && valid) p.ids[static_cast<int64_t>(b) * p.N + i] = bi;
    }
}

}  // namespace fs
}  // namespace km
