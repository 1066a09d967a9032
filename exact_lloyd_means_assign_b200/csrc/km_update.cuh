// km_update.cuh -- Sort-Inverse Update: argsort of the assignment vector, then a segmented
// reduction with one atomic merge per run (technologypulse.uk Flash-KMeans article,
// "Bottleneck 2"; wispaper blog "2. Sort-Inverse Update").
//
//   hist       per-tile histogram of ids in shared memory, merged into counts[B,K]
//   scan       per batch exclusive prefix of counts -> offsets[B,K+1], cursor[B,K]
//   scatter    counting-sort scatter: each tile reserves its slots per cluster with one atomic
//              on the cursor, then ranks its points in shared memory -> perm[B,N]; every
//              cluster's points end up in one contiguous segment [offsets[k], offsets[k+1])
//   segreduce  each warp walks a contiguous range of sorted positions, gathers X rows by index
//              (X itself is never permuted in memory), accumulates sum w*x and sum w in
//              registers while the cluster id stays the same, and merges each run into
//              sums[B,K,d] with vector atomics (red.global.add.v4.f32): one per run per
//              4-column group, i.e. O((K + N/range) * d) atomics instead of O(N * d).
//
// The order of points inside a segment is not fixed (tiles reserve their slots atomically), so
// fp32 sums may differ in the last bits from run to run; the set of points per segment, the
// counts and the offsets are exact.
#pragma once

#include <limits.h>

#include "km_common.cuh"

namespace km {
namespace upd {

constexpr int TILE = 8192;          // points per histogram / scatter tile
constexpr int TILE_THREADS = 512;
constexpr int SMEM_K_MAX = 16384;   // bins kept in shared memory
constexpr int SCAN_THREADS = 1024;
constexpr int SEG_THREADS = 256;

__global__ void __launch_bounds__(TILE_THREADS)
    hist_kernel(const int32_t *__restrict__ ids, int N, int K, int32_t *__restrict__ counts,
                int use_smem) {
    extern __shared__ int hsm[];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * TILE;
    const int t1 = min(N, t0 + TILE);
    const int32_t *idb = ids + static_cast<int64_t>(b) * N;
    int32_t *cb = counts + static_cast<int64_t>(b) * K;
    // ids outside [0, K) are not counted (and so never reach the reduction)
    if (use_smem) {
        for (int k = threadIdx.x; k < K; k += blockDim.x) hsm[k] = 0;
        __syncthreads();
        for (int i = t0 + threadIdx.x; i < t1; i += blockDim.x) {
            const int k = idb[i];
            if (static_cast<unsigned>(k) < static_cast<unsigned>(K)) atomicAdd(&hsm[k], 1);
        }
        __syncthreads();
        for (int k = threadIdx.x; k < K; k += blockDim.x)
            if (hsm[k]) atomicAdd(&cb[k], hsm[k]);
    } else {
        for (int i = t0 + threadIdx.x; i < t1; i += blockDim.x) {
            const int k = idb[i];
            if (static_cast<unsigned>(k) < static_cast<unsigned>(K)) atomicAdd(&cb[k], 1);
        }
    }
}

__global__ void __launch_bounds__(SCAN_THREADS)
    scan_kernel(const int32_t *__restrict__ counts, int K, int32_t *__restrict__ offsets,
                int32_t *__restrict__ cursor) {
    __shared__ int wtot[SCAN_THREADS / 32];
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int32_t *cb = counts + static_cast<int64_t>(b) * K;
    int32_t *ob = offsets + static_cast<int64_t>(b) * (K + 1);
    int32_t *cur = cursor + static_cast<int64_t>(b) * K;
    int carry = 0;
    for (int base = 0; base < K; base += 4 * SCAN_THREADS) {
        const int k0 = base + 4 * tid;
        int v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = (k0 + e < K) ? cb[k0 + e] : 0;
        const int tsum = v[0] + v[1] + v[2] + v[3];
        int incl = tsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wtot[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int x = wtot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            wtot[lane] = x;
        }
        __syncthreads();
        int ex = carry + incl - tsum + (wid > 0 ? wtot[wid - 1] : 0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (k0 + e < K) {
                ob[k0 + e] = ex;
                cur[k0 + e] = ex;
            }
            ex += v[e];
        }
        carry += wtot[SCAN_THREADS / 32 - 1];
        __syncthreads();
    }
    if (tid == 0) ob[K] = carry;
}

__global__ void __launch_bounds__(TILE_THREADS)
    scatter_kernel(const int32_t *__restrict__ ids, int N, int K, int32_t *__restrict__ cursor,
                   int32_t *__restrict__ perm, int use_smem) {
    extern __shared__ int ssm[];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * TILE;
    const int t1 = min(N, t0 + TILE);
    const int32_t *idb = ids + static_cast<int64_t>(b) * N;
    int32_t *cur = cursor + static_cast<int64_t>(b) * K;
    int32_t *pb = perm + static_cast<int64_t>(b) * N;
    if (use_smem) {
        int *h = ssm;
        int *tids = ssm + K;
        for (int k = threadIdx.x; k < K; k += blockDim.x) h[k] = 0;
        for (int i = t0 + threadIdx.x; i < t1; i += blockDim.x) tids[i - t0] = idb[i];
        __syncthreads();
        for (int i = threadIdx.x; i < t1 - t0; i += blockDim.x) {
            const int k = tids[i];
            if (static_cast<unsigned>(k) < static_cast<unsigned>(K)) atomicAdd(&h[k], 1);
        }
        __syncthreads();
        for (int k = threadIdx.x; k < K; k += blockDim.x)
            if (h[k]) h[k] = atomicAdd(&cur[k], h[k]);
        __syncthreads();
        for (int i = threadIdx.x; i < t1 - t0; i += blockDim.x) {
            const int k = tids[i];
            if (static_cast<unsigned>(k) < static_cast<unsigned>(K)) {
                const int pos = atomicAdd(&h[k], 1);
                pb[pos] = t0 + i;
            }
        }
    } else {
        for (int i = t0 + threadIdx.x; i < t1; i += blockDim.x) {
            const int k = idb[i];
            if (static_cast<unsigned>(k) < static_cast<unsigned>(K)) {
                const int pos = atomicAdd(&cur[k], 1);
                pb[pos] = i;
            }
        }
    }
}

template <typename T, int VEC> struct alignas(sizeof(T) * VEC) VecT {
    T v[VEC];
};

template <int VEC> __device__ __forceinline__ void red_add_row(float *dst, const float (&a)[VEC]) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + e), "f"(a[e]),
                         "f"(a[e + 1]), "f"(a[e + 2]), "f"(a[e + 3])
                         : "memory");
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) atomicAdd(dst + e, a[e]);
    }
}

// G lanes cooperate on one row (G a power of two), each lane covering VEC consecutive columns;
// a warp handles 32 / G rows per step. Column block blockIdx.y covers columns
// [blockIdx.y * G * VEC, +G * VEC).
template <typename T, int VEC, int G>
__global__ void __launch_bounds__(SEG_THREADS, 3)
    segreduce_kernel(const T *__restrict__ X, const float *__restrict__ w,
                     const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets, int B,
                     int N, int K, int d, int range, int ranges_per_batch, float *__restrict__ sums,
                     float *__restrict__ wsum) {
    constexpr int NG = 32 / G;           // rows per warp step
    constexpr int SB = G < 8 ? G : 8;    // rows gathered per lane before they are consumed
    constexpr unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * (SEG_THREADS / 32) + (threadIdx.x >> 5);
    if (gw >= static_cast<int64_t>(B) * ranges_per_batch) return;
    const int b = static_cast<int>(gw / ranges_per_batch);
    const int32_t *offb = offsets + static_cast<int64_t>(b) * (K + 1);
    // only the sorted positions that hold a point (offb[K] = number of in-range ids)
    const int p0 = static_cast<int>(gw % ranges_per_batch) * range;
    const int p1 = min(offb[K], p0 + range);
    if (p0 >= p1) return;
    const int g = lane / G, lg = lane % G;
    const int col = blockIdx.y * (G * VEC) + lg * VEC;
    const bool colok = col < d;
    const int32_t *permb = perm + static_cast<int64_t>(b) * N;
    const T *Xb = X + static_cast<int64_t>(b) * N * d;
    const float *wb = w ? w + static_cast<int64_t>(b) * N : nullptr;
    float *sb = sums + static_cast<int64_t>(b) * K * d;
    float *wsb = wsum ? wsum + static_cast<int64_t>(b) * K : nullptr;

    // segment holding p0: the largest k with offb[k] <= p0 (offb[0] = 0, offb[K] = N > p0)
    int lo = 0, hi = K - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offb[mid] <= p0) lo = mid; else hi = mid - 1;
    }
    int kcur = lo;

    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    float wacc = 0.f;
    int acck = -1;

    auto flush = [&](int k) {
        if (colok) red_add_row<VEC>(sb + static_cast<int64_t>(k) * d + col, acc);
        if (wsb && lg == 0 && blockIdx.y == 0) atomicAdd(wsb + k, wacc);
    };

    for (int q = p0; q < p1; q += 32) {
        const int pl = min(q + lane, p1 - 1);
        const int my_i = permb[pl];
        const float my_w = wb ? wb[my_i] : 1.f;
        // segment of pl = kcur + #{j >= 1 : offb[kcur + j] <= pl}; 32 offsets per probe round
        int base = kcur, my_k = -1;
        while (true) {
            const int idx = base + 1 + lane;
            const int o = idx <= K ? offb[idx] : INT_MAX;
            int cnt = 0;
#pragma unroll
            for (int st = 16; st > 0; st >>= 1) {
                const int pr = __shfl_sync(FULL, o, cnt + st - 1);
                if (pr <= pl) cnt += st;
            }
            const int o31 = __shfl_sync(FULL, o, 31);
            if (cnt == 31 && o31 <= pl) cnt = 32;
            if (my_k < 0 && cnt < 32) my_k = base + cnt;
            if (!__any_sync(FULL, my_k < 0)) break;
            base += 32;
        }
        kcur = __shfl_sync(FULL, my_k, 31);

#pragma unroll
        for (int s0 = 0; s0 < G; s0 += SB) {
            VecT<T, VEC> xv[SB];
            int kk[SB];
            float wv[SB];
            bool rv[SB];
#pragma unroll
            for (int s = 0; s < SB; ++s) {
                const int rr = (s0 + s) * NG + g;
                const int ii = __shfl_sync(FULL, my_i, rr);
                kk[s] = __shfl_sync(FULL, my_k, rr);
                wv[s] = __shfl_sync(FULL, my_w, rr);
                rv[s] = q + rr < p1;
                if (rv[s] && colok) {
                    xv[s] = *reinterpret_cast<const VecT<T, VEC> *>(Xb + static_cast<int64_t>(ii) * d + col);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) xv[s].v[e] = Cvt<T>::from_f(0.f);
                }
            }
#pragma unroll
            for (int s = 0; s < SB; ++s) {
                if (rv[s]) {
                    if (kk[s] != acck) {
                        if (acck >= 0) flush(acck);
                        acck = kk[s];
#pragma unroll
                        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
                        wacc = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] = fmaf(wv[s], Cvt<T>::to_f(xv[s].v[e]), acc[e]);
                    wacc += wv[s];
                }
            }
        }
    }
    if (acck >= 0) flush(acck);
}

}  // namespace upd
}  // namespace km
