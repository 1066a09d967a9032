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

// Block-wide bitonic sort of NP (a power of two) (value, index) pairs in shared memory, ascending
// by value; padding entries carry +inf. Ends with the block synchronised.
__device__ __forceinline__ void sort_pairs_smem(float *xs, int *is, int NP) {
    for (int k = 2; k <= NP; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = threadIdx.x; t < (NP >> 1); t += blockDim.x) {
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

    sort_pairs_smem(xs, is, NP);
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

// ---------------------------------------------------------------------------------------------
// Warp-per-row form (K <= 32), for many rows. The fused kernel above keeps a row on chip, so only
// a few rows fit on an SM and every phase of an iteration waits on the slowest thread of its row;
// with thousands of rows it is latency-bound. Here the per-row state that an iteration needs is
// reduced once, up front, to arrays in device memory:
//   fit1d_sort_kernel  (one CTA per row): the sorted values, their original indices and the
//                      prefix sums P0 = sum w, P1 = sum w*x and, when the objective is wanted,
//                      P2 = sum w*x^2 over the sorted order (fp64, P[0] = 0);
//   fit1d_iter_kernel  (one warp per row, every row resident at once): per iteration the K - 1
//                      cluster boundaries by binary search over the sorted values (the same
//                      exact-argmin test as above), then each cluster's weight, weighted sum and
//                      objective from two prefix-sum reads:
//                        W = P0[e] - P0[s], S = P1[e] - P1[s],
//                        sum w (x - c)^2 = (P2[e] - P2[s]) - 2 c S + c^2 W.
// An iteration then costs O(K log N) per row, independent of how many points each cluster holds.
constexpr int ITER_WARPS = 4;   // rows per block of the iteration kernel
constexpr int ITER_KMAX = 32;   // one centroid per lane

// Order-preserving unsigned keys of the stored values (finite inputs): flip every bit of a
// negative value, set the sign bit of a non-negative one.
template <typename T> struct SortKey;
template <> struct SortKey<float> {
    static constexpr int BITS = 32;
    using Word = uint32_t;   // shared-memory key storage
    static __device__ __forceinline__ uint32_t key(float v) {
        const uint32_t u = __float_as_uint(v);
        return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    static __device__ __forceinline__ float value(uint32_t k) {
        return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
    }
};
template <typename H, int DUMMY> struct SortKey16 {
    static constexpr int BITS = 16;
    using Word = uint16_t;
    static __device__ __forceinline__ uint32_t key(uint32_t u) {
        return (u & 0x8000u) ? (~u & 0xffffu) : (u | 0x8000u);
    }
    static __device__ __forceinline__ uint16_t raw(uint32_t k) {
        return static_cast<uint16_t>((k & 0x8000u) ? (k ^ 0x8000u) : (~k & 0xffffu));
    }
};
template <> struct SortKey<__half> : SortKey16<__half, 0> {
    static __device__ __forceinline__ uint32_t key(__half v) { return SortKey16::key(__half_as_ushort(v)); }
    static __device__ __forceinline__ float value(uint32_t k) { return __half2float(__ushort_as_half(raw(k))); }
};
template <> struct SortKey<__nv_bfloat16> : SortKey16<__nv_bfloat16, 0> {
    static __device__ __forceinline__ uint32_t key(__nv_bfloat16 v) {
        return SortKey16::key(__bfloat16_as_ushort(v));
    }
    static __device__ __forceinline__ float value(uint32_t k) {
        return __bfloat162float(__ushort_as_bfloat16(raw(k)));
    }
};

// Stable LSD radix sort of one row in shared memory, 8-bit digits (2 passes for 16-bit values, 4
// for fp32), by the block's THREADS threads. Warp w owns the contiguous positions
// [w * seg, (w + 1) * seg) and walks them 32 at a time: lanes holding the same digit find each
// other (eight ballots, one per digit bit), take consecutive slots after the warp's running
// count for that digit, and the lowest of them advances the count. A block-wide scan over
// (digit, warp) then turns the
// per-warp counts into destinations. Equal keys keep their order, so ties stay in index order.
// Padding positions carry the largest key and sort to the end. Result in (ka, ia).
constexpr int RADIX_WARPS = THREADS / 32;
constexpr int RADIX_MAX_ROUNDS = NMAX / RADIX_WARPS / 32;

template <int BITS, typename Word>
__device__ __forceinline__ void radix_sort_row(Word *ka, uint16_t *ia, Word *kb, uint16_t *ib,
                                               int (*hist)[256], int seg) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rounds = seg >> 5;
    const unsigned lt = (1u << lane) - 1u;
    for (int shift = 0; shift < BITS; shift += 8) {
        for (int i = lane; i < 256; i += 32) hist[warp][i] = 0;
        __syncwarp();
        int local[RADIX_MAX_ROUNDS];
#pragma unroll
        for (int r = 0; r < RADIX_MAX_ROUNDS; ++r) {
            if (r < rounds) {
                const int pos = warp * seg + r * 32 + lane;
                const int dg = (ka[pos] >> shift) & 255;
                // the lanes holding the same digit: those agreeing on all eight bits (eight
                // ballots; measured faster here than one match instruction)
                unsigned m = 0xffffffffu;
#pragma unroll
                for (int bit = 0; bit < 8; ++bit) {
                    const unsigned bal = __ballot_sync(0xffffffffu, (dg >> bit) & 1);
                    m &= ((dg >> bit) & 1) ? bal : ~bal;
                }
                const int base = hist[warp][dg];
                local[r] = base + __popc(m & lt);
                __syncwarp();
                if ((m & lt) == 0) hist[warp][dg] = base + __popc(m);
                __syncwarp();
            }
        }
        __syncthreads();
        // thread t = digit t: warp bases for this digit, then an exclusive scan over digits
        {
            int tot = 0;
            for (int v = 0; v < RADIX_WARPS; ++v) tot += hist[v][tid];
            int inc = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += u;
            }
            __shared__ int wsum[RADIX_WARPS];
            if (lane == 31) wsum[warp] = inc;
            __syncthreads();
            int run = inc - tot;
            for (int v = 0; v < warp; ++v) run += wsum[v];
            for (int v = 0; v < RADIX_WARPS; ++v) {
                const int c = hist[v][tid];
                hist[v][tid] = run;
                run += c;
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RADIX_MAX_ROUNDS; ++r) {
            if (r < rounds) {
                const int pos = warp * seg + r * 32 + lane;
                const Word k = ka[pos];
                const int dst = hist[warp][(k >> shift) & 255] + local[r];
                kb[dst] = k;
                ib[dst] = ia[pos];
            }
        }
        __syncthreads();
        Word *tk = ka;
        ka = kb;
        kb = tk;
        uint16_t *ti = ia;
        ia = ib;
        ib = ti;
    }
}

template <typename T>
__global__ void __launch_bounds__(THREADS, 4)
    fit1d_sort_kernel(const T *__restrict__ X, const float *__restrict__ w, int N, int NP,
                      float *__restrict__ xs_out, int32_t *__restrict__ is_out,
                      double *__restrict__ P0, double *__restrict__ P1, double *__restrict__ P2) {
    // shared memory: (keys, indices) twice, NP = 8 * seg entries each; keys are 16- or 32-bit
    // words. The second pair is contiguous, so after the sort it serves as NP floats.
    using Word = typename SortKey<T>::Word;
    extern __shared__ uint8_t sm[];
    Word *ka = reinterpret_cast<Word *>(sm);
    uint16_t *ia = reinterpret_cast<uint16_t *>(ka + NP);
    Word *kb = reinterpret_cast<Word *>(ia + NP);
    uint16_t *ib = reinterpret_cast<uint16_t *>(kb + NP);
    __shared__ int hist[RADIX_WARPS][256];
    __shared__ double wtot[3][THREADS / 32];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const T *xb = X + static_cast<int64_t>(b) * N;
    for (int p = tid; p < NP; p += THREADS) {
        ka[p] = static_cast<Word>(p < N ? SortKey<T>::key(xb[p]) : 0xffffffffu);
        ia[p] = static_cast<uint16_t>(p);
    }
    __syncthreads();
    radix_sort_row<SortKey<T>::BITS, Word>(ka, ia, kb, ib, hist, NP / RADIX_WARPS);
    // an even number of passes leaves the result in (ka, ia)
    const int64_t rb = static_cast<int64_t>(b) * N, pb = static_cast<int64_t>(b) * (N + 1);
    // prefix sums over the sorted order, THREADS positions at a time (coalesced stores); the
    // running totals before each tile are the same in every thread. P2 may be null (no objective).
    if (tid == 0) {
        P0[pb] = 0.0;
        P1[pb] = 0.0;
        if (P2) P2[pb] = 0.0;
    }
    // the weights in sorted order, gathered 8 per thread at a time into the sort's scratch pair
    // (free now; at least 4 contiguous bytes per position), before the scan needs them
    float *wsm = reinterpret_cast<float *>(kb);
    if (w) {
        for (int q = 0; q < N; q += 8 * THREADS) {
            float t8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = q + j * THREADS + tid;
                t8[j] = p < N ? w[rb + ia[p]] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int p = q + j * THREADS + tid;
                if (p < N) wsm[p] = t8[j];
            }
        }
        __syncthreads();
    }
    double c0 = 0.0, c1 = 0.0, c2 = 0.0;
    for (int base = 0; base < N; base += THREADS) {
        const int p = base + tid;
        double v0 = 0.0, v1 = 0.0, v2 = 0.0;
        if (p < N) {
            const double x = SortKey<T>::value(ka[p]), wt = w ? wsm[p] : 1.f;
            v0 = wt;
            v1 = wt * x;
            v2 = v1 * x;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // inclusive scan within the warp
            const double u0 = __shfl_up_sync(0xffffffffu, v0, o);
            const double u1 = __shfl_up_sync(0xffffffffu, v1, o);
            const double u2 = __shfl_up_sync(0xffffffffu, v2, o);
            if (lane >= o) {
                v0 += u0;
                v1 += u1;
                v2 += u2;
            }
        }
        if (lane == 31) {
            wtot[0][warp] = v0;
            wtot[1][warp] = v1;
            wtot[2][warp] = v2;
        }
        __syncthreads();
        double o0 = c0, o1 = c1, o2 = c2;
        for (int v = 0; v < RADIX_WARPS; ++v) {
            if (v < warp) {
                o0 += wtot[0][v];
                o1 += wtot[1][v];
                o2 += wtot[2][v];
            }
            c0 += wtot[0][v];
            c1 += wtot[1][v];
            c2 += wtot[2][v];
        }
        if (p < N) {
            P0[pb + p + 1] = o0 + v0;
            P1[pb + p + 1] = o1 + v1;
            if (P2) P2[pb + p + 1] = o2 + v2;
        }
        __syncthreads();   // wtot is rewritten by the next tile
    }
    for (int p = tid; p < N; p += THREADS) {
        xs_out[rb + p] = SortKey<T>::value(ka[p]);
        is_out[rb + p] = ia[p];
    }
}

// KT: a power of two >= K, fixed per instantiation, so every lane keeps the rounded centroids in
// registers for the whole iteration (entries K .. KT-1 hold NaN, which never compares below a
// distance) and a probe's scan over them is unrolled with no memory access.
template <typename T, int KT>
__global__ void __launch_bounds__(ITER_WARPS * 32)
    fit1d_iter_kernel(const float *__restrict__ xs, const int32_t *__restrict__ is,
                      const double *__restrict__ P0, const double *__restrict__ P1,
                      const double *__restrict__ P2, int B, int N, int K, int iters,
                      float *__restrict__ C, int32_t *__restrict__ ids,
                      double *__restrict__ inertia_hist, float *__restrict__ C_hist) {
    constexpr unsigned FULL = 0xffffffffu;
    __shared__ float cx_s[ITER_WARPS][ITER_KMAX];   // rounded centroids, by index
    __shared__ int rank_s[ITER_WARPS][ITER_KMAX];   // rank of centroid k in (cx, k) order
    __shared__ int order_s[ITER_WARPS][ITER_KMAX];  // centroid at each rank
    __shared__ int E_s[ITER_WARPS][ITER_KMAX];      // #points whose nearest centroid has rank <= q
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * ITER_WARPS + warp;
    if (b >= B) return;   // whole warps only; nothing below synchronises the block
    float *cxw = cx_s[warp];
    int *rankw = rank_s[warp], *orderw = order_s[warp], *Ew = E_s[warp];
    const int64_t rb = static_cast<int64_t>(b) * N, pb = static_cast<int64_t>(b) * (N + 1);
    const float *xr = xs + rb;
    const bool own = lane < K;   // lane k holds centroid k
    float cm = own ? C[static_cast<int64_t>(b) * K + lane] : 0.f;
    if (own && C_hist) C_hist[static_cast<int64_t>(b) * K + lane] = cm;
    int steps = 0;   // halvings that take a range of N + 1 candidates down to one
    while ((1 << steps) <= N) ++steps;

    for (int t = 0; t <= iters; ++t) {
        const bool final_pass = (t == iters);
        if (final_pass && !ids) break;
        const float cxk = own ? round_through<T>(cm) : 0.f;
        if (own) cxw[lane] = cxk;
        __syncwarp();
        int r = 0;
        if (own) {
            for (int j = 0; j < K; ++j) {
                const float u = cxw[j];
                r += (u < cxk) || (u == cxk && j < lane);
            }
            rankw[lane] = r;
            orderw[r] = lane;
        }
        __syncwarp();
        float creg[KT];
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            const float v = __shfl_sync(FULL, cxk, k);
            creg[k] = k < K ? v : __int_as_float(0x7fffffff);
        }
        // boundary q = lane: first sorted position whose nearest centroid ranks above q
        int lo = 0, len = N;
        for (int st = 0; st < steps; ++st) {
            const int half = len >> 1;
            const int mid = lo + half;
            const float x = len > 0 ? xr[mid] : 0.f;
            float best = INFINITY;
            int bi = 0;
#pragma unroll
            for (int k = 0; k < KT; ++k) {   // the first strict minimum: the lowest index on ties
                const float dx = x - creg[k];
                const float dd = dx * dx;
                if (dd < best) {
                    best = dd;
                    bi = k;
                }
            }
            if (len > 0) {
                if (rankw[bi] <= lane) {
                    lo = mid + 1;
                    len -= half + 1;
                } else {
                    len = half;
                }
            }
        }
        const int Eq = lane < K - 1 ? lo : N;
        if (own) Ew[lane] = Eq;
        __syncwarp();
        if (final_pass) {
            for (int p = lane; p < N; p += 32) {
                int q = 0;
                while (Ew[q] <= p) ++q;
                ids[rb + is[rb + p]] = orderw[q];
            }
            break;
        }
        // cluster of rank q = lane: sorted positions [s, Eq), centroid orderw[q]
        const int s = (own && lane > 0) ? Ew[lane - 1] : 0;
        double W = 0.0, S = 0.0, Q = 0.0;
        int cnt = 0;
        if (own) {
            cnt = Eq - s;
            W = P0[pb + Eq] - P0[pb + s];
            S = P1[pb + Eq] - P1[pb + s];
            Q = P2 ? P2[pb + Eq] - P2[pb + s] : 0.0;
        }
        const double c = own ? static_cast<double>(cxw[orderw[lane]]) : 0.0;
        if (inertia_hist) {   // warp-uniform
            double iner = own ? (Q - 2.0 * c * S) + c * c * W : 0.0;
            iner = warp_sum(iner);
            if (lane == 0) inertia_hist[static_cast<int64_t>(t) * B + b] = iner;
        }
        const bool moved = own && cnt > 0 && W > 0.0;
        const float nv = moved ? __double2float_rn(__ddiv_rn(S, W)) : 0.f;
        const unsigned moved_mask = __ballot_sync(FULL, moved);
        const int my_rank = own ? rankw[lane] : 0;
        const float got = __shfl_sync(FULL, nv, my_rank);
        if (own && ((moved_mask >> my_rank) & 1u)) cm = got;
        if (own && C_hist) C_hist[(static_cast<int64_t>(t + 1) * B + b) * K + lane] = cm;
        __syncwarp();
    }
    if (own) C[static_cast<int64_t>(b) * K + lane] = cm;
}

}  // namespace fit1d
}  // namespace km
