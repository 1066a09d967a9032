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

// Log2 of the search span: the smallest power of two above K (the count of sorted entries at or
// below a value runs from 0 to K).
__host__ __device__ constexpr int enc_logp(int K) {
    int l = 0;
    while ((1 << l) <= K) ++l;
    return l;
}

// LOGP = enc_logp(K), fixed per instantiation so the binary search unrolls and a thread's values
// are searched side by side. VEC: N is a multiple of 16 and X, codes are 16-byte aligned, so a
// thread reads its 16 consecutive values with vector loads and writes their codes as one 16-byte
// store; otherwise thread t takes values t, t + 256, ... of the block's range.
template <typename T, int LOGP, bool VEC>
__global__ void __launch_bounds__(ENC_THREADS)
    encode1d_kernel(const T *__restrict__ X, int64_t N, const float *__restrict__ C, int K,
                    uint8_t *__restrict__ codes) {
    constexpr int P = 1 << LOGP;
    __shared__ float cv[ENC_KMAX];       // the rounded centroids in index order
    __shared__ float sv[P];              // the same ascending by (value, index), then NaN
    __shared__ int si[ENC_KMAX];         // their indices
    __shared__ float4 br[ENC_KMAX + 1];  // per count lo of entries <= x: sorted entries lo-1, lo,
    __shared__ int2 bi[ENC_KMAX + 1];    // lo-2, lo+1 (+-inf past the ends); indices of lo-1, lo
    const int b = blockIdx.y, tid = threadIdx.x;
    const T *xb = X + static_cast<int64_t>(b) * N;
    uint8_t *ob = codes + static_cast<int64_t>(b) * N;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * (ENC_THREADS * ENC_VPT);
    // this thread's values are requested first, so their latency overlaps the codebook's setup
    float x[ENC_VPT];
    const int64_t i0 = base + static_cast<int64_t>(tid) * ENC_VPT;
    const bool vin = VEC && i0 < N;   // the vector form's values are all in range or all out
    if constexpr (VEC) {
        constexpr int PER = 16 / sizeof(T);   // values per 16-byte load
        uint4 raw[ENC_VPT / PER];
#pragma unroll
        for (int q = 0; q < ENC_VPT / PER; ++q)
            raw[q] = vin ? __ldg(reinterpret_cast<const uint4 *>(xb + i0) + q) : make_uint4(0, 0, 0, 0);
        const T *tv = reinterpret_cast<const T *>(raw);
#pragma unroll
        for (int v = 0; v < ENC_VPT; ++v) x[v] = Cvt<T>::to_f(tv[v]);
    } else {
#pragma unroll
        for (int v = 0; v < ENC_VPT; ++v) {
            const int64_t i = base + static_cast<int64_t>(v) * ENC_THREADS + tid;
            x[v] = i < N ? Cvt<T>::to_f(xb[i]) : 0.f;
        }
    }
    const float *Cb = C + static_cast<int64_t>(b) * K;
    if (tid < K) cv[tid] = round_through<T>(Cb[tid]);
    // NaN padding: `pad <= x` is false for every x, so the count never runs past K
    for (int t = K + tid; t < P; t += ENC_THREADS) sv[t] = __int_as_float(0x7fffffff);
    __syncthreads();
    if (tid < K) {
        const float v = cv[tid];
        int r = 0;
        for (int j = 0; j < K; ++j) {
            const float u = cv[j];
            r += (u < v) || (u == v && j < tid);
        }
        sv[r] = v;
        si[r] = tid;
    }
    __syncthreads();
    for (int lo = tid; lo <= K; lo += ENC_THREADS) {
        br[lo] = make_float4(lo > 0 ? sv[lo - 1] : -INFINITY, lo < K ? sv[lo] : INFINITY,
                             lo > 1 ? sv[lo - 2] : -INFINITY, lo + 1 < K ? sv[lo + 1] : INFINITY);
        bi[lo] = make_int2(si[lo > 0 ? lo - 1 : 0], si[lo < K ? lo : K - 1]);
    }
    __syncthreads();
    uint32_t packed[ENC_VPT / 4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int v = 0; v < ENC_VPT; ++v) {
        const float xv = x[v];
        int lo = 0;   // number of sorted entries <= x
#pragma unroll
        for (int s = LOGP - 1; s >= 0; --s)
            if (sv[lo + (1 << s) - 1] <= xv) lo += 1 << s;
        const float4 e = br[lo];
        const int2 ix = bi[lo];
        // the nearest sits on one of the two entries bracketing x (an infinite side never wins)
        const float tl = xv - e.x, tr = xv - e.y;
        const float dl = tl * tl, dr = tr * tr;
        const float best = fminf(dl, dr);
        int idx = dr < dl ? ix.y : ix.x;
        if (dr == dl) idx = min(ix.x, ix.y);
        // a third centroid can tie only with exactly the same rounded distance (rare)
        const float t2 = xv - e.z, t3 = xv - e.w;
        if (t2 * t2 == best || t3 * t3 == best) {
            for (int q = lo - 2; q >= 0; --q) {   // distances grow leftwards
                const float t = xv - sv[q];
                if (t * t != best) break;
                idx = min(idx, si[q]);
            }
            for (int q = lo + 1; q < K; ++q) {    // and rightwards
                const float t = xv - sv[q];
                if (t * t != best) break;
                idx = min(idx, si[q]);
            }
        }
        if constexpr (VEC) {
            packed[v >> 2] |= static_cast<uint32_t>(idx & 0xff) << (8 * (v & 3));
        } else {
            const int64_t i = base + static_cast<int64_t>(v) * ENC_THREADS + tid;
            if (i < N) ob[i] = static_cast<uint8_t>(idx);
        }
    }
    if constexpr (VEC) {
        if (vin) *reinterpret_cast<uint4 *>(ob + i0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

constexpr int PP_THREADS = 512;
constexpr int PP_PER = 16;      // points per thread: rows of up to PP_THREADS * PP_PER values
constexpr int PP_NMAX = PP_THREADS * PP_PER;

// One block per row; thread t owns the contiguous points [t * per, t * per + per), so a block scan
// of the per-thread masses gives running sums in point order. PER >= per bounds the thread's
// arrays: rows of up to 4096 values take PER = 8, which leaves room for two blocks per SM.
template <typename T, int PER>
__global__ void __launch_bounds__(PP_THREADS, PER <= 8 ? 2 : 1)
    kmeanspp1d_kernel(const T *__restrict__ X, const float *__restrict__ w, int N, int K,
                      const float *__restrict__ u, float *__restrict__ C,
                      int32_t *__restrict__ chosen) {
    constexpr int NW = PP_THREADS / 32;
    __shared__ double wtot[NW];
    __shared__ int last_mass;
    // the chosen point as (index << 32) | its value's bits, all ones while none: the lowest
    // claimant wins, and the index and value always come from the same thread
    __shared__ unsigned long long pick;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (N + PP_THREADS - 1) / PP_THREADS;
    const int p0 = min(N, tid * per);
    const int np = min(N, p0 + per) - p0;
    const int64_t rb = static_cast<int64_t>(b) * N;
    float xv[PER], wv[PER];
    double d2[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const bool in = e < np;
        xv[e] = in ? Cvt<T>::to_f(X[rb + p0 + e]) : 0.f;
        wv[e] = in ? (w ? w[rb + p0 + e] : 1.f) : 0.f;
        d2[e] = 1.0;   // the first draw is proportional to the weights alone
    }
    const float *ub = u + static_cast<int64_t>(b) * K;
    float u_next = ub[0];   // each draw's uniform is requested one draw ahead
    for (int k = 0; k < K; ++k) {
        const float uk = u_next;
        if (k + 1 < K) u_next = ub[k + 1];
        double loc = 0.0;
        int mylast = -1;   // this thread's last point with mass
#pragma unroll
        for (int e = 0; e < PER; ++e) {
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
            pick = ~0ull;
            last_mass = -1;
        }
        __syncthreads();
        if (mylast >= 0) atomicMax(&last_mass, mylast);
        // the warps' totals scanned across the lanes of every warp: this warp's offset and the row's total
        double ws = lane < NW ? wtot[lane] : 0.0;
#pragma unroll
        for (int o = 1; o < NW; o <<= 1) {
            const double t = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += t;
        }
        const double total = __shfl_sync(0xffffffffu, ws, NW - 1);
        const double wprev = __shfl_sync(0xffffffffu, ws, warp > 0 ? warp - 1 : 0);
        const double off = warp > 0 ? wprev : 0.0;
        if (total > 0.0) {
            const double target = static_cast<double>(uk) * total;
            double run = off + inc - loc;
            if (run <= target && run + loc > target) {
#pragma unroll
                for (int e = 0; e < PER; ++e) {
                    const double m = static_cast<double>(wv[e]) * d2[e];
                    run += m;
                    if (e < np && m > 0.0 && run > target) {
                        atomicMin(&pick, (static_cast<unsigned long long>(p0 + e) << 32) | __float_as_uint(xv[e]));
                        break;
                    }
                }
            }
        }
        __syncthreads();
        // no mass left: point 0; rounding left the target at the total: the last point with mass
        if (tid == 0 && pick == ~0ull) {
            const int f = last_mass >= 0 ? last_mass : 0;
            pick = (static_cast<unsigned long long>(f) << 32) | __float_as_uint(Cvt<T>::to_f(X[rb + f]));
        }
        __syncthreads();
        const unsigned long long pv = pick;
        const int i = static_cast<int>(pv >> 32);
        const float c = __uint_as_float(static_cast<uint32_t>(pv));
        if (tid == 0) {
            C[static_cast<int64_t>(b) * K + k] = c;
            if (chosen) chosen[static_cast<int64_t>(b) * K + k] = i;
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const double t = static_cast<double>(xv[e]) - static_cast<double>(c);
            const double dd = t * t;
            d2[e] = (k == 0) ? dd : fmin(d2[e], dd);
        }
        __syncthreads();   // wtot and pick are rewritten by the next draw
    }
}

}  // namespace cb
}  // namespace km
