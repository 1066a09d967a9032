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
//              Two forms: segreduce_rows_kernel for d = 32 * V (one warp load per row, the run
//              logic warp-uniform, many warps per SM to keep the random row gathers in flight)
//              and segreduce_kernel for any other d (G lanes per row, column blocks).
//
// The order of points inside a segment is not fixed (tiles reserve their slots atomically), so
// fp32 sums may differ in the last bits from run to run; the set of points per segment, the
// counts and the offsets are exact.
#pragma once

#include <limits.h>

#include <type_traits>

#include "km_common.cuh"

namespace km {
namespace upd {

constexpr int TILE = 8192;          // points per histogram / scatter tile
constexpr int TILE_THREADS = 512;
constexpr int SCATTER_PPT = TILE / TILE_THREADS;   // points per thread of a scatter tile
constexpr int SCATTER_SORT_K_MAX = 4096;           // tiles sorted in shared memory up to this K
static_assert(TILE <= 8192 && SCATTER_SORT_K_MAX <= (1 << 18), "(cluster, point) packs in 31 bits");
constexpr int SMEM_K_MAX = 16384;   // bins kept in shared memory
constexpr int SCAN_THREADS = 1024;
constexpr int SEG_THREADS = 256;
constexpr int SEG_BLOCKS_PER_SM = 2;

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

// `tile` <= TILE points per block (smaller tiles give small problems more blocks).
__global__ void __launch_bounds__(TILE_THREADS)
    scatter_kernel(const int32_t *__restrict__ ids, int N, int K, int32_t *__restrict__ cursor,
                   int32_t *__restrict__ perm, int use_smem, int tile) {
    extern __shared__ int ssm[];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * tile;
    const int t1 = min(N, t0 + tile);
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

// dst[i] += src[i] (per-cluster counts of one chunk of points added to the running counts)
__global__ void add_i32_kernel(int32_t *__restrict__ dst, const int32_t *__restrict__ src, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) dst[i] += src[i];
}

template <typename T, int VEC> struct alignas(sizeof(T) * VEC) VecT {
    T v[VEC];
};

// The reducing kernels never read the sums back, so the vector reduction carries no memory
// clobber and loads may be scheduled across it.
template <int VEC> __device__ __forceinline__ void red_add_row(float *dst, const float (&a)[VEC]) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + e), "f"(a[e]),
                         "f"(a[e + 1]), "f"(a[e + 2]), "f"(a[e + 3]));
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) atomicAdd(dst + e, a[e]);
    }
}

// G lanes cooperate on one row (G a power of two), each lane covering VEC consecutive columns;
// a warp handles 32 / G rows per step. Column block blockIdx.y covers columns
// [blockIdx.y * G * VEC, +G * VEC).
//
// Per chunk of 32 sorted positions the warp loads the chunk's point indices (prefetched one
// chunk ahead), issues the row gathers at once (SB rows per lane in flight), and only then
// looks up the segment (cluster) of each position, so the lookup's reads of the offsets
// overlap the gathers instead of delaying them.
template <typename T, int VEC, int G>
__global__ void __launch_bounds__(SEG_THREADS, SEG_BLOCKS_PER_SM)
    segreduce_kernel(const T *__restrict__ X, const float *__restrict__ w,
                     const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets, int B,
                     int N, int K, int d, int range, int ranges_per_batch, float *__restrict__ sums,
                     float *__restrict__ wsum) {
    constexpr int NG = 32 / G;           // rows per warp step
    // rows gathered per lane before they are consumed (bf16 rows take more registers to
    // convert, so fewer are kept in flight there)
    constexpr int SBMAX = std::is_same<T, __nv_bfloat16>::value ? 8 : 16;
    constexpr int SB = G < SBMAX ? G : SBMAX;
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

    int next_i = permb[min(p0 + lane, p1 - 1)];
    for (int q = p0; q < p1; q += 32) {
        const int pl = min(q + lane, p1 - 1);
        const int my_i = next_i;
        if (q + 32 < p1) next_i = permb[min(q + 32 + lane, p1 - 1)];
        const float my_w = wb ? wb[my_i] : 1.f;
        int kseg = 0;

#pragma unroll
        for (int s0 = 0; s0 < G; s0 += SB) {
            VecT<T, VEC> xv[SB];
            bool rv[SB];
#pragma unroll
            for (int s = 0; s < SB; ++s) {
                const int rr = (s0 + s) * NG + g;
                const int ii = __shfl_sync(FULL, my_i, rr);
                rv[s] = q + rr < p1;
                if (rv[s] && colok) {
                    xv[s] = *reinterpret_cast<const VecT<T, VEC> *>(Xb + static_cast<int64_t>(ii) * d + col);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) xv[s].v[e] = Cvt<T>::from_f(0.f);
                }
            }
            if (s0 == 0) {
                // segment of pl = kcur + #{j >= 1 : offb[kcur + j] <= pl}; 32 offsets per probe
                // round (runs while the gathers above are in flight)
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
                kseg = my_k;
            }
#pragma unroll
            for (int s = 0; s < SB; ++s) {
                const int rr = (s0 + s) * NG + g;
                const int kk = __shfl_sync(FULL, kseg, rr);
                const float wv = __shfl_sync(FULL, my_w, rr);
                if (rv[s]) {
                    if (kk != acck) {
                        if (acck >= 0) flush(acck);
                        acck = kk;
#pragma unroll
                        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
                        wacc = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] = fmaf(wv, Cvt<T>::to_f(xv[s].v[e]), acc[e]);
                    wacc += wv;
                }
            }
        }
    }
    if (acck >= 0) flush(acck);
}

// The segmented reduction for d = 32 * V (V * sizeof(T) of 4, 8 or 16 bytes): lane l of a warp
// owns columns [l * V, l * V + V), so one warp load fetches one whole row (coalesced) and the
// cluster of a row, the end of a run and the flush are warp-uniform (one vector atomic per lane
// per run). Each warp walks chunks of 32 sorted positions; the chunk's point indices are
// fetched one chunk ahead, and its rows are loaded R at a time into registers (R rows of
// V * sizeof(T) bytes per lane = 2 KB per warp) before any of them is summed. R is what fits
// in the 64 registers that four blocks per SM allow without spilling: 4 KB per warp spilled
// and measured 9-17 % slower, fewer warps per SM (more registers) slower still.
constexpr int ROWS_THREADS = 256;
constexpr int ROWS_BLOCKS_PER_SM = 4;

template <typename T, int V, bool WEIGHTED>
__global__ void __launch_bounds__(ROWS_THREADS, ROWS_BLOCKS_PER_SM)
    segreduce_rows_kernel(const T *__restrict__ X, const float *__restrict__ w,
                          const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets,
                          int B, int N, int K, int range, int ranges_per_batch,
                          float *__restrict__ sums, float *__restrict__ wsum) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int d = 32 * V;
    constexpr int R = 64 / static_cast<int>(V * sizeof(T));    // rows in flight per lane
    const int lane = threadIdx.x & 31;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * (ROWS_THREADS / 32) + (threadIdx.x >> 5);
    if (gw >= static_cast<int64_t>(B) * ranges_per_batch) return;
    const int b = static_cast<int>(gw / ranges_per_batch);
    const int32_t *offb = offsets + static_cast<int64_t>(b) * (K + 1);
    const int p0 = static_cast<int>(gw % ranges_per_batch) * range;
    const int p1 = min(offb[K], p0 + range);
    if (p0 >= p1) return;
    const int nchunks = (p1 - p0 + 31) / 32;
    const int col = lane * V;
    const int32_t *permb = perm + static_cast<int64_t>(b) * N;
    const T *Xb = X + static_cast<int64_t>(b) * N * d + col;
    const float *wb = WEIGHTED ? w + static_cast<int64_t>(b) * N : nullptr;
    float *sb = sums + static_cast<int64_t>(b) * K * d + col;
    float *wsb = wsum ? wsum + static_cast<int64_t>(b) * K : nullptr;   // wanted with or without weights

    // segment holding p0: the largest k with offb[k] <= p0 (offb[0] = 0, offb[K] = N > p0)
    int lo = 0, hi = K - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offb[mid] <= p0) lo = mid; else hi = mid - 1;
    }
    int kcur = lo;

    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    float wacc = 0.f;
    int acck = -1;
    auto flush = [&](int k) {
        red_add_row<V>(sb + static_cast<int64_t>(k) * d, acc);
        if (wsb && lane == 0) atomicAdd(wsb + k, wacc);
    };

    auto load_idx = [&](int c) {
        const int pos = p0 + 32 * c + lane;
        return (c < nchunks && pos < p1) ? permb[pos] : -1;
    };
    int idx_next = load_idx(0);
    for (int c = 0; c < nchunks; ++c) {
        const int my_i = idx_next;
        idx_next = load_idx(c + 1);
        const int q = p0 + 32 * c;
        const int nrows = min(32, p1 - q);
        unsigned starts = 0;
        int my_k = 0;
        float my_w = 1.f;
#pragma unroll 1
        for (int h = 0; h < 32; h += R) {
            if (h < nrows) {   // warp-uniform
                VecT<T, V> xv[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int ri = __shfl_sync(FULL, my_i, h + r);
                    if (h + r < nrows) xv[r] = *reinterpret_cast<const VecT<T, V> *>(Xb + static_cast<int64_t>(ri) * d);
                }
                if (h == 0) {
                    // clusters of the chunk's positions, while the first rows are in flight:
                    // segment of pl = kcur + #{j >= 1 : offb[kcur + j] <= pl}
                    const int pl = min(q + lane, p1 - 1);
                    int base = kcur;
                    my_k = -1;
                    while (true) {
                        const int idx = base + 1 + lane;
                        const int o = idx <= K ? offb[idx] : INT_MAX;
                        int cnt = 0;
#pragma unroll
                        for (int stp = 16; stp > 0; stp >>= 1) {
                            const int pr = __shfl_sync(FULL, o, cnt + stp - 1);
                            if (pr <= pl) cnt += stp;
                        }
                        const int o31 = __shfl_sync(FULL, o, 31);
                        if (cnt == 31 && o31 <= pl) cnt = 32;
                        if (my_k < 0 && cnt < 32) my_k = base + cnt;
                        if (!__any_sync(FULL, my_k < 0)) break;
                        base += 32;
                    }
                    kcur = __shfl_sync(FULL, my_k, 31);
                    if (WEIGHTED) my_w = my_i >= 0 ? wb[my_i] : 0.f;
                    // rows that start a new run (their cluster differs from the previous row's)
                    int prev_k = __shfl_up_sync(FULL, my_k, 1);
                    if (lane == 0) prev_k = acck;
                    starts = __ballot_sync(FULL, lane < nrows && my_k != prev_k);
                }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int rr = h + r;
                    if (rr < nrows) {   // warp-uniform
                        if ((starts >> rr) & 1u) {   // warp-uniform, about once per run
                            if (acck >= 0) flush(acck);
                            acck = __shfl_sync(FULL, my_k, rr);
#pragma unroll
                            for (int e = 0; e < V; ++e) acc[e] = 0.f;
                            wacc = 0.f;
                        }
                        if constexpr (WEIGHTED) {
                            const float wv = __shfl_sync(FULL, my_w, rr);
#pragma unroll
                            for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, Cvt<T>::to_f(xv[r].v[e]), acc[e]);
                            wacc += wv;
                        } else {
#pragma unroll
                            for (int e = 0; e < V; ++e) acc[e] += Cvt<T>::to_f(xv[r].v[e]);
                            wacc += 1.f;
                        }
                    }
                }
            }
        }
    }
    if (acck >= 0) flush(acck);
}

// ------------------------------------------------------------------ reduce and divide in one pass
//
// segreduce_final_kernel is the segmented reduction above fused with the final divide, for
// d = 32 * V with rows of 128, 256 or 512 bytes. Two differences from segreduce_rows_kernel:
//
// Row gathers go through the tensor-memory-access engine: each warp owns a ring of S stages of
// 32 rows in shared memory, and for every chunk of 32 sorted positions eight of its lanes issue
// one four-row gather each (cp.async.bulk.tensor tile::gather4 on a [B*N, d] view of X, box one
// row high), completing on the stage's mbarrier. S - 1 chunks are in flight while the warp sums
// the current one out of shared memory, so the bytes in flight are bounded by shared memory,
// not by registers (the register-staged form is bound by gather latency).
//
// No per-cluster sums array: a run that lies entirely inside the warp's range of sorted positions
// is a whole cluster, so the warp divides it by its count (or weight sum) and writes C_new, and
// when asked the rounded Cx, ||Cx||^2 and the weight sum. A cluster whose segment crosses range
// boundaries leaves one partial per range it touches in a per-range slot (side 0: the range's
// first run, side 1: its last run), then counts itself on the cluster's arrival counter; the
// warp that arrives last (the count of ranges touching the segment is known from the offsets)
// adds the partials in range order and finalizes. Nobody waits, so there is no spin. Empty
// clusters are written by scan_final_kernel.
constexpr int FZ_CHUNK = 32;

struct FinalParams {
    int B, N, K, range, rpb;
    int xld, x0;        // X rows of batch element b: b * xld + x0 + [0, N) (a mini-batch view)
    const int32_t *perm, *offsets;
    const float *w;     // weights of batch element b at w + b * xld + x0
    const float *C_prev;
    float *C_new;
    void *Cx;
    float *cn;
    float *wsum;        // per-cluster weight sums out (counts when unweighted), or null
    const int32_t *rseg;  // [B * rpb] the segment holding each range's first position, or null
    float *slots;       // [B * rpb * 2, d] partials of split segments
    float *wslots;      // [B * rpb * 2] their weight sums
    int32_t *arrive;    // [B, K] arrival counters, zeroed by scan_final_kernel
    // moving-average form (e-means): the batch statistics enter the state (C, Nc) instead of
    // replacing C, and are added to the epoch totals (eS may be null; eW null when unweighted)
    float alpha;
    float *Nc, *eS, *eW;
    int32_t *eCnt;
};

// warps per CTA and ring depth for a row of RB bytes (one CTA per SM, 192 KB of rings). The
// summing loop is bound by the latency of its own instruction chains, so the rings favour more
// warps over deeper rings (measured: 12 warps x 2 stages of 32 rows beat 8 x 3 for 256-byte rows).
__host__ __device__ constexpr int fz_warps(int RB) { return RB >= 512 ? 6 : (RB >= 256 ? 12 : 16); }
__host__ __device__ constexpr int fz_stages(int RB) { return RB >= 128 && RB < 256 ? 3 : 2; }
__host__ __device__ constexpr int fz_smem(int RB) {
    return fz_warps(RB) * fz_stages(RB) * FZ_CHUNK * RB + 1024;
}

__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *tm, uint32_t bar, int col,
                                            int r0, int r1, int r2, int r3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(dst),
        "l"(tm), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar), "l"(policy)
        : "memory");
}

template <typename T, int V> struct RowLd;
template <typename T> struct RowLd<T, 2> { using U = uint32_t; };     // 16-bit V=2: 4 B
template <> struct RowLd<float, 1> { using U = float; };
template <typename T> struct RowLd<T, 4> { using U = uint2; };
template <> struct RowLd<float, 2> { using U = float2; };
template <typename T> struct RowLd<T, 8> { using U = uint4; };
template <> struct RowLd<float, 4> { using U = float4; };

// The V elements lane `lane` owns of one row in shared memory, as fp32.
template <typename T, int V>
__device__ __forceinline__ void row_vals(const uint8_t *row, int lane, float (&x)[V]) {
    using U = typename RowLd<T, V>::U;
    const U u = reinterpret_cast<const U *>(row)[lane];
    const T *t = reinterpret_cast<const T *>(&u);
#pragma unroll
    for (int e = 0; e < V; ++e) x[e] = Cvt<T>::to_f(t[e]);
}

// acc += the V elements lane `lane` owns of one row. For 16-bit rows a mixed-precision FMA
// (x * 1 + acc in fp32, the product exact) adds each element without a separate conversion.
template <typename T> __device__ __forceinline__ float add_lo_hi(uint32_t w, float &hi_acc, float lo_acc);
template <> __device__ __forceinline__ float add_lo_hi<__half>(uint32_t w, float &hi_acc, float lo_acc) {
    asm("{\n\t.reg .b16 l, h, one;\n\tmov.b32 {l, h}, %2;\n\tmov.b16 one, 0x3C00;\n\t"
        "fma.rn.f32.f16 %0, l, one, %0;\n\tfma.rn.f32.f16 %1, h, one, %1;\n\t}"
        : "+f"(lo_acc), "+f"(hi_acc) : "r"(w));
    return lo_acc;
}
template <> __device__ __forceinline__ float add_lo_hi<__nv_bfloat16>(uint32_t w, float &hi_acc, float lo_acc) {
    asm("{\n\t.reg .b16 l, h, one;\n\tmov.b32 {l, h}, %2;\n\tmov.b16 one, 0x3F80;\n\t"
        "fma.rn.f32.bf16 %0, l, one, %0;\n\tfma.rn.f32.bf16 %1, h, one, %1;\n\t}"
        : "+f"(lo_acc), "+f"(hi_acc) : "r"(w));
    return lo_acc;
}
template <typename T, int V>
__device__ __forceinline__ void row_add(const uint8_t *row, int lane, float (&acc)[V]) {
    if constexpr (sizeof(T) == 2) {
        using U = typename RowLd<T, V>::U;
        const U u = reinterpret_cast<const U *>(row)[lane];
        const uint32_t *w = reinterpret_cast<const uint32_t *>(&u);
#pragma unroll
        for (int e = 0; e < V / 2; ++e) acc[2 * e] = add_lo_hi<T>(w[e], acc[2 * e + 1], acc[2 * e]);
    } else {
        float x[V];
        row_vals<T, V>(row, lane, x);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += x[e];
    }
}

// C_new (and optionally Cx, ||Cx||^2, the weight sum) of cluster row `row` from its sums.
template <typename T, int V>
__device__ __forceinline__ void finalize_one(const FinalParams &p, int64_t row, int lane,
                                             const float (&acc)[V], float wacc, int cnt,
                                             bool weighted) {
    constexpr int D = 32 * V;
    const float div = weighted ? wacc : static_cast<float>(cnt);
    const bool upd = cnt > 0 && div > 0.f;
    const int64_t e0 = row * D + lane * V;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < V; ++e) {
        const float v = upd ? acc[e] / div : p.C_prev[e0 + e];
        p.C_new[e0 + e] = v;
        if (p.Cx) {
            const T t = Cvt<T>::from_f(v);
            static_cast<T *>(p.Cx)[e0 + e] = t;
            const float f = Cvt<T>::to_f(t);
            s = fmaf(f, f, s);
        }
    }
    if (p.cn) {
        s = warp_sum(s);
        if (lane == 0) p.cn[row] = s;
    }
    if (p.wsum && lane == 0) p.wsum[row] = wacc;
}

// The moving-average step of e-means for cluster row `row` with batch sums s, size n (count,
// or weight sum) and point count cnt. The state is (C, Nc) with S = C * Nc (the two are equal
// at the start, after every step and after a split):
//     Nc' = (1 - a) Nc + a n,   C' = ((1 - a) Nc C + a s) / Nc'   (C kept when Nc' == 0);
// Cx and cn follow C', and the batch statistics are added to the epoch totals.
//
// The cluster's state before this batch (count, centroid slice, epoch sum slice) is loaded when
// the warp meets the cluster's first row, so the loads run under its accumulation; only the
// finalizing warp uses them and nothing writes them before that finalize.
template <int V>
struct EmaPre {
    float nold;
    float c[V], es[V];
};
template <typename T, int V>
__device__ __forceinline__ void ema_prefetch(const FinalParams &p, int64_t row, int lane, EmaPre<V> &q) {
    constexpr int D = 32 * V;
    const int64_t e0 = row * D + lane * V;
    q.nold = p.Nc[row];
#pragma unroll
    for (int e = 0; e < V; ++e) {
        q.c[e] = p.C_new[e0 + e];
        q.es[e] = p.eS ? p.eS[e0 + e] : 0.f;
    }
}

template <typename T, int V>
__device__ __forceinline__ void finalize_ema(const FinalParams &p, int64_t row, int lane,
                                             const float (&s)[V], float wacc, int cnt,
                                             bool weighted, const EmaPre<V> &q) {
    constexpr int D = 32 * V;
    const float a = p.alpha, a1 = 1.f - a;
    const float n = weighted ? wacc : static_cast<float>(cnt);
    const float nold = q.nold;
    const float nn = a1 * nold + a * n;
    const int64_t e0 = row * D + lane * V;
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < V; ++e) {
        const float c = q.c[e];
        const float v = nn > 0.f ? (a1 * nold * c + a * s[e]) / nn : c;
        p.C_new[e0 + e] = v;
        const T t = Cvt<T>::from_f(v);
        static_cast<T *>(p.Cx)[e0 + e] = t;
        const float f = Cvt<T>::to_f(t);
        sq = fmaf(f, f, sq);
        if (p.eS) p.eS[e0 + e] = q.es[e] + s[e];
    }
    sq = warp_sum(sq);
    if (lane == 0) {
        p.cn[row] = sq;
        p.Nc[row] = nn;
        p.eCnt[row] += cnt;
        if (p.eW) p.eW[row] += wacc;
    }
}

template <typename T, int V, bool WEIGHTED, bool EMA>
__global__ void __launch_bounds__(fz_warps(32 * V * sizeof(T)) * 32, 1)
    segreduce_final_kernel(const __grid_constant__ CUtensorMap tmX, const FinalParams p) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int D = 32 * V;
    constexpr int RB = D * static_cast<int>(sizeof(T));
    constexpr int NW = fz_warps(RB);
    constexpr int S = fz_stages(RB);
    constexpr uint32_t STAGE = FZ_CHUNK * RB;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[NW][S];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t ring = ((raw + 1023u) & ~1023u) + warp * S * STAGE;
    const uint8_t *ring_g = smem_raw + (ring - raw);
    const uint32_t bar0 = smem_u32(&bars[warp][0]);

    const int64_t gw = static_cast<int64_t>(blockIdx.x) * NW + warp;
    if (gw >= static_cast<int64_t>(p.B) * p.rpb) return;
    const int b = static_cast<int>(gw / p.rpb);
    const int r = static_cast<int>(gw % p.rpb);
    const int32_t *offb = p.offsets + static_cast<int64_t>(b) * (p.K + 1);
    const int p0 = r * p.range;
    const int p1 = min(offb[p.K], p0 + p.range);
    if (p0 >= p1) return;
    const int nchunks = (p1 - p0 + FZ_CHUNK - 1) / FZ_CHUNK;
    const int32_t *permb = p.perm + static_cast<int64_t>(b) * p.N;
    const float *wb = WEIGHTED ? p.w + static_cast<int64_t>(b) * p.xld + p.x0 : nullptr;
    const int64_t rowbase = static_cast<int64_t>(b) * p.K;
    const uint64_t pol = l2_policy_evict_first();

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    // point index of each lane's position in chunk c (-1 past the range)
    auto load_idx = [&](int c) {
        const int pos = p0 + FZ_CHUNK * c + lane;
        return (c < nchunks && pos < p1) ? permb[pos] : -1;
    };
    // gathers of chunk c's 32 rows into stage c % S (rows past the range repeat a valid one)
    auto issue = [&](int c, int idx) {
        const int first = __shfl_sync(FULL, idx, 0);
        const int row = b * p.xld + p.x0 + (idx >= 0 ? idx : first);
        const int q1 = __shfl_down_sync(FULL, row, 1);
        const int q2 = __shfl_down_sync(FULL, row, 2);
        const int q3 = __shfl_down_sync(FULL, row, 3);
        const uint32_t bar = bar0 + 8u * (c % S);
        if (lane == 0) mbar_arrive_expect_tx(bar, STAGE);
        __syncwarp();
        if ((lane & 3) == 0)
            tma_gather4(ring + (c % S) * STAGE + (lane >> 2) * 4 * RB, &tmX, bar, 0, row, q1, q2, q3, pol);
    };

    // segment holding p0: the largest k with offb[k] <= p0 (from the scatter's table when given)
    int lo = 0;
    if (p.rseg) {
        lo = p.rseg[gw];
    } else {
        int hi = p.K - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offb[mid] <= p0) lo = mid; else hi = mid - 1;
        }
    }
    // A window of 32 segment ends kept in registers: lane l holds offb[wbase + 1 + l] (INT_MAX
    // past K) and wstart = offb[wbase]. Positions only grow, so the window only slides forward
    // and the per-chunk lookup needs no memory access until a chunk passes its last end.
    int wbase = lo;
    int wstart = offb[wbase];
    int wend = wbase + 1 + lane <= p.K ? offb[wbase + 1 + lane] : INT_MAX;

    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    float wacc = 0.f;
    int acck = -1, seg_s = 0, seg_e = 0;
    EmaPre<V> pre;   // the moving-average form's prefetched cluster state

    auto flush = [&]() {
        const int cnt = seg_e - seg_s;
        if (seg_s >= p0 && seg_e <= p1) {   // the whole cluster lies in this range
            if constexpr (EMA) finalize_ema<T, V>(p, rowbase + acck, lane, acc, wacc, cnt, WEIGHTED, pre);
            else finalize_one<T, V>(p, rowbase + acck, lane, acc, wacc, cnt, WEIGHTED);
            return;
        }
        const int side = seg_s < p0 ? 0 : 1;
        const int64_t slot = (gw * 2 + side);
        float *sp = p.slots + slot * D + lane * V;
#pragma unroll
        for (int e = 0; e < V; ++e) sp[e] = acc[e];
        if (lane == 0) p.wslots[slot] = wacc;
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(p.arrive + rowbase + acck, 1);
        old = __shfl_sync(FULL, old, 0);
        const int r0 = seg_s / p.range, r1 = (seg_e - 1) / p.range;
        if (old != r1 - r0) return;        // not the last range of this segment to arrive
        __threadfence();
        float tot[V];
#pragma unroll
        for (int e = 0; e < V; ++e) tot[e] = 0.f;
        float wt = 0.f;
        for (int rr = r0; rr <= r1; ++rr) {
            const int64_t sl = (static_cast<int64_t>(b) * p.rpb + rr) * 2 + (rr == r0 ? 1 : 0);
            const float *q = p.slots + sl * D + lane * V;
#pragma unroll
            for (int e = 0; e < V; ++e) tot[e] += __ldcg(q + e);
            wt += __ldcg(p.wslots + sl);
        }
        if constexpr (EMA) finalize_ema<T, V>(p, rowbase + acck, lane, tot, wt, cnt, WEIGHTED, pre);
        else finalize_one<T, V>(p, rowbase + acck, lane, tot, wt, cnt, WEIGHTED);
    };

    // prologue: S - 1 chunks in flight; qi[j] holds the point indices of chunk c + j (loaded
    // two iterations before their gathers are issued)
    constexpr int Q = S + 1;
    int qi[Q];
#pragma unroll
    for (int j = 0; j < Q; ++j) qi[j] = load_idx(j);
#pragma unroll
    for (int j = 0; j < S - 1; ++j)
        if (j < nchunks) issue(j, qi[j]);
    uint32_t phase_bits = 0;   // bit s: parity of the next completion of stage s

    for (int c = 0; c < nchunks; ++c) {
        const int slot_c = c % S;
        const int my_i = qi[0];
        // refill: chunk c + S - 1 goes into the stage chunk c - 1 used (read and fenced below)
        if (c + S - 1 < nchunks) issue(c + S - 1, qi[S - 1]);
        float my_w = 1.f;
        if constexpr (WEIGHTED) my_w = my_i >= 0 ? wb[my_i] : 0.f;
        const int q = p0 + FZ_CHUNK * c;
        const int nrows = min(FZ_CHUNK, p1 - q);
        // clusters of the chunk's positions: segment of pl = wbase + #{j : offb[wbase+1+j] <= pl},
        // with the segment bounds [my_s, my_e) taken from the window by shuffles
        const int pl = min(q + lane, p1 - 1);
        int my_k = -1, my_s = 0, my_e = 0;
        while (true) {
            int cnt = 0;
#pragma unroll
            for (int stp = 16; stp > 0; stp >>= 1) {
                const int pr = __shfl_sync(FULL, wend, cnt + stp - 1);
                if (pr <= pl) cnt += stp;
            }
            const int w31 = __shfl_sync(FULL, wend, 31);
            if (cnt == 31 && w31 <= pl) cnt = 32;
            const int e_here = __shfl_sync(FULL, wend, cnt & 31);
            const int s_here = __shfl_sync(FULL, wend, (cnt + 31) & 31);
            if (my_k < 0 && cnt < 32) {
                my_k = wbase + cnt;
                my_e = e_here;
                my_s = cnt == 0 ? wstart : s_here;
            }
            if (!__any_sync(FULL, my_k < 0)) break;
            // some position lies past the window: slide it by 32 segments
            wbase += 32;
            wstart = w31;
            wend = wbase + 1 + lane <= p.K ? offb[wbase + 1 + lane] : INT_MAX;
        }
        int prev_k = __shfl_up_sync(FULL, my_k, 1);
        if (lane == 0) prev_k = acck;
        const unsigned starts = __ballot_sync(FULL, lane < nrows && my_k != prev_k);
        // the indices of the chunk issued two iterations from now
#pragma unroll
        for (int j = 0; j + 1 < Q; ++j) qi[j] = qi[j + 1];
        qi[Q - 1] = load_idx(c + Q);

        if (!mbar_wait_warp(bar0 + 8u * slot_c, (phase_bits >> slot_c) & 1u, nullptr)) {
            // the wait ran out (recorded in the device error word): let every gather issued so
            // far land (each wait bounded again) before the CTA's shared memory goes away
            for (int cc = c; cc < min(nchunks, c + S); ++cc)
                mbar_wait_warp(bar0 + 8u * (cc % S), static_cast<uint32_t>((cc / S) & 1), nullptr);
            return;
        }
        phase_bits ^= 1u << slot_c;
        const uint8_t *stage = ring_g + slot_c * STAGE;
        // run by run: rows [rr, re) belong to one cluster (all warp-uniform)
        for (int rr = 0; rr < nrows;) {
            if ((starts >> rr) & 1u) {
                if (acck >= 0) flush();
                acck = __shfl_sync(FULL, my_k, rr);
                seg_s = __shfl_sync(FULL, my_s, rr);
                seg_e = __shfl_sync(FULL, my_e, rr);
                if constexpr (EMA) ema_prefetch<T, V>(p, rowbase + acck, lane, pre);
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] = 0.f;
                wacc = 0.f;
            }
            const unsigned later = rr < 31 ? starts & (~0u << (rr + 1)) : 0u;
            const int re = later ? min(nrows, __ffs(later) - 1) : nrows;
            if constexpr (WEIGHTED) {
                for (; rr < re; ++rr) {
                    const float wv = __shfl_sync(FULL, my_w, rr);
                    float x[V];
                    row_vals<T, V>(stage + rr * RB, lane, x);
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = fmaf(wv, x[e], acc[e]);
                    wacc += wv;
                }
            } else {
                wacc += static_cast<float>(re - rr);
#pragma unroll 4
                for (; rr < re; ++rr) row_add<T, V>(stage + rr * RB, lane, acc);
            }
        }
        // this stage's reads are done before the engine writes it again
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
    }
    if (acck >= 0) flush();
}

// Per batch element (one block): offsets[b, 0..K] and cursor[b, k] as scan_kernel, the arrival
// counters of segreduce_final_kernel zeroed, and the outputs of every empty cluster written
// (C_new = C_prev, its rounding, norm and a zero weight sum). In the moving-average form (Nc
// given) a cluster without points in the batch only decays its count, Nc <- (1 - alpha) Nc: its
// centroid (S / Nc with both decayed) and so Cx and cn stay as they are.
template <typename T>
__global__ void __launch_bounds__(SCAN_THREADS)
    scan_final_kernel(const int32_t *__restrict__ counts, int K, int d, int32_t *__restrict__ offsets,
                      int32_t *__restrict__ cursor, int32_t *__restrict__ arrive, const float *C_prev,
                      float *C_new, T *__restrict__ Cx, float *__restrict__ cn, float *__restrict__ wsum,
                      float *__restrict__ Nc, float alpha) {
    __shared__ int wtot[SCAN_THREADS / 32];
    __shared__ int elist[4 * SCAN_THREADS];   // empty clusters of one pass over 4096 counts
    __shared__ int ecount;
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int32_t *cb = counts + static_cast<int64_t>(b) * K;
    int32_t *ob = offsets + static_cast<int64_t>(b) * (K + 1);
    int32_t *cur = cursor + static_cast<int64_t>(b) * K;
    int32_t *ar = arrive + static_cast<int64_t>(b) * K;
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
        unsigned empty = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (k0 + e < K) {
                ob[k0 + e] = ex;
                cur[k0 + e] = ex;
                ar[k0 + e] = 0;
                if (v[e] == 0) empty |= 1u << e;
            }
            ex += v[e];
        }
        if (Nc) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((empty >> e) & 1u) Nc[static_cast<int64_t>(b) * K + k0 + e] *= 1.f - alpha;
            empty = 0;
        }
        if (tid == 0) ecount = 0;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if ((empty >> e) & 1u) elist[atomicAdd(&ecount, 1)] = k0 + e;
        __syncthreads();
        // an empty cluster keeps its centroid: one warp per listed row
        for (int i = wid; i < ecount; i += SCAN_THREADS / 32) {
            const int64_t row = static_cast<int64_t>(b) * K + elist[i];
            float s = 0.f;
            for (int j = lane; j < d; j += 32) {
                const float c = C_prev[row * d + j];
                C_new[row * d + j] = c;
                if (Cx) {
                    const T t = Cvt<T>::from_f(c);
                    Cx[row * d + j] = t;
                    const float f = Cvt<T>::to_f(t);
                    s = fmaf(f, f, s);
                }
            }
            if (cn) {
                s = warp_sum(s);
                if (lane == 0) cn[row] = s;
            }
            if (wsum && lane == 0) wsum[row] = 0.f;
        }
        carry += wtot[SCAN_THREADS / 32 - 1];
        __syncthreads();
    }
    if (tid == 0) ob[K] = carry;
}

// Exclusive scan in place of a[0..K) (shared, 16-byte aligned) by one block of TILE_THREADS
// threads; returns the total. 4 * TILE_THREADS entries per pass: thread t takes 4 consecutive
// entries with one 16-byte access (a warp reads 512 contiguous bytes: no bank conflicts).
__device__ __forceinline__ int block_exscan(int *a, int K, int *wtot) {
    constexpr int NW = TILE_THREADS / 32;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int carry = 0;
    for (int base = 0; base < K; base += 4 * TILE_THREADS) {
        const int kk = base + 4 * tid;
        int v[4];
        if (kk + 3 < K) {
            const int4 q = *reinterpret_cast<const int4 *>(a + kk);
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = kk + e < K ? a[kk + e] : 0;
        }
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
            int x = lane < NW ? wtot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane < NW) wtot[lane] = x;
        }
        __syncthreads();
        int ex = carry + incl - tsum + (wid > 0 ? wtot[wid - 1] : 0);
        int o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o4[e] = ex;
            ex += v[e];
        }
        if (kk + 3 < K) {
            *reinterpret_cast<int4 *>(a + kk) = make_int4(o4[0], o4[1], o4[2], o4[3]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (kk + e < K) a[kk + e] = o4[e];
        }
        carry += wtot[NW - 1];
        __syncthreads();
    }
    return carry;
}

// Each cluster present in a scatter tile gets its slot range: h[k] <- offs[k] + (old fill[k])
// - base[k] (base null: 0), with fill[k] += h[k]. A thread's clusters are taken eight at a time
// so that their atomics are in flight together instead of one round trip after another.
__device__ __forceinline__ void reserve_slots(int *h, const int *offs, const int *base,
                                              int32_t *__restrict__ fillb, int K, int tid) {
    constexpr int RB = 8;
    for (int k0 = tid; k0 < K; k0 += RB * TILE_THREADS) {
        int hv[RB], r[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int k = k0 + u * TILE_THREADS;
            hv[u] = k < K ? h[k] : 0;
        }
#pragma unroll
        for (int u = 0; u < RB; ++u) r[u] = hv[u] ? atomicAdd(fillb + k0 + u * TILE_THREADS, hv[u]) : 0;
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int k = k0 + u * TILE_THREADS;
            if (hv[u]) h[k] = offs[k] + r[u] - (base ? base[k] : 0);
        }
    }
}

// The counting-sort scatter with the scan folded in (K <= SMEM_K_MAX; tile <= SCATTER_PPT *
// TILE_THREADS, each thread keeping its points' labels in registers so the tile's histogram and
// ranking issue all their shared-memory atomics back to back). With K <= SCATTER_SORT_K_MAX the
// tile is first sorted by cluster in shared memory (a tile-local scan of its histogram, then
// cursors), and perm is written in that order: each cluster's run of the tile leaves as
// contiguous stores instead of one scattered 4-byte store per point. Shared memory: 2K + 1 ints,
// plus (sorted form) K + tile ints from a 16-byte boundary. Every block computes its problem's exclusive offsets of the counts in shared
// memory, reserves each cluster of its tile a slot range at offs[k] + atomicAdd(fill[b, k],
// h[k]) (fill zeroed beforehand) and ranks its points into it. The blocks of a problem also
// share the per-cluster work scan_final_kernel does: tile 0 writes offsets[b, 0..K]; each block
// zeroes the arrival counters of its share of the clusters and writes the outputs of the empty
// ones there (C_new = C_prev, Cx, cn, a zero weight sum; in the moving-average form only
// Nc <- (1 - alpha) Nc).
template <typename T>
__global__ void __launch_bounds__(TILE_THREADS)
    scatter_final_kernel(const int32_t *__restrict__ ids, const int32_t *__restrict__ counts, int N,
                         int K, int d, int tile, int32_t *__restrict__ fill,
                         int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                         int32_t *__restrict__ arrive, const float *C_prev, float *C_new,
                         T *__restrict__ Cx, float *__restrict__ cn, float *__restrict__ wsum,
                         float *__restrict__ Nc, float alpha, int range, int rpb,
                         int32_t *__restrict__ rseg) {
    constexpr int NW = TILE_THREADS / 32;
    extern __shared__ __align__(16) int ssm[];
    int *offs = ssm;             // [K + 1]: the counts, then their exclusive prefix
    int *h = ssm + K + 1;        // [K]: the tile's histogram, then its reserved slots
    const bool sorted_form = K <= SCATTER_SORT_K_MAX;
    int *lofs = ssm + ((2 * K + 1 + 3) & ~3);   // [K] (sorted form): the histogram's prefix, then cursors
    int *srt = lofs + K;                        // [tile] (sorted form): (cluster, point) by cluster
    __shared__ int wtot[NW];
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int t0 = blockIdx.x * tile;
    const int t1 = min(N, t0 + tile);
    const int64_t kb = static_cast<int64_t>(b) * K;
    const int32_t *idb = ids + static_cast<int64_t>(b) * N;
    // this thread's points t0 + tid + m * TILE_THREADS: labels loaded first, all in flight
    int lab[SCATTER_PPT];
#pragma unroll
    for (int m = 0; m < SCATTER_PPT; ++m) {
        const int i = t0 + tid + m * TILE_THREADS;
        lab[m] = i < t1 ? idb[i] : -1;
    }
    for (int k = tid; k < K; k += TILE_THREADS) {
        offs[k] = counts[kb + k];
        h[k] = 0;
    }
    __syncthreads();
    const int total = block_exscan(offs, K, wtot);
    if (tid == 0) offs[K] = total;
    // the tile's histogram
#pragma unroll
    for (int m = 0; m < SCATTER_PPT; ++m)
        if (static_cast<unsigned>(lab[m]) < static_cast<unsigned>(K)) atomicAdd(&h[lab[m]], 1);
    __syncthreads();
    // this problem's offsets and range-start table: every tile holds the whole scan, so with many
    // clusters (the unsorted form) the tiles share the writing, else tile 0 does it alone
    const int kb0 = static_cast<int>(static_cast<int64_t>(K) * blockIdx.x / gridDim.x);
    const int kb1 = static_cast<int>(static_cast<int64_t>(K) * (blockIdx.x + 1) / gridDim.x);
    const bool share = !sorted_form;
    const int ok0 = share ? kb0 : (blockIdx.x == 0 ? 0 : K), ok1 = share ? kb1 : K;
    for (int k = ok0 + tid; k < ok1; k += TILE_THREADS) offsets[static_cast<int64_t>(b) * (K + 1) + k] = offs[k];
    if (blockIdx.x == (share ? gridDim.x - 1 : 0) && tid == 0) offsets[static_cast<int64_t>(b) * (K + 1) + K] = offs[K];
    // the segment holding the first position of each range of the reduction that follows
    const int rb0 = share ? static_cast<int>(static_cast<int64_t>(rpb) * blockIdx.x / gridDim.x)
                          : (blockIdx.x == 0 ? 0 : rpb);
    const int rb1 = share ? static_cast<int>(static_cast<int64_t>(rpb) * (blockIdx.x + 1) / gridDim.x) : rpb;
    for (int r = rb0 + tid; r < rb1; r += TILE_THREADS) {
        const int p0 = r * range;
        int lo = 0, hi = K - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offs[mid] <= p0) lo = mid; else hi = mid - 1;
        }
        rseg[static_cast<int64_t>(b) * rpb + r] = lo;
    }
    for (int k = kb0 + tid; k < kb1; k += TILE_THREADS) {
        arrive[kb + k] = 0;
        if (Nc && offs[k + 1] == offs[k]) Nc[kb + k] *= 1.f - alpha;
    }
    if (!Nc) {
        for (int k = kb0 + wid; k < kb1; k += NW) {   // empty clusters keep their centroid
            if (offs[k + 1] != offs[k]) continue;
            const int64_t row = kb + k;
            float s = 0.f;
            for (int j = lane; j < d; j += 32) {
                const float c = C_prev[row * d + j];
                C_new[row * d + j] = c;
                if (Cx) {
                    const T t = Cvt<T>::from_f(c);
                    Cx[row * d + j] = t;
                    const float f = Cvt<T>::to_f(t);
                    s = fmaf(f, f, s);
                }
            }
            if (cn) {
                s = warp_sum(s);
                if (lane == 0) cn[row] = s;
            }
            if (wsum && lane == 0) wsum[row] = 0.f;
        }
    }
    int32_t *pb = perm + static_cast<int64_t>(b) * N;
    if (sorted_form) {
        for (int k = tid; k < K; k += TILE_THREADS) lofs[k] = h[k];
        __syncthreads();
        const int nvalid = block_exscan(lofs, K, wtot);
        // each cluster's slot range, kept as (global slot - tile-local position)
        reserve_slots(h, offs, lofs, fill + kb, K, tid);
        __syncthreads();
#pragma unroll
        for (int m = 0; m < SCATTER_PPT; ++m)
            if (static_cast<unsigned>(lab[m]) < static_cast<unsigned>(K))
                srt[atomicAdd(&lofs[lab[m]], 1)] = (lab[m] << 13) | (tid + m * TILE_THREADS);
        __syncthreads();
        for (int lp = tid; lp < nvalid; lp += TILE_THREADS) {
            const int e = srt[lp];
            pb[lp + h[e >> 13]] = t0 + (e & 8191);
        }
        return;
    }
    // reserve each cluster of the tile a slot range, then rank the points into it
    reserve_slots(h, offs, nullptr, fill + kb, K, tid);
    __syncthreads();
    int pos[SCATTER_PPT];
#pragma unroll
    for (int m = 0; m < SCATTER_PPT; ++m)
        pos[m] = static_cast<unsigned>(lab[m]) < static_cast<unsigned>(K) ? atomicAdd(&h[lab[m]], 1) : -1;
#pragma unroll
    for (int m = 0; m < SCATTER_PPT; ++m)
        if (pos[m] >= 0) pb[pos[m]] = t0 + tid + m * TILE_THREADS;
}

}  // namespace upd
}  // namespace km
