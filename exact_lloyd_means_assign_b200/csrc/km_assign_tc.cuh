// km_assign_tc.cuh -- FlashAssign on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The assignment argmin_k ||x - c_k||^2 = argmin_k (||c_k||^2 - 2 <x, c_k>) is computed tile by
// tile: point tiles and centroid tiles stream from HBM/L2 into shared memory, the inner products
// are formed on the tensor cores, and a running (min, argmin) per point is kept in registers, so
// the N x K score matrix never reaches HBM (technologypulse.uk Flash-KMeans article,
// "Bottleneck 1"; wispaper blog "1. FlashAssign"; the online argmin is described there too).
// The pages' kernel is Triton on H200; this one is written for sm_100a:
//
//   * persistent CTAs, one per SM, each looping over (batch, 128-point tile) work items;
//   * warp 0: TMA producer. The point tile [128 x d] (double-buffered) and centroid tiles
//     [bn x 64] (a ring of `stages`) are loaded with 128-byte swizzling; centroid tiles carry an
//     L2 evict-last hint because every CTA re-reads them, point tiles evict-first;
//   * warp 1: allocates 512 TMEM columns and issues tcgen05.mma (M=128, N=bn, K=16, fp32
//     accumulate) into one of two 256-column accumulators, committing to mbarriers;
//   * warps 2..9: epilogue. TMEM lane quarter = warp % 4, column half = (warp - 2) / 4. Each
//     thread owns one point row: it loads 32 accumulator columns at a time (tcgen05.ld), forms
//     s = cn_k - 2 <x, c_k> with one FMA and keeps the running minimum and its index. The two
//     column halves of a row are merged at the end of the work item (lowest index on ties);
//     ||x||^2 is added only for the reported distance and inertia.
//
// All mbarrier waits are bounded (see km_common.cuh). On a timeout every role leaves its loop,
// the producer waits for the copies it issued, the MMA warp waits for its MMAs, TMEM is freed.
#pragma once

#include "km_common.cuh"

namespace km {
namespace tc {

constexpr int BM = 128;                    // points per tile (TMEM lanes)
constexpr int KC = 64;                     // 16-bit elements per 128-byte swizzle row
constexpr uint32_t XCHUNK = BM * 128;      // bytes of one [128 x 64] point chunk
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;       // TMEM columns between the two accumulators
constexpr int MAX_STAGES = 8;
constexpr uint32_t SMEM_LIMIT = 232448;    // 227 KB opt-in per block on sm_100
constexpr uint32_t SMEM_ATTR = SMEM_LIMIT - 1024;  // dynamic request cap (static smem is tiny)

struct Layout {
    uint32_t x_off, c_off, bar_off, slot_off, merge_off, total;
};

__host__ __device__ inline Layout make_layout(int nkc, int bn, int stages) {
    Layout L;
    L.x_off = 0;
    L.c_off = 2u * nkc * XCHUNK;
    L.bar_off = L.c_off + static_cast<uint32_t>(stages) * bn * 128u;
    const uint32_t nbar = 2 + 2 + 2 * stages + 2 + 2 + 1;
    L.slot_off = L.bar_off + nbar * 8u;
    L.merge_off = (L.slot_off + 16u + 15u) & ~15u;
    L.total = L.merge_off + 2u * BM * 8u;
    return L;
}

// Largest ring depth that fits the shared-memory budget (at least 2).
__host__ inline int pick_stages(int nkc, int bn) {
    int s = MAX_STAGES;
    while (s > 2 && make_layout(nkc, bn, s).total + 1024u > SMEM_ATTR) --s;
    return s;
}

struct Params {
    int B, N, K, d;
    int nkc;      // ceil(d / 64) chunks of the reduction dimension
    int bn;       // centroids per tile: 64, 128 or 256 (MMA N)
    int nct;      // centroid tiles: ceil(K / bn)
    int mtiles;   // point tiles per batch: ceil(N / 128)
    int stages;   // centroid ring depth
    int need_xn;  // 1 when the distance / inertia is requested
    uint32_t idesc;
    const float *cnp;  // [B, Kp] padded ||c||^2 (+inf beyond K)
    int Kp;
    const float *w;
    int32_t *ids;
    float *mind;
    double *inertia;
};

template <typename T>
__device__ __forceinline__ float row_sqnorm_swizzled(const uint8_t *row_base) {
    // A 128-byte row of 64 16-bit values; the swizzle only permutes 16-byte units within the
    // row, which does not change a sum of squares.
    const uint4 *rp = reinterpret_cast<const uint4 *>(row_base);
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint4 v = rp[u];
        const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            T lo, hi;
            const uint16_t l16 = static_cast<uint16_t>(wds[e] & 0xFFFFu);
            const uint16_t h16 = static_cast<uint16_t>(wds[e] >> 16);
            memcpy(&lo, &l16, 2);
            memcpy(&hi, &h16, 2);
            const float a = Cvt<T>::to_f(lo), c = Cvt<T>::to_f(hi);
            s = fmaf(a, a, s);
            s = fmaf(c, c, s);
        }
    }
    return s;
}

template <typename T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ int abort_flag;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const Layout L = make_layout(p.nkc, p.bn, p.stages);
    const int S = p.stages;
    const uint32_t bar0 = sbase + L.bar_off;
    // barrier addresses
    auto X_FULL = [&](int i) { return bar0 + 8u * i; };
    auto X_EMPTY = [&](int i) { return bar0 + 8u * (2 + i); };
    auto C_FULL = [&](int s) { return bar0 + 8u * (4 + s); };
    auto C_EMPTY = [&](int s) { return bar0 + 8u * (4 + S + s); };
    auto ACC_FULL = [&](int i) { return bar0 + 8u * (4 + 2 * S + i); };
    auto ACC_EMPTY = [&](int i) { return bar0 + 8u * (6 + 2 * S + i); };
    const uint32_t DRAIN = bar0 + 8u * (8 + 2 * S);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abortp = &abort_flag;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(X_FULL(i), 1);
            mbar_init(X_EMPTY(i), 1 + (p.need_xn ? BM : 0));
            mbar_init(ACC_FULL(i), 1);
            mbar_init(ACC_EMPTY(i), NUM_EPI_WARPS * 32);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(C_FULL(s), 1);
            mbar_init(C_EMPTY(s), 1);
        }
        mbar_init(DRAIN, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(sbase + L.slot_off, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(sgen + L.slot_off);
    const int total = p.B * p.mtiles;
    const uint32_t cstage_bytes = static_cast<uint32_t>(p.bn) * 128u;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_first();
            const uint64_t pol_c = l2_policy_evict_last();
            int stage = 0;
            uint32_t cph = 0;
            long long n_c = 0;
            int n_x = 0;
            bool ok = true;
            int local = 0;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++local) {
                const int b = t / p.mtiles, m0 = (t % p.mtiles) * BM;
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                if (!mbar_wait(X_EMPTY(xb), xph ^ 1u, abortp)) { ok = false; break; }
                mbar_arrive_expect_tx(X_FULL(xb), p.nkc * XCHUNK);
                for (int kc = 0; kc < p.nkc; ++kc)
                    tma_load_3d(sbase + L.x_off + (xb * p.nkc + kc) * XCHUNK, &tmX, X_FULL(xb),
                                kc * KC, m0, b, pol_x);
                ++n_x;
                for (int j = 0; j < p.nct && ok; ++j) {
                    for (int kc = 0; kc < p.nkc; ++kc) {
                        if (!mbar_wait(C_EMPTY(stage), cph ^ 1u, abortp)) { ok = false; break; }
                        mbar_arrive_expect_tx(C_FULL(stage), cstage_bytes);
                        tma_load_3d(sbase + L.c_off + stage * cstage_bytes, &tmC, C_FULL(stage),
                                    kc * KC, j * p.bn, b, pol_c);
                        ++n_c;
                        if (++stage == S) { stage = 0; cph ^= 1u; }
                    }
                }
            }
            if (!ok) {
                // Let every copy issued by this CTA land before its shared memory is released.
                for (int s = 0; s < S; ++s) {
                    const long long uses = n_c > s ? (n_c - 1 - s) / S + 1 : 0;
                    if (uses) mbar_wait(C_FULL(s), static_cast<uint32_t>((uses - 1) & 1), nullptr);
                }
                for (int i = 0; i < 2; ++i) {
                    const int uses = n_x > i ? (n_x - 1 - i) / 2 + 1 : 0;
                    if (uses) mbar_wait(X_FULL(i), static_cast<uint32_t>((uses - 1) & 1), nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t cph = 0;
            int abuf = 0;
            uint32_t aph = 0;
            bool ok = true;
            int local = 0;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++local) {
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                if (!mbar_wait(X_FULL(xb), xph, abortp)) { ok = false; break; }
                tc_fence_after();
                for (int j = 0; j < p.nct && ok; ++j) {
                    if (!mbar_wait(ACC_EMPTY(abuf), aph ^ 1u, abortp)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dcol = tmem_base + abuf * ACC_STRIDE;
                    for (int kc = 0; kc < p.nkc; ++kc) {
                        if (!mbar_wait(C_FULL(stage), cph, abortp)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t xa = sbase + L.x_off + (xb * p.nkc + kc) * XCHUNK;
                        const uint32_t ca = sbase + L.c_off + stage * cstage_bytes;
                        const int rem = p.d - kc * KC;
                        const int nk = rem >= KC ? 4 : (rem + 15) / 16;
                        for (int kk = 0; kk < nk; ++kk)
                            tc_mma_f16(dcol, sw128_kmajor_desc(xa + kk * 32),
                                       sw128_kmajor_desc(ca + kk * 32), p.idesc,
                                       (kc | kk) != 0 ? 1u : 0u);
                        tc_commit(C_EMPTY(stage));
                        if (++stage == S) { stage = 0; cph ^= 1u; }
                    }
                    if (!ok) break;
                    tc_commit(ACC_FULL(abuf));
                    abuf ^= 1;
                    if (abuf == 0) aph ^= 1u;
                }
                if (!ok) break;
                tc_commit(X_EMPTY(xb));
            }
            // Every MMA issued above completes before TMEM is released.
            tc_commit(DRAIN);
            mbar_wait(DRAIN, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int q = warp & 3;
        const int h = ew >> 2;
        const int row = q * 32 + lane;
        const int half = p.bn >> 1;
        const int nchunk = half >> 5;
        float *mval = reinterpret_cast<float *>(sgen + L.merge_off);
        int *midx = reinterpret_cast<int *>(sgen + L.merge_off + 2u * BM * 4u);
        int abuf = 0;
        uint32_t aph = 0;
        int local = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
            const int b = t / p.mtiles, m0 = (t % p.mtiles) * BM;
            const int xb = local & 1;
            const uint32_t xph = (local >> 1) & 1;
            bool ok = true;
            float xn = 0.f;
            if (p.need_xn && h == 0) {
                if (mbar_wait(X_FULL(xb), xph, abortp)) {
                    for (int kc = 0; kc < p.nkc; ++kc)
                        xn += row_sqnorm_swizzled<T>(sgen + L.x_off + (xb * p.nkc + kc) * XCHUNK +
                                                     row * 128);
                    mbar_arrive(X_EMPTY(xb));
                } else {
                    ok = false;
                }
            }
            float best = INFINITY;
            int bidx = 0;
            const float *cnb = p.cnp + static_cast<size_t>(b) * p.Kp;
            for (int j = 0; j < p.nct && ok; ++j) {
                if (!mbar_wait(ACC_FULL(abuf), aph, abortp)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                      abuf * ACC_STRIDE + h * half;
                for (int c = 0; c < nchunk; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tcol + c * 32, v);
                    tmem_wait_ld(v);
                    const int k0 = j * p.bn + h * half + c * 32;
                    const float4 *cp = reinterpret_cast<const float4 *>(cnb + k0);
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 cc = __ldg(cp + i4);
                        const float cv[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float s = fmaf(-2.f, __uint_as_float(v[4 * i4 + e]), cv[e]);
                            if (s < best) {
                                best = s;
                                bidx = k0 + 4 * i4 + e;
                            }
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(ACC_EMPTY(abuf));
                abuf ^= 1;
                if (abuf == 0) aph ^= 1u;
            }
            // Merge the two column halves of each row (both warps of a pair always reach this
            // barrier once per work item, then leave together if anything gave up).
            const int mb = (local & 1) * BM;
            if (h == 1) {
                mval[mb + row] = best;
                midx[mb + row] = bidx;
            }
            named_barrier_sync(1 + q, 64);
            if (*abortp) break;
            if (h == 0) {
                const float ob = mval[mb + row];
                const int oi = midx[mb + row];
                if (ob < best || (ob == best && oi < bidx)) {
                    best = ob;
                    bidx = oi;
                }
                const int i = m0 + row;
                double contrib = 0.0;
                if (i < p.N) {
                    const size_t gi = static_cast<size_t>(b) * p.N + i;
                    p.ids[gi] = bidx;
                    if (p.need_xn) {
                        const float md = fmaxf(0.f, xn + best);
                        if (p.mind) p.mind[gi] = md;
                        contrib = static_cast<double>(p.w ? p.w[gi] : 1.f) * static_cast<double>(md);
                    }
                }
                if (p.inertia) {
                    contrib = warp_sum(contrib);
                    if (lane == 0) atomicAdd(p.inertia + b, contrib);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace tc
}  // namespace km
