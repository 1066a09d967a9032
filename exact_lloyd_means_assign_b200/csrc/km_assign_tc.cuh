// km_assign_tc.cuh -- FlashAssign on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// one SM pair per tile (cta_group::2).
//
// The assignment argmin_k ||x - c_k||^2 is computed tile by tile: point tiles and centroid tiles
// stream from HBM/L2 into shared memory, the tensor cores form the distances, and a running
// (min, argmin) per point is kept in registers, so the N x K distance matrix never reaches HBM
// (technologypulse.uk Flash-KMeans article, "Bottleneck 1"; wispaper blog "1. FlashAssign",
// online argmin). The pages' kernel is Triton on H200; this one is written for sm_100a.
//
// What the tensor cores compute. Per 256-point x bn-centroid tile the accumulator in TMEM is
//     acc[i,k] = -<x_i, c_k> + (||x_i||^2 / 2)~ + ||c_k||^2 / 2  =  d(i,k) / 2 - delta_i
// The first term is the main reduction (fp16/bf16 operands, the A operand negated through the
// instruction descriptor). The other two are one extra K=16 step with bf16 operands: the point
// side carries [x1, x2, 1, 1, 1, 0...] with x1 + x2 ~ ||x||^2 / 2 (delta_i is the rounding of that
// two-piece split, a constant per row that cannot change the argmin and is added back for the
// reported distance), the centroid side [1, 1, a, b, c, 0...] with a + b + c = ||c||^2 / 2 to about
// 2^-27 relative. Padding centroids carry 1e30 so they never win.
//
// Because the accumulator is (half) the distance itself, the epilogue keeps the argmin as a
// packed key: the low 5 mantissa bits are replaced by the column index within a 32-column chunk,
// and one three-input float min per two columns keeps both the minimum and its position (equal
// keys resolve to the lower index; values closer than 2^-18 relative resolve by index, far inside
// the near-tie band). Per score: one LOP3 and half a FMNMX.
//
// SM pairs. A cluster of two CTAs runs one tcgen05.mma.cta_group::2 per K step: M = 256 points
// (128 per CTA, each CTA's rows in its own shared memory and its own TMEM lanes) by N = bn
// centroids (each CTA holds bn/2 of the centroid rows). Every SM therefore loads and feeds the
// tensor cores only half of each centroid tile. The even CTA (the leader) issues the MMAs and
// owns the "full" barriers; both CTAs' centroid loads complete on them (2-SM TMA form), and MMA
// completion is committed to both CTAs' barriers (multicast commit). No TMA load uses multicast.
//
// Keeping the tensor pipe fed. The MMA queue is shallow, so the issuing thread must not spend
// long between tiles: one ring stage holds a whole centroid tile (all K chunks plus its
// augmentation rows) behind one barrier, so a tile costs the MMA thread two barrier checks
// (accumulator free, operands landed; the first probe is non-blocking) and two commits around
// its MMAs, with descriptors formed by adding offsets to precomputed words. Point tiles come from
// their own producer warp, so the centroid stream never waits behind the epilogue.
//
// Roles per CTA (persistent clusters, 15 warps):
//   warp 0    centroid producer: own half of each centroid tile [bn/2 x d] and its augmentation
//             rows [bn/2 x 16] into one stage of a ring (L2 evict-last: every CTA re-reads them).
//   warp 1    TMEM allocation (512 columns, both CTAs); in the leader also the MMA issuer.
//   warps 2-9 epilogue: TMEM lane quarter = warp % 4, column half = (warp - 2) / 4; one point
//             row per thread; TMEM loads pipelined one chunk ahead; accumulator released as soon
//             as its last chunk is in registers.
//   warps 10-13 norms: ||x||^2 of the point tile as soon as it lands and the point-side
//             augmentation row, so the MMA never waits for the epilogue between work items.
//   warp 14   point producer: own point tile [128 x d], double-buffered (L2 evict-first).
//
// All mbarrier waits are bounded (km_common.cuh). On a timeout every role leaves its loop, the
// producers wait for the copies they issued, the leader drains its MMAs, the pair synchronises
// and TMEM is freed.
#pragma once

#include "km_common.cuh"

namespace km {
namespace tc {

constexpr int BM = 128;                     // points per CTA (TMEM lanes); 256 per pair
constexpr int KC = 64;                      // 16-bit elements per 128-byte swizzle row
constexpr uint32_t XCHUNK = BM * 128;       // bytes of one [128 x 64] point chunk
constexpr uint32_t XAUG_BYTES = BM * 32;    // [128 x 16] bf16 point-side augmentation
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_NORM_WARPS = 4;
constexpr int WARP_CPROD = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_EPI0 = 2;
constexpr int WARP_NORM0 = 10;
constexpr int WARP_XPROD = 14;
constexpr int NUM_THREADS = 32 * 15;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;        // TMEM columns between the two accumulators
constexpr int MAX_STAGES = 8;
constexpr uint32_t SMEM_LIMIT = 232448;     // 227 KB opt-in per block on sm_100
constexpr uint32_t SMEM_ATTR = SMEM_LIMIT - 1024;  // dynamic request cap (static smem is tiny)

// Bytes one CTA stages per centroid tile: nkc chunks of [bn/2 x 64] plus [bn/2 x 16] bf16.
__host__ __device__ inline uint32_t cstage_bytes(int nkc, int bn) {
    return static_cast<uint32_t>(nkc) * (bn / 2) * 128u + (bn / 2) * 32u;
}

struct Layout {
    uint32_t x_off, xaug_off, c_off, stage, bar_off, slot_off, merge_off, total;
};

__host__ __device__ inline Layout make_layout(int nkc, int bn, int stages) {
    Layout L;
    L.x_off = 0;
    L.xaug_off = 2u * nkc * XCHUNK;
    L.c_off = L.xaug_off + 2u * XAUG_BYTES;
    L.stage = (cstage_bytes(nkc, bn) + 1023u) & ~1023u;
    L.bar_off = L.c_off + static_cast<uint32_t>(stages) * L.stage;
    const uint32_t nbar = 11 + 2 * stages;
    L.slot_off = L.bar_off + nbar * 8u;
    L.merge_off = (L.slot_off + 16u + 15u) & ~15u;
    L.total = L.merge_off + 2u * BM * 8u;
    return L;
}

// Deepest centroid ring that fits the shared-memory budget; 0 when not even 2 stages fit.
__host__ inline int pick_stages(int nkc, int bn) {
    for (int s = MAX_STAGES; s >= 2; --s)
        if (make_layout(nkc, bn, s).total + 1024u <= SMEM_ATTR) return s;
    return 0;
}

struct Params {
    int B, N, K, d;
    int nkc;      // ceil(d / 64) chunks of the reduction dimension
    int nct;      // centroid tiles: Kp / bn
    int mtiles;   // 256-point pair tiles per batch: ceil(N / 256)
    int stages;   // centroid ring depth
    int need_dist;  // 1 when the distance / inertia is requested
    uint32_t idesc_main, idesc_aug;
    const float *w;
    int32_t *ids;
    float *mind;
    double *inertia;
};

// Upper 32 bits of a K-major shared-memory matrix descriptor (stride byte offset, version 1,
// layout code: 2 = 128-byte swizzle, 6 = 32-byte swizzle) and the constant part of the lower word
// (leading byte offset 16 B, unused for swizzled K-major layouts). The start address goes in the
// low 14 bits, in 16-byte units; stepping K by 16 elements inside a 128-byte row adds 2.
constexpr uint32_t DESC_HI_SW128 = (1024u >> 4) | (1u << 14) | (2u << 29);
constexpr uint32_t DESC_HI_SW32 = (256u >> 4) | (1u << 14) | (6u << 29);
constexpr uint32_t DESC_LO_LBO = 1u << 16;
__device__ __forceinline__ uint64_t make_desc(uint32_t addr16, uint32_t hi) {
    return (static_cast<uint64_t>(hi) << 32) | (DESC_LO_LBO | (addr16 & 0x3FFFu));
}

// ------------------------------------------------------------------ pair / cluster helpers

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// 2-SM tensor load: lands in this CTA's shared memory, completes on the leader's barrier.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *tm,
                                                 uint32_t leader_bar, int c0, int c1, int c2,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(tm), "r"(leader_bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when all MMAs issued so far
// by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair_self(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

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
__device__ __forceinline__ float tile_row_sqnorm(const uint8_t *xbuf, int nkc, int row) {
    float xn = 0.f;
    for (int kc = 0; kc < nkc; ++kc) xn += row_sqnorm_swizzled<T>(xbuf + kc * XCHUNK + row * 128);
    return xn;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint16_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return static_cast<uint32_t>(l) | (static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Distance bits with the low 5 mantissa bits replaced by the column index inside the chunk.
__device__ __forceinline__ float key(uint32_t v, uint32_t i) {
    return __uint_as_float((v & 0xFFFFFFE0u) | i);
}

// Minimum packed key of a 32-column chunk (four independent chains for ILP).
__device__ __forceinline__ float chunk_min(const uint32_t (&v)[32]) {
    float m[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const int o = 8 * g;
        float t = min3f(key(v[o], o), key(v[o + 1], o + 1), key(v[o + 2], o + 2));
        t = min3f(t, key(v[o + 3], o + 3), key(v[o + 4], o + 4));
        t = min3f(t, key(v[o + 5], o + 5), key(v[o + 6], o + 6));
        m[g] = fminf(t, key(v[o + 7], o + 7));
    }
    return fminf(min3f(m[0], m[1], m[2]), m[3]);
}

template <typename T, int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmA, const Params p) {
    constexpr int HALF = BN / 2;        // accumulator columns per epilogue column-half
    constexpr int NCH = HALF / 32;
    constexpr int CROWS = BN / 2;       // centroid rows each CTA stages per tile
    constexpr uint32_t CCHUNK = CROWS * 128u;   // one [bn/2 x 64] centroid chunk
    extern __shared__ uint8_t smem_raw[];
    __shared__ int abort_flag;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const Layout L = make_layout(p.nkc, BN, p.stages);
    const int S = p.stages;
    const uint32_t bar0 = sbase + L.bar_off;
    auto X_FULL = [&](int i) { return bar0 + 8u * i; };
    auto X_EMPTY = [&](int i) { return bar0 + 8u * (2 + i); };
    auto XAUG_FULL = [&](int i) { return bar0 + 8u * (4 + i); };
    auto ACC_FULL = [&](int i) { return bar0 + 8u * (6 + i); };
    auto ACC_EMPTY = [&](int i) { return bar0 + 8u * (8 + i); };
    const uint32_t DRAIN = bar0 + 8u * 10;
    auto C_FULL = [&](int s) { return bar0 + 8u * (11 + s); };
    auto C_EMPTY = [&](int s) { return bar0 + 8u * (11 + S + s); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    volatile int *abortp = &abort_flag;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(X_FULL(i), 1);
            // the leader's commit + own norm warps + own h=0 epilogue warps (distance readers)
            mbar_init(X_EMPTY(i), 1 + NUM_NORM_WARPS + NUM_EPI_WARPS / 2);
            mbar_init(XAUG_FULL(i), 2 * NUM_NORM_WARPS);      // (leader) norm warps of both CTAs
            mbar_init(ACC_FULL(i), 1);
            mbar_init(ACC_EMPTY(i), 2 * NUM_EPI_WARPS);       // (leader) epilogue warps of both
        }
        mbar_init(DRAIN, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(C_FULL(s), 1);
            mbar_init(C_EMPTY(s), 1);
        }
        fence_mbar_init();
    }
    if (warp == WARP_CPROD && lane == 0) {
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmA);
    }
    if (warp == WARP_XPROD && lane == 0) tma_prefetch_desc(&tmX);
    if (warp == WARP_MMA) {
        tmem_alloc_pair(sbase + L.slot_off, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // barriers of both CTAs initialised before any cross-CTA traffic
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(sgen + L.slot_off);
    const int total = p.B * p.mtiles;
    const int cluster_id = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;
    const uint32_t stage_tx = 2u * cstage_bytes(p.nkc, BN);   // both CTAs' halves of a tile

    if (warp == WARP_CPROD) {
        // ------------------------------------------------------------ centroid producer
        if (lane == 0) {
            const uint64_t pol_c = l2_policy_evict_last();
            int stage = 0;
            uint32_t cph = 0;
            long long n_c = 0;
            bool ok = true;
            for (int t = cluster_id; t < total && ok; t += nclusters) {
                const int b = t / p.mtiles;
                for (int j = 0; j < p.nct; ++j) {
                    const int crow = j * BN + static_cast<int>(rank) * CROWS;
                    if (!mbar_wait(C_EMPTY(stage), cph ^ 1u, abortp)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(C_FULL(stage), stage_tx);
                    const uint32_t sdst = sbase + L.c_off + stage * L.stage;
                    const uint32_t lbar = map_to_rank(C_FULL(stage), 0);
                    for (int kc = 0; kc < p.nkc; ++kc)
                        tma_load_3d_pair(sdst + kc * CCHUNK, &tmC, lbar, kc * KC, crow, b, pol_c);
                    tma_load_3d_pair(sdst + p.nkc * CCHUNK, &tmA, lbar, 0, crow, b, pol_c);
                    ++n_c;
                    if (++stage == S) { stage = 0; cph ^= 1u; }
                }
            }
            if (!ok && leader) {
                // Let every pair copy issued into the ring land before shared memory goes away.
                for (int s = 0; s < S; ++s) {
                    const long long uses = n_c > s ? (n_c - 1 - s) / S + 1 : 0;
                    if (uses) mbar_wait(C_FULL(s), static_cast<uint32_t>((uses - 1) & 1), nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == WARP_XPROD) {
        // ------------------------------------------------------------ point producer
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_first();
            int n_x = 0;
            bool ok = true;
            int local = 0;
            for (int t = cluster_id; t < total; t += nclusters, ++local) {
                const int b = t / p.mtiles;
                const int m0 = (t % p.mtiles) * (2 * BM) + static_cast<int>(rank) * BM;
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                if (!mbar_wait(X_EMPTY(xb), xph ^ 1u, abortp)) { ok = false; break; }
                mbar_arrive_expect_tx(X_FULL(xb), p.nkc * XCHUNK);
                for (int kc = 0; kc < p.nkc; ++kc)
                    tma_load_3d(sbase + L.x_off + (xb * p.nkc + kc) * XCHUNK, &tmX, X_FULL(xb),
                                kc * KC, m0, b, pol_x);
                ++n_x;
            }
            if (!ok) {
                for (int i = 0; i < 2; ++i) {
                    const int uses = n_x > i ? (n_x - 1 - i) / 2 + 1 : 0;
                    if (uses) mbar_wait(X_FULL(i), static_cast<uint32_t>((uses - 1) & 1), nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t cph = 0;
            int abuf = 0;
            uint32_t aph = 0;
            bool ok = true;
            int local = 0;
            const uint32_t cbase16 = (sbase + L.c_off) >> 4;
            const uint32_t stage16 = L.stage >> 4;
            const uint32_t cchunk16 = CCHUNK >> 4;
            for (int t = cluster_id; t < total && ok; t += nclusters, ++local) {
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                // both CTAs' point tiles have landed and their augmentation rows are written
                if (!mbar_wait(XAUG_FULL(xb), xph, abortp)) { ok = false; break; }
                const uint32_t x16 = (sbase + L.x_off + xb * p.nkc * XCHUNK) >> 4;
                const uint32_t xaug16 = (sbase + L.xaug_off + xb * XAUG_BYTES) >> 4;
                for (int j = 0; j < p.nct; ++j) {
                    if (!mbar_wait(ACC_EMPTY(abuf), aph ^ 1u, abortp)) { ok = false; break; }
                    tc_fence_after();   // the epilogue's TMEM reads of this buffer come first
                    if (!mbar_wait(C_FULL(stage), cph, abortp)) { ok = false; break; }
                    const uint32_t dcol = tmem_base + abuf * ACC_STRIDE;
                    const uint32_t c16 = cbase16 + stage * stage16;
                    uint32_t acc = 0;
                    for (int kc = 0; kc < p.nkc; ++kc) {
                        const int rem = p.d - kc * KC;
                        const int nk = rem >= KC ? 4 : (rem + 15) / 16;
                        for (int kk = 0; kk < nk; ++kk) {
                            tc_mma_pair(dcol, make_desc(x16 + kc * (XCHUNK >> 4) + kk * 2, DESC_HI_SW128),
                                        make_desc(c16 + kc * cchunk16 + kk * 2, DESC_HI_SW128),
                                        p.idesc_main, acc);
                            acc = 1;
                        }
                    }
                    tc_mma_pair(dcol, make_desc(xaug16, DESC_HI_SW32),
                                make_desc(c16 + p.nkc * cchunk16, DESC_HI_SW32), p.idesc_aug, 1u);
                    tc_commit_pair_both(C_EMPTY(stage));
                    tc_commit_pair_both(ACC_FULL(abuf));
                    if (++stage == S) { stage = 0; cph ^= 1u; }
                    abuf ^= 1;
                    if (abuf == 0) aph ^= 1u;
                }
                if (!ok) break;
                tc_commit_pair_both(X_EMPTY(xb));
            }
            // Every MMA issued above completes before TMEM is released.
            tc_commit_pair_self(DRAIN);
            mbar_wait(DRAIN, 0, nullptr);
        }
        __syncwarp();
    } else if (warp >= WARP_NORM0) {
        // ------------------------------------------------------------ norms (both CTAs)
        const int row = (warp - WARP_NORM0) * 32 + lane;
        int local = 0;
        for (int t = cluster_id; t < total; t += nclusters, ++local) {
            const int xb = local & 1;
            const uint32_t xph = (local >> 1) & 1;
            if (!mbar_wait(X_FULL(xb), xph, abortp)) break;
            const float half_xn =
                0.5f * tile_row_sqnorm<T>(sgen + L.x_off + xb * p.nkc * XCHUNK, p.nkc, row);
            const float x1 = __bfloat162float(__float2bfloat16_rn(half_xn));
            const float x2 = __bfloat162float(__float2bfloat16_rn(half_xn - x1));
            // Row of the point-side augmentation in the 32-byte-swizzled layout: the two 16-byte
            // halves of rows 4..7 of every 8-row group trade places.
            const uint4 data = make_uint4(pack_bf16x2(x1, x2), pack_bf16x2(1.f, 1.f),
                                          pack_bf16x2(1.f, 0.f), 0u);
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            uint8_t *rp = sgen + L.xaug_off + xb * XAUG_BYTES + row * 32;
            const int sw = (row >> 2) & 1;
            *reinterpret_cast<uint4 *>(rp + 16 * sw) = data;
            *reinterpret_cast<uint4 *>(rp + 16 * (1 - sw)) = zero;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_cluster(map_to_rank(XAUG_FULL(xb), 0));
                mbar_arrive(X_EMPTY(xb));
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - WARP_EPI0;
        const int q = warp & 3;
        const int h = ew >> 2;
        const int row = q * 32 + lane;
        float *mval = reinterpret_cast<float *>(sgen + L.merge_off);
        int *midx = reinterpret_cast<int *>(sgen + L.merge_off + 2u * BM * 4u);
        int abuf = 0;
        uint32_t aph = 0;
        int local = 0;
        for (int t = cluster_id; t < total; t += nclusters, ++local) {
            const int b = t / p.mtiles;
            const int m0 = (t % p.mtiles) * (2 * BM) + static_cast<int>(rank) * BM;
            const int xb = local & 1;
            const uint32_t xph = (local >> 1) & 1;
            bool ok = true;
            float best_v = INFINITY;
            int best_i = 0;
            for (int j = 0; j < p.nct && ok; ++j) {
                if (!mbar_wait(ACC_FULL(abuf), aph, abortp)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                      abuf * ACC_STRIDE + h * HALF;
                const int kbase = j * BN + h * HALF;
                uint32_t va[32], vb[32];
                tmem_ld_32x32b_x32(tcol, va);
                tmem_wait_ld(va);
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    uint32_t(&cur)[32] = (c & 1) ? vb : va;
                    uint32_t(&nxt)[32] = (c & 1) ? va : vb;
                    if (c + 1 < NCH) {
                        tmem_ld_32x32b_x32(tcol + (c + 1) * 32, nxt);
                    } else {
                        // every column of this accumulator is in registers: hand it back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(map_to_rank(ACC_EMPTY(abuf), 0));
                    }
                    const float m = chunk_min(cur);
                    const uint32_t mb = __float_as_uint(m);
                    const float mv = __uint_as_float(mb & 0xFFFFFFE0u);
                    if (mv < best_v) {
                        best_v = mv;
                        best_i = kbase + c * 32 + static_cast<int>(mb & 31u);
                    }
                    if (c + 1 < NCH) tmem_wait_ld(nxt);
                }
                abuf ^= 1;
                if (abuf == 0) aph ^= 1u;
            }
            // The reported distance adds back delta, the rounding of this row's two-piece
            // ||x||^2/2 split, recomputed from the point tile (still resident: X_EMPTY waits for
            // these warps too).
            float delta = 0.f;
            if (h == 0) {
                if (p.need_dist && ok && mbar_wait(X_FULL(xb), xph, abortp)) {
                    const float half_xn =
                        0.5f * tile_row_sqnorm<T>(sgen + L.x_off + xb * p.nkc * XCHUNK, p.nkc, row);
                    const float x1 = __bfloat162float(__float2bfloat16_rn(half_xn));
                    const float x2 = __bfloat162float(__float2bfloat16_rn(half_xn - x1));
                    delta = (half_xn - x1) - x2;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(X_EMPTY(xb));
            }
            // Merge the two column halves of each row (both warps of a pair always reach this
            // barrier once per work item, then leave together if anything gave up).
            const int mb2 = (local & 1) * BM;
            if (h == 1) {
                mval[mb2 + row] = best_v;
                midx[mb2 + row] = best_i;
            }
            named_barrier_sync(1 + q, 64);
            if (*abortp) break;
            if (h == 0) {
                const float ob = mval[mb2 + row];
                const int oi = midx[mb2 + row];
                if (ob < best_v || (ob == best_v && oi < best_i)) {
                    best_v = ob;
                    best_i = oi;
                }
                const int i = m0 + row;
                double contrib = 0.0;
                if (i < p.N) {
                    const size_t gi = static_cast<size_t>(b) * p.N + i;
                    p.ids[gi] = best_i;
                    if (p.need_dist) {
                        const float md = fmaxf(0.f, 2.f * (best_v + delta));
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

    // Both CTAs are done with each other's barriers and the leader's MMAs have drained.
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == WARP_MMA) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace tc
}  // namespace km
