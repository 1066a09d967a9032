// km_assign_tc.cuh -- FlashAssign on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The assignment argmin_k ||x - c_k||^2 is computed tile by tile: point tiles and centroid tiles
// stream from HBM/L2 into shared memory, the tensor cores form the distances, and a running
// (min, argmin) per point is kept in registers, so the N x K distance matrix never reaches HBM
// (technologypulse.uk Flash-KMeans article, "Bottleneck 1"; wispaper blog "1. FlashAssign",
// online argmin). The pages' kernel is Triton on H200; this one is written for sm_100a.
//
// What the tensor cores compute. Per 128-point x bn-centroid tile the accumulator in TMEM is
//     acc[i,k] = -<x_i, c_k> + (||x_i||^2 / 2)~ + ||c_k||^2 / 2  =  d(i,k) / 2 - delta_i
// The first term is the main reduction (fp16/bf16 operands, the A operand negated through the
// instruction descriptor). The other two are one extra K=16 step with bf16 operands: the point
// side carries [x1, x2, 1, 1, 1, 0...] with x1 + x2 ~ ||x||^2 / 2 (delta_i is the rounding of that
// two-piece split, a constant per row that cannot change the argmin and is added back for the
// reported distance), the centroid side [1, 1, a, b, c, 0...] with a + b + c = ||c||^2 / 2 to about
// 2^-27 relative. Padding centroids carry 1e30 so they never win.
//
// Because the accumulator is (half) the distance itself, the epilogue can keep the argmin as a
// packed key: the low 5 mantissa bits are replaced by the column index within a 32-column chunk,
// and one three-input float min per two columns keeps both the minimum and its position (equal
// keys resolve to the lower index; values closer than 2^-18 relative resolve by index, far inside
// the near-tie band). Per score that is one LOP3 and half a FMNMX, instead of an FMA, a compare
// and two selects.
//
// Roles (persistent CTAs, one per SM, 10 warps):
//   warp 0   TMA producer: point tile [128 x d] double-buffered (L2 evict-first), centroid tiles
//            [bn x 64] through a ring of `stages` (L2 evict-last: every CTA re-reads them), and
//            the centroid augmentation [bn x 16] through a 2-slot ring; 128/32-byte swizzles.
//   warp 1   allocates 512 TMEM columns, issues tcgen05.mma (M=128, N=bn, K=16, fp32 accumulate)
//            into two 256-column accumulators, commits to mbarriers.
//   warps 2-9 epilogue. TMEM lane quarter = warp % 4, column half = (warp - 2) / 4; one point row
//            per thread. The h=0 warps also compute ||x||^2 from the swizzled point tile and write
//            the point-side augmentation row. TMEM loads are software-pipelined one chunk ahead
//            and the accumulator is released as soon as its last chunk is in registers.
//
// All mbarrier waits are bounded (km_common.cuh). On a timeout every role leaves its loop, the
// producer waits for the copies it issued, the MMA warp drains its MMAs, and TMEM is freed.
#pragma once

#include "km_common.cuh"

namespace km {
namespace tc {

constexpr int BM = 128;                     // points per tile (TMEM lanes)
constexpr int KC = 64;                      // 16-bit elements per 128-byte swizzle row
constexpr uint32_t XCHUNK = BM * 128;       // bytes of one [128 x 64] point chunk
constexpr uint32_t XAUG_BYTES = BM * 32;    // [128 x 16] bf16 point-side augmentation
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;        // TMEM columns between the two accumulators
constexpr int MAX_STAGES = 8;
constexpr int AUG_STAGES = 2;
constexpr uint32_t SMEM_LIMIT = 232448;     // 227 KB opt-in per block on sm_100
constexpr uint32_t SMEM_ATTR = SMEM_LIMIT - 1024;  // dynamic request cap (static smem is tiny)

struct Layout {
    uint32_t x_off, xaug_off, c_off, caug_off, bar_off, slot_off, merge_off, total;
};

__host__ __device__ inline Layout make_layout(int nkc, int bn, int stages) {
    Layout L;
    L.x_off = 0;
    L.xaug_off = 2u * nkc * XCHUNK;
    L.c_off = L.xaug_off + 2u * XAUG_BYTES;
    L.caug_off = L.c_off + static_cast<uint32_t>(stages) * bn * 128u;
    L.bar_off = L.caug_off + static_cast<uint32_t>(AUG_STAGES) * bn * 32u;
    const uint32_t nbar = 15 + 2 * stages;
    L.slot_off = L.bar_off + nbar * 8u;
    L.merge_off = (L.slot_off + 16u + 15u) & ~15u;
    L.total = L.merge_off + 2u * BM * 8u;
    return L;
}

// Largest centroid ring depth that fits the shared-memory budget (at least 2).
__host__ inline int pick_stages(int nkc, int bn) {
    int s = MAX_STAGES;
    while (s > 2 && make_layout(nkc, bn, s).total + 1024u > SMEM_ATTR) --s;
    return s;
}

struct Params {
    int B, N, K, d;
    int nkc;      // ceil(d / 64) chunks of the reduction dimension
    int nct;      // centroid tiles: Kp / bn
    int mtiles;   // point tiles per batch: ceil(N / 128)
    int stages;   // centroid ring depth
    int need_dist;  // 1 when the distance / inertia is requested
    uint32_t idesc_main, idesc_aug;
    const float *w;
    int32_t *ids;
    float *mind;
    double *inertia;
};

// Shared-memory descriptor, K-major, 32-byte swizzle: rows of 32 bytes (16 bf16 = one K=16
// step), 8-row groups 256 bytes apart, layout code 6 (SWIZZLE_32B).
__device__ __forceinline__ uint64_t sw32_kmajor_desc(uint32_t saddr) {
    uint64_t desc = 0;
    desc |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    desc |= static_cast<uint64_t>(1u) << 16;
    desc |= static_cast<uint64_t>(256u >> 4) << 32;
    desc |= static_cast<uint64_t>(1u) << 46;
    desc |= static_cast<uint64_t>(6u) << 61;
    return desc;
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
__global__ void __launch_bounds__(NUM_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmA, const Params p) {
    constexpr int HALF = BN / 2;
    constexpr int NCH = HALF / 32;
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
    auto CAUG_FULL = [&](int i) { return bar0 + 8u * (6 + i); };
    auto CAUG_EMPTY = [&](int i) { return bar0 + 8u * (8 + i); };
    auto ACC_FULL = [&](int i) { return bar0 + 8u * (10 + i); };
    auto ACC_EMPTY = [&](int i) { return bar0 + 8u * (12 + i); };
    const uint32_t DRAIN = bar0 + 8u * 14;
    auto C_FULL = [&](int s) { return bar0 + 8u * (15 + s); };
    auto C_EMPTY = [&](int s) { return bar0 + 8u * (15 + S + s); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int *abortp = &abort_flag;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(X_FULL(i), 1);
            mbar_init(X_EMPTY(i), 1 + BM);        // MMA commit + the 128 ||x||^2 readers
            mbar_init(XAUG_FULL(i), BM);
            mbar_init(CAUG_FULL(i), 1);
            mbar_init(CAUG_EMPTY(i), 1);
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
        tma_prefetch_desc(&tmA);
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
    constexpr uint32_t CSTAGE = BN * 128u;
    constexpr uint32_t ASTAGE = BN * 32u;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_first();
            const uint64_t pol_c = l2_policy_evict_last();
            int stage = 0, astage = 0;
            uint32_t cph = 0, aph = 0;
            long long n_c = 0, n_a = 0;
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
                        mbar_arrive_expect_tx(C_FULL(stage), CSTAGE);
                        tma_load_3d(sbase + L.c_off + stage * CSTAGE, &tmC, C_FULL(stage), kc * KC,
                                    j * BN, b, pol_c);
                        ++n_c;
                        if (++stage == S) { stage = 0; cph ^= 1u; }
                    }
                    if (!ok) break;
                    if (!mbar_wait(CAUG_EMPTY(astage), aph ^ 1u, abortp)) { ok = false; break; }
                    mbar_arrive_expect_tx(CAUG_FULL(astage), ASTAGE);
                    tma_load_3d(sbase + L.caug_off + astage * ASTAGE, &tmA, CAUG_FULL(astage), 0,
                                j * BN, b, pol_c);
                    ++n_a;
                    if (++astage == AUG_STAGES) { astage = 0; aph ^= 1u; }
                }
            }
            if (!ok) {
                // Let every copy issued by this CTA land before its shared memory is released.
                for (int s = 0; s < S; ++s) {
                    const long long uses = n_c > s ? (n_c - 1 - s) / S + 1 : 0;
                    if (uses) mbar_wait(C_FULL(s), static_cast<uint32_t>((uses - 1) & 1), nullptr);
                }
                for (int i = 0; i < AUG_STAGES; ++i) {
                    const long long uses = n_a > i ? (n_a - 1 - i) / AUG_STAGES + 1 : 0;
                    if (uses) mbar_wait(CAUG_FULL(i), static_cast<uint32_t>((uses - 1) & 1), nullptr);
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
            int stage = 0, astage = 0;
            uint32_t cph = 0, asph = 0;
            int abuf = 0;
            uint32_t aph = 0;
            bool ok = true;
            int local = 0;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++local) {
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                if (!mbar_wait(X_FULL(xb), xph, abortp)) { ok = false; break; }
                tc_fence_after();
                const uint32_t xaug = sbase + L.xaug_off + xb * XAUG_BYTES;
                for (int j = 0; j < p.nct && ok; ++j) {
                    if (!mbar_wait(ACC_EMPTY(abuf), aph ^ 1u, abortp)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dcol = tmem_base + abuf * ACC_STRIDE;
                    for (int kc = 0; kc < p.nkc; ++kc) {
                        if (!mbar_wait(C_FULL(stage), cph, abortp)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t xa = sbase + L.x_off + (xb * p.nkc + kc) * XCHUNK;
                        const uint32_t ca = sbase + L.c_off + stage * CSTAGE;
                        const int rem = p.d - kc * KC;
                        const int nk = rem >= KC ? 4 : (rem + 15) / 16;
                        for (int kk = 0; kk < nk; ++kk)
                            tc_mma_f16(dcol, sw128_kmajor_desc(xa + kk * 32),
                                       sw128_kmajor_desc(ca + kk * 32), p.idesc_main,
                                       (kc | kk) != 0 ? 1u : 0u);
                        tc_commit(C_EMPTY(stage));
                        if (++stage == S) { stage = 0; cph ^= 1u; }
                    }
                    if (!ok) break;
                    if (j == 0 && !mbar_wait(XAUG_FULL(xb), xph, abortp)) { ok = false; break; }
                    if (!mbar_wait(CAUG_FULL(astage), asph, abortp)) { ok = false; break; }
                    tc_fence_after();
                    tc_mma_f16(dcol, sw32_kmajor_desc(xaug),
                               sw32_kmajor_desc(sbase + L.caug_off + astage * ASTAGE), p.idesc_aug, 1u);
                    tc_commit(CAUG_EMPTY(astage));
                    if (++astage == AUG_STAGES) { astage = 0; asph ^= 1u; }
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
            float delta = 0.f;   // (||x||^2/2) minus its two-piece bf16 split, for this row
            if (h == 0) {
                if (mbar_wait(X_FULL(xb), xph, abortp)) {
                    float xn = 0.f;
                    for (int kc = 0; kc < p.nkc; ++kc)
                        xn += row_sqnorm_swizzled<T>(sgen + L.x_off + (xb * p.nkc + kc) * XCHUNK +
                                                     row * 128);
                    const float half_xn = 0.5f * xn;
                    const float x1 = __bfloat162float(__float2bfloat16_rn(half_xn));
                    const float x2 = __bfloat162float(__float2bfloat16_rn(half_xn - x1));
                    delta = (half_xn - x1) - x2;
                    // Row of the point-side augmentation in the 32-byte-swizzled layout: the two
                    // 16-byte halves of rows 4..7 of every 8-row group trade places.
                    const uint4 data = make_uint4(pack_bf16x2(x1, x2), pack_bf16x2(1.f, 1.f),
                                                  pack_bf16x2(1.f, 0.f), 0u);
                    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
                    uint8_t *rp = sgen + L.xaug_off + xb * XAUG_BYTES + row * 32;
                    const int sw = (row >> 2) & 1;
                    *reinterpret_cast<uint4 *>(rp + 16 * sw) = data;
                    *reinterpret_cast<uint4 *>(rp + 16 * (1 - sw)) = zero;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(XAUG_FULL(xb));
                    mbar_arrive(X_EMPTY(xb));
                } else {
                    ok = false;
                }
            }
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
                        mbar_arrive(ACC_EMPTY(abuf));
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

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace tc
}  // namespace km
