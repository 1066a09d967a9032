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
// side carries [x1, x2, 1, 1, 1, 0...] with x1 + x2 ~ (1 + 2^-12) ||x||^2 / 2 (delta_i, minus the
// raise and the rounding of that two-piece split, is a constant per row that cannot change the
// argmin and is added back for the reported distance; the raise keeps the accumulator positive),
// the centroid side [1, 1, a, b, c, 0...] with a + b + c = ||c||^2 / 2 to about
// 2^-27 relative. Padding centroids carry 1e30 so they never win.
//
// Because the accumulator is (half) the distance itself, the epilogue keeps the argmin as a
// packed key: the low log2(W) mantissa bits (W = columns one warp reads per tile, at most 64)
// are replaced by the column index, and one three-input float min per two columns keeps both
// the minimum and its position (equal keys resolve to the lower index; values closer than 2^-17
// relative resolve by index, far inside the near-tie band). Per score: one LOP3 and half a FMNMX.
//
// SM pairs. A cluster of two CTAs runs one tcgen05.mma.cta_group::2 per K step: M = 256 points
// (128 per CTA, each CTA's rows in its own shared memory and its own TMEM lanes) by N = bn
// centroids (each CTA holds bn/2 of the centroid rows). Every SM therefore loads and feeds the
// tensor cores only half of each centroid tile. The even CTA (the leader) issues the MMAs and
// owns the "full" barriers; both CTAs' centroid loads complete on them (2-SM TMA form), and MMA
// completion is committed to both CTAs' barriers (multicast commit). No TMA load uses multicast.
//
// Keeping the tensor pipe fed. The MMA queue holds only a couple of instructions, so whatever
// the issuing warp does between the last MMA of one tile and the first of the next is a bubble.
// That gap is kept to one commit: a ring stage holds a whole centroid tile behind one barrier,
// and the stage and the point buffer are handed back by the epilogue (which has seen the tile's
// completion) rather than by further commits. An MMA warp runs converged and issues from one
// elected lane, so its addresses and descriptors stay warp-uniform.
//
// Keeping the epilogue off the critical path. TMEM loads have a long latency, so each epilogue
// warp issues all of its columns of a tile at once (one wait per tile) and sixteen warps share
// the accumulator: four TMEM lane quarters x four column quarters. The accumulator is released
// as soon as the registers hold it; the min/argmin math runs while the next tile is computed.
//
// Issuing MMAs costs the SM sub-partition that hosts the issuing warp a large share of its
// issue slots (measured: the epilogue warps beside it finish their tiles last), so two warps
// on different sub-partitions take turns: tile j is issued by the warp that owns accumulator
// j % 2.
//
// Roles per CTA (persistent clusters, 20 warps: five per SM sub-partition, which leaves 96
// registers per thread):
//   warp 0      centroid producer: own half of each centroid tile [bn/2 x d] and its augmentation
//               rows [bn/2 x 16] into one stage of a ring (L2 evict-last: every CTA re-reads them).
//   warp 1      TMEM allocation (512 columns, both CTAs); in the leader the MMA issuer for even
//               tiles (accumulator 0).
//   warp 2      point producer: own point tile [128 x d], double-buffered (L2 evict-first); then
//               ||x||^2 of the tile as soon as it lands, the point-side augmentation rows and
//               delta, so the MMA never waits for the epilogue between work items.
//   warp 3      in the leader the MMA issuer for odd tiles (accumulator 1).
//   warps 4-19  epilogue: TMEM lane quarter = warp % 4, column quarter = (warp - 4) / 4; one point
//               row per thread.
//
// All mbarrier waits are bounded (km_common.cuh). On a timeout every role leaves its loop, the
// producers wait for the copies they issued, the leader drains its MMAs, the pair synchronises
// and TMEM is freed.
#pragma once

#include <utility>

#include "km_common.cuh"

namespace km {
namespace tc {

constexpr int BM = 128;                     // points per CTA (TMEM lanes); 256 per pair
constexpr int KC = 64;                      // 16-bit elements per 128-byte swizzle row
constexpr uint32_t XCHUNK = BM * 128;       // bytes of one [128 x 64] point chunk
constexpr uint32_t XAUG_BYTES = BM * 32;    // [128 x 16] bf16 point-side augmentation
constexpr int NUM_EPI_WARPS = 16;
constexpr int WARP_CPROD = 0;
constexpr int WARP_MMA = 1;       // even tiles (accumulator 0); allocates TMEM
constexpr int WARP_XPROD = 2;     // point tiles and their norms
constexpr int WARP_MMA_ODD = 3;   // odd tiles (accumulator 1)
constexpr int WARP_EPI0 = 4;
constexpr int NUM_THREADS = 32 * (WARP_EPI0 + NUM_EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;        // TMEM columns between the two accumulators
constexpr int MAX_STAGES = 8;
// Slots of the per-row norm roundings (delta): the point buffer is handed back as soon as the
// item's last accumulator is complete, before the epilogue reads the item's delta, so the
// producer may run two items ahead of that read.
constexpr uint32_t DELTA_SLOTS = 4;
constexpr uint32_t SMEM_LIMIT = 232448;     // 227 KB opt-in per block on sm_100
constexpr uint32_t SMEM_ATTR = SMEM_LIMIT - 1024;  // dynamic request cap (static smem is tiny)
constexpr int NUM_BARS_FIXED = 19;

// Bytes one CTA stages per centroid tile: nkc chunks of [bn/2 x 64] plus [bn/2 x 16] bf16.
__host__ __device__ inline uint32_t cstage_bytes(int nkc, int bn) {
    return static_cast<uint32_t>(nkc) * (bn / 2) * 128u + (bn / 2) * 32u;
}

struct Layout {
    uint32_t x_off, xaug_off, c_off, stage, bar_off, slot_off, delta_off, merge_off, total;
};

__host__ __device__ inline Layout make_layout(int nkc, int bn, int stages) {
    Layout L;
    L.x_off = 0;
    L.xaug_off = 2u * nkc * XCHUNK;
    L.c_off = L.xaug_off + 2u * XAUG_BYTES;
    L.stage = (cstage_bytes(nkc, bn) + 1023u) & ~1023u;
    L.bar_off = L.c_off + static_cast<uint32_t>(stages) * L.stage;
    const uint32_t nbar = NUM_BARS_FIXED + 2 * stages;
    L.slot_off = L.bar_off + nbar * 8u;
    L.delta_off = (L.slot_off + 16u + 15u) & ~15u;
    L.merge_off = L.delta_off + DELTA_SLOTS * BM * 4u;
    // per point buffer: three column quarters x 128 rows of (value, index)
    L.total = L.merge_off + 2u * 3u * BM * 8u;
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
    int resident; // 1 when stages == nct: centroid tiles stay in shared memory per batch element
    int need_dist;  // 1 when the distance / inertia is requested
    uint32_t idesc_main, idesc_aug;
    const float *w;
    int64_t wld;    // elements between the weights of consecutive batch elements (>= N)
    int32_t *ids;
    float *mind;
    double *inertia;
    int32_t *counts;   // per-cluster point counts (added to; zeroed by the host), or null
};

// Upper 32 bits of a K-major shared-memory matrix descriptor (stride byte offset, version 1,
// layout code: 2 = 128-byte swizzle, 6 = 32-byte swizzle) and the constant part of the lower word
// (leading byte offset 16 B, unused for swizzled K-major layouts). The start address goes in the
// low 14 bits, in 16-byte units; stepping K by 16 elements inside a 128-byte row adds 2.
constexpr uint32_t DESC_HI_SW128 = (1024u >> 4) | (1u << 14) | (2u << 29);
constexpr uint32_t DESC_HI_SW32 = (256u >> 4) | (1u << 14) | (6u << 29);
constexpr uint32_t DESC_LO_LBO = 1u << 16;
// Low descriptor word of a shared-memory address (16-byte units; shared memory is below 256 KB,
// so the 14-bit field never carries into the leading byte offset when offsets are added).
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr) { return DESC_LO_LBO | (saddr >> 4); }

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
// Remote arrive without release semantics (see mbar_arrive_relaxed).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
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
// Descriptors passed as (low, high) 32-bit words: only the low word (the start address) changes
// from one K step to the next.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                            uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
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

// s + lo^2 + hi^2 for the two 16-bit values of `w`, with fp32 accumulation. The square of a
// 16-bit float is exact in fp32, so this equals converting first and using fmaf; the
// mixed-precision FMA just needs no conversion instructions.
template <typename T> __device__ __forceinline__ float sq2_acc(uint32_t w, float s);
template <> __device__ __forceinline__ float sq2_acc<__half>(uint32_t w, float s) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\t"
        "fma.rn.f32.f16 %0, l, l, %0;\n\tfma.rn.f32.f16 %0, h, h, %0;\n\t}"
        : "+f"(s) : "r"(w));
    return s;
}
template <> __device__ __forceinline__ float sq2_acc<__nv_bfloat16>(uint32_t w, float s) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\t"
        "fma.rn.f32.bf16 %0, l, l, %0;\n\tfma.rn.f32.bf16 %0, h, h, %0;\n\t}"
        : "+f"(s) : "r"(w));
    return s;
}

template <typename T>
__device__ __forceinline__ float row_sqnorm_swizzled(const uint8_t *row_base, int row) {
    // A 128-byte row of 64 16-bit values; the 128-byte swizzle stores logical 16-byte unit u of
    // row r at position u ^ (r % 8), which a sum of squares does not care about. Reading the
    // units in that rotated order makes the 32 lanes (32 consecutive rows) of a warp touch all
    // 32 banks instead of the same 4. Four partial sums keep the FMA chains short.
    const uint4 *rp = reinterpret_cast<const uint4 *>(row_base);
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint4 v = rp[u ^ (row & 7)];
        s[0] = sq2_acc<T>(v.x, s[0]);
        s[1] = sq2_acc<T>(v.y, s[1]);
        s[2] = sq2_acc<T>(v.z, s[2]);
        s[3] = sq2_acc<T>(v.w, s[3]);
    }
    return (s[0] + s[1]) + (s[2] + s[3]);
}

template <typename T>
__device__ __forceinline__ float tile_row_sqnorm(const uint8_t *xbuf, int nkc, int row) {
    float xn = 0.f;
    for (int kc = 0; kc < nkc; ++kc) xn += row_sqnorm_swizzled<T>(xbuf + kc * XCHUNK + row * 128, row);
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

// Packed key of column I: the distance bits with the low log2(W) mantissa bits replaced by I.
// One three-input logic op with the mask held in a register (`mask` = ~(W - 1), kept live by the
// caller) and I as the immediate; written in PTX so the two constants cannot turn into two ops.
template <int I>
__device__ __forceinline__ float pkey(uint32_t v, uint32_t mask) {
    uint32_t k;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(k) : "r"(v), "r"(mask), "n"(I));   // (v & mask) | I
    return __uint_as_float(k);
}
// Minimum of W packed keys and one carried value, as a queue of 3-input mins: W + 1 inputs
// (odd) take exactly W / 2 operations, and the first W / 6 of them are independent.
template <int W, int... I>
__device__ __forceinline__ float keys_min_seq(const uint32_t (&v)[W], uint32_t mask, float carry,
                                              std::integer_sequence<int, I...>) {
    static_assert(W % 2 == 0, "an odd number of inputs reduces by 3-input mins alone");
    float q[2 * W + 1] = {pkey<I>(v[I], mask)..., carry};
    int head = 0, tail = W + 1;
#pragma unroll
    for (int s = 0; s < W / 2; ++s) {
        q[tail++] = min3f(q[head], q[head + 1], q[head + 2]);
        head += 3;
    }
    return q[head];
}
template <int W>
__device__ __forceinline__ float keys_min(const uint32_t (&v)[W], uint32_t mask, float carry) {
    return keys_min_seq<W>(v, mask, carry, std::make_integer_sequence<int, W>{});
}

// NKC = ceil(d / 64): the number of 64-wide chunks of the reduction, fixed per instantiation so
// the issue loop unrolls into MMAs whose descriptors differ by constants.
template <typename T, int BN, int NKC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmA, const Params p) {
    constexpr int W = BN / 4;           // accumulator columns per epilogue warp
    constexpr uint32_t IMASK = W - 1;
    // Split tiles (bn = 256): each tile's MMAs run as two N = 128 halves with their own
    // completion and hand-back barriers. Column quarters 0-1 read half 0 while half 1 is still
    // being computed, so the two warp pairs of a sub-partition work half a tile apart and one
    // pair's TMEM load overlaps the other pair's compare work. Each CTA supplies 64 centroid rows
    // per half, so accumulator column c of half h holds centroid (c < 64 ? h * 64 + c :
    // 128 + h * 64 + c - 64) of the tile: column quarters 0, 1, 2, 3 hold tile columns 0-63,
    // 128-191, 64-127, 192-255.
    constexpr bool SPLIT = BN == 256;
    constexpr int CROWS = BN / 2;       // centroid rows each CTA stages per tile
    constexpr uint32_t CCHUNK = CROWS * 128u;   // one [bn/2 x 64] centroid chunk
    extern __shared__ uint8_t smem_raw[];
    __shared__ int abort_flag;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sgen = smem_raw + (sbase - raw);
    const Layout L = make_layout(NKC, BN, p.stages);
    const int S = p.stages;
    const uint32_t bar0 = sbase + L.bar_off;
    auto X_FULL = [&](int i) { return bar0 + 8u * i; };
    auto X_EMPTY = [&](int i) { return bar0 + 8u * (2 + i); };
    auto XAUG_FULL = [&](int i) { return bar0 + 8u * (4 + i); };
    // accumulator i = 2 * buffer + half (half 1 only with split tiles)
    auto ACC_FULL = [&](int i) { return bar0 + 8u * (6 + i); };
    auto ACC_EMPTY = [&](int i) { return bar0 + 8u * (10 + i); };
    const uint32_t DRAIN = bar0 + 8u * 14;
    auto DELTA_FULL = [&](int i) { return bar0 + 8u * (15 + i); };   // i < DELTA_SLOTS
    auto C_FULL = [&](int s) { return bar0 + 8u * (NUM_BARS_FIXED + s); };
    auto C_EMPTY = [&](int s) { return bar0 + 8u * (NUM_BARS_FIXED + S + s); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    volatile int *abortp = &abort_flag;

    // Warps computing the point tiles' norms: the point warp, joined in resident mode by the
    // centroid warp (which then only hands stages back), so the work is spread over two
    // sub-partitions instead of loading one.
    const int nnorm = p.resident ? 2 : 1;
    // Rows [r0, r1) of point buffer xb (work item `local`): ||x||^2/2 split into two bf16 pieces
    // for the point side of the norm step, and delta, the rounding left over.
    auto norm_rows = [&](int xb, int local, int r0, int r1) {
        float *dbuf = reinterpret_cast<float *>(sgen + L.delta_off);
        const int lane = threadIdx.x & 31;
#pragma unroll 2
        for (int row = r0 + lane; row < r1; row += 32) {
            const float half_xn =
                0.5f * tile_row_sqnorm<T>(sgen + L.x_off + xb * NKC * XCHUNK, NKC, row);
            // The split carries ||x||^2/2 raised by 2^-12 of itself. The accumulator is then
            // d/2 + (about 2^-13 ||x||^2), positive even for a point on its centroid, since the
            // two-piece split (2^-18 relative) and the fp32 reduction (below 2^-15 ||x||^2) err
            // by less. Keys of positive floats order ties by index the way the min expects
            // (lowest index wins); delta takes the raise back out of the reported distance, and
            // a constant per row cannot change the argmin.
            const float tgt = fmaf(half_xn, 0x1p-12f, half_xn);
            const float x1 = __bfloat162float(__float2bfloat16_rn(tgt));
            const float x2 = __bfloat162float(__float2bfloat16_rn(tgt - x1));
            dbuf[(local & (DELTA_SLOTS - 1)) * BM + row] = (half_xn - x1) - x2;
            // Row of the point-side augmentation in the 32-byte-swizzled layout: the two
            // 16-byte halves of rows 4..7 of every 8-row group trade places.
            const uint4 data = make_uint4(pack_bf16x2(x1, x2), pack_bf16x2(1.f, 1.f),
                                          pack_bf16x2(1.f, 0.f), 0u);
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            uint8_t *rp = sgen + L.xaug_off + xb * XAUG_BYTES + row * 32;
            const int sw = (row >> 2) & 1;
            *reinterpret_cast<uint4 *>(rp + 16 * sw) = data;
            *reinterpret_cast<uint4 *>(rp + 16 * (1 - sw)) = zero;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
    };
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(X_FULL(i), 1);
            // own point warp (done reading the tile) + own column-quarter-0 epilogue warps (the
            // item's last accumulator seen complete, so every MMA reading the tile is done)
            mbar_init(X_EMPTY(i), nnorm + 4);
            mbar_init(XAUG_FULL(i), 2 * nnorm);   // (leader) the norm warps of both CTAs
            for (int h = 0; h < 2; ++h) {
                mbar_init(ACC_FULL(2 * i + h), 1);
                // (leader) the epilogue warps of both CTAs that read this accumulator (half)
                mbar_init(ACC_EMPTY(2 * i + h), SPLIT ? NUM_EPI_WARPS : 2 * NUM_EPI_WARPS);
            }
        }
        mbar_init(DRAIN, 2);   // one commit per MMA warp
        for (int i = 0; i < static_cast<int>(DELTA_SLOTS); ++i) mbar_init(DELTA_FULL(i), nnorm);
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
    // Each cluster takes a contiguous range of work items, so it changes batch element (and,
    // with resident centroids, reloads them) as rarely as possible.
    const int cluster_id = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;
    const int per_cluster = (total + nclusters - 1) / nclusters;
    const int t_begin = min(total, cluster_id * per_cluster);
    const int t_end = min(total, t_begin + per_cluster);
    const uint32_t stage_tx = 2u * cstage_bytes(NKC, BN);   // both CTAs' halves of a tile

    if (warp == WARP_CPROD) {
        // ------------------------------------------------------------ centroid producer
        // (all lanes wait, lane 0 issues; in resident mode the warp also computes the second
        // half of each point tile's norms before handing the item's stages back)
        const uint64_t pol_c = l2_policy_evict_last();
        const uint32_t xaug_full_leader0 = map_to_rank(XAUG_FULL(0), 0);
        const uint32_t xaug_full_leader1 = map_to_rank(XAUG_FULL(1), 0);
        int stage = 0;
        uint32_t cph = 0;
        long long n_c = 0;
        bool ok = true;
        int cur_b = -1;   // batch element whose centroid tiles the ring holds (resident mode)
        int local = 0;
        for (int t = t_begin; t < t_end && ok; ++t, ++local) {
            const int b = t / p.mtiles;
            if (p.resident) {
                const int xb = local & 1;
                if (!mbar_wait_warp(X_FULL(xb), (local >> 1) & 1, abortp)) { ok = false; break; }
                norm_rows(xb, local, BM / 2, BM);
                if (lane == 0) {
                    mbar_arrive_cluster(xb ? xaug_full_leader1 : xaug_full_leader0);
                    mbar_arrive(DELTA_FULL(local & (DELTA_SLOTS - 1)));
                    mbar_arrive(X_EMPTY(xb));
                }
            }
            // Resident mode (the ring holds every tile of a batch element: stage j = tile j):
            // the tiles are loaded again only when the batch element changes; otherwise the
            // stage's phase just advances.
            const bool reload = !p.resident || b != cur_b;
            cur_b = b;
            for (int j = 0; j < p.nct; ++j) {
                const int crow = j * BN + static_cast<int>(rank) * CROWS;
                if (!mbar_wait_warp(C_EMPTY(stage), cph ^ 1u, abortp)) { ok = false; break; }
                if (lane == 0) {
                    if (!reload) {
                        if (leader) mbar_arrive(C_FULL(stage));
                    } else {
                        if (leader) mbar_arrive_expect_tx(C_FULL(stage), stage_tx);
                        const uint32_t sdst = sbase + L.c_off + stage * L.stage;
                        const uint32_t lbar = map_to_rank(C_FULL(stage), 0);
                        for (int kc = 0; kc < NKC; ++kc)
                            tma_load_3d_pair(sdst + kc * CCHUNK, &tmC, lbar, kc * KC, crow, b, pol_c);
                        tma_load_3d_pair(sdst + NKC * CCHUNK, &tmA, lbar, 0, crow, b, pol_c);
                    }
                }
                __syncwarp();
                ++n_c;
                if (++stage == S) { stage = 0; cph ^= 1u; }
            }
        }
        if (!ok && leader && lane == 0) {
            // Let every pair copy issued into the ring land before shared memory goes away
            // (n_c counts every use of the ring, so each stage's last phase is known).
            for (int s = 0; s < S; ++s) {
                const long long uses = n_c > s ? (n_c - 1 - s) / S + 1 : 0;
                if (uses) mbar_wait(C_FULL(s), static_cast<uint32_t>((uses - 1) & 1), nullptr);
            }
        }
        __syncwarp();
    } else if (warp == WARP_XPROD) {
        // ------------------------------------------------------------ point tiles and norms
        const uint64_t pol_x = l2_policy_evict_first();
        // test-only fault switch (off by default): withhold the first point tile of pair 0
        const bool withhold = blockIdx.x == 0 && *reinterpret_cast<volatile int *>(&g_km_inject) == 1;
        const uint32_t xaug_full_leader0 = map_to_rank(XAUG_FULL(0), 0);
        const uint32_t xaug_full_leader1 = map_to_rank(XAUG_FULL(1), 0);
        int n_x = 0;
        bool ok = true;
        int local = 0;
        for (int t = t_begin; t < t_end; ++t, ++local) {
            const int b = t / p.mtiles;
            const int m0 = (t % p.mtiles) * (2 * BM) + static_cast<int>(rank) * BM;
            const int xb = local & 1;
            const uint32_t xph = (local >> 1) & 1;
            if (!mbar_wait_warp(X_EMPTY(xb), xph ^ 1u, abortp)) { ok = false; break; }
            const bool request = !(withhold && local == 0);
            if (lane == 0 && request) {
                mbar_arrive_expect_tx(X_FULL(xb), NKC * XCHUNK);
                for (int kc = 0; kc < NKC; ++kc)
                    tma_load_3d(sbase + L.x_off + (xb * NKC + kc) * XCHUNK, &tmX, X_FULL(xb),
                                kc * KC, m0, b, pol_x);
            }
            __syncwarp();
            if (request) ++n_x;
            // The tile's norms as soon as it lands (this warp has nothing else to do until the
            // next buffer is handed back at the end of the work item before this one).
            if (!mbar_wait_warp(X_FULL(xb), xph, abortp)) { ok = false; break; }
            norm_rows(xb, local, 0, BM / nnorm);
            if (lane == 0) {
                mbar_arrive_cluster(xb ? xaug_full_leader1 : xaug_full_leader0);
                mbar_arrive(DELTA_FULL(local & (DELTA_SLOTS - 1)));
                mbar_arrive(X_EMPTY(xb));
            }
        }
        if (!ok && lane == 0) {
            // Let every point copy issued land before shared memory goes away.
            for (int i = 0; i < 2; ++i) {
                const int uses = n_x > i ? (n_x - 1 - i) / 2 + 1 : 0;
                if (uses) mbar_wait(X_FULL(i), static_cast<uint32_t>((uses - 1) & 1), nullptr);
            }
        }
        __syncwarp();
    } else if (warp == WARP_MMA || warp == WARP_MMA_ODD) {
        // ------------------------------------------------------------ MMA issuers (leader)
        if (leader) {
            const int abuf = warp == WARP_MMA ? 0 : 1;   // this warp's accumulator and tiles
            const bool issuer = elect_one();   // the same lane issues every MMA and commit
            uint32_t aph = 0;
            // tile sequence number g = local * nct + j; this warp takes g % 2 == abuf
            int local = 0, j = abuf;
            int t = t_begin;
            while (j >= p.nct) { j -= p.nct; ++local; ++t; }
            int g = abuf;
            int xaug_local = -1;   // the work item whose point rows were last seen ready
            const uint32_t cbase_lo = desc_lo(sbase + L.c_off);
            const uint32_t xbase_lo = desc_lo(sbase + L.x_off);
            const uint32_t xaug_lo = desc_lo(sbase + L.xaug_off);
            const uint32_t stage16 = L.stage >> 4;
            constexpr uint32_t cchunk16 = CCHUNK >> 4;
            constexpr uint32_t xchunk16 = XCHUNK >> 4;
            const int nk_last = (p.d - (NKC - 1) * KC + 15) / 16;   // K steps of the last chunk
            // split tiles issue N = BN / 2 per MMA (the N field of the instruction descriptor)
            constexpr uint32_t NMASK = 0x3Fu << 17;
            const uint32_t idesc_main = SPLIT ? (p.idesc_main & ~NMASK) | ((BN / 2 >> 3) << 17) : p.idesc_main;
            const uint32_t idesc_aug = SPLIT ? (p.idesc_aug & ~NMASK) | ((BN / 2 >> 3) << 17) : p.idesc_aug;
            while (t < t_end) {
                const int xb = local & 1;
                const uint32_t xph = (local >> 1) & 1;
                const int stage = g % S;
                const uint32_t cph = (g / S) & 1;
                // both CTAs' point tiles landed and their augmentation rows are written; the
                // epilogue has read this accumulator; the centroid tile has landed
                if (xaug_local != local) {
                    if (!mbar_wait_warp(XAUG_FULL(xb), xph, abortp)) break;
                    xaug_local = local;
                }
                if (!mbar_wait_warp(C_FULL(stage), cph, abortp)) break;
                const uint32_t b_lo = cbase_lo + stage * stage16;
                const uint32_t a_lo = xbase_lo + xb * (NKC * xchunk16);
                bool fail = false;
#pragma unroll
                for (int h = 0; h < (SPLIT ? 2 : 1); ++h) {
                    if (!mbar_wait_warp(ACC_EMPTY(2 * abuf + h), aph ^ 1u, abortp)) { fail = true; break; }
                    tc_fence_after();
                    // half h: accumulator columns h * 128.., centroid rows h * 64.. of each CTA
                    const uint32_t dcol = tmem_base + abuf * ACC_STRIDE + h * (BN / 2);
                    const uint32_t bm_lo = b_lo + h * ((BN / 4) * 128u >> 4);
                    const uint32_t ba_lo = b_lo + NKC * cchunk16 + h * ((BN / 4) * 32u >> 4);
                    if (issuer) {
#pragma unroll
                        for (int kc = 0; kc < NKC; ++kc)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                if (kc + 1 < NKC || kk < nk_last)
                                    tc_mma_pair(dcol, a_lo + kc * xchunk16 + kk * 2, DESC_HI_SW128,
                                                bm_lo + kc * cchunk16 + kk * 2, DESC_HI_SW128,
                                                idesc_main, (kc | kk) != 0 ? 1u : 0u);
                        tc_mma_pair(dcol, xaug_lo + xb * (XAUG_BYTES >> 4), DESC_HI_SW32,
                                    ba_lo, DESC_HI_SW32, idesc_aug, 1u);
                        tc_commit_pair_both(ACC_FULL(2 * abuf + h));
                    }
                    __syncwarp();
                }
                if (fail) break;
                __syncwarp();
                aph ^= 1u;
                g += 2;
                j += 2;
                while (j >= p.nct) { j -= p.nct; ++local; ++t; }
            }
            // Every MMA issued above completes before TMEM is released.
            if (issuer) tc_commit_pair_self(DRAIN);
            __syncwarp();
            mbar_wait_warp(DRAIN, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - WARP_EPI0;
        const int q = warp & 3;          // TMEM lane quarter this warp may read
        const int cq = ew >> 2;          // column quarter of the accumulator
        const int row = q * 32 + lane;
        const float *dbuf = reinterpret_cast<const float *>(sgen + L.delta_off);
        float *mval = reinterpret_cast<float *>(sgen + L.merge_off);
        int *midx = reinterpret_cast<int *>(sgen + L.merge_off + 2u * 3u * BM * 4u);
        const int half = SPLIT ? cq >> 1 : 0;   // the accumulator half this warp reads
        const uint32_t acc_empty_leader0 = map_to_rank(ACC_EMPTY(half), 0);
        const uint32_t acc_empty_leader1 = map_to_rank(ACC_EMPTY(2 + half), 0);
        const uint32_t tlane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + cq * W;
        // first tile column of this warp's accumulator columns
        const int cbase = SPLIT ? (cq & 1) * 128 + (cq >> 1) * 64 : cq * W;
        uint32_t kmask = ~IMASK;                 // the key mask, held in a register
        asm volatile("" : "+r"(kmask));
        // Whole-tile completions are seen by warps of the last half: the last one hands the
        // centroid stages back, and column quarter 2 (0 without split tiles) the point buffer.
        const int last_cq = SPLIT ? 2 : 0;
        const bool stage_owner = ew == (SPLIT ? 8 : 0);
        const bool nct_even = (p.nct & 1) == 0;
        int abuf = 0;
        uint32_t aph = 0;
        int stage = 0;
        // One accumulator tile: wait for its MMAs, load this warp's columns, hand the buffer
        // back and fold the columns into the running best. `ab` is a constant on the paired path.
        auto tile = [&](int ab, int j, int xb, float &best_v, uint32_t &best_m, int &best_j) -> bool {
            if (!mbar_wait_warp(ACC_FULL(2 * ab + half), aph, abortp)) return false;
            tc_fence_after();
            // The item's last tile is complete, so every MMA reading its point tile is done:
            // the point buffer goes back to the producer now, not after this tile's epilogue.
            if (cq == last_cq && j == p.nct - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(X_EMPTY(xb));
            }
            // The tile's MMAs are complete: its centroid stage may be refilled.
            if (stage_owner) {
                if (lane == 0) mbar_arrive_relaxed(C_EMPTY(stage));
                if (++stage == S) stage = 0;
            }
            __syncwarp();
            uint32_t v[W];
            if constexpr (W == 64) tmem_ld_32x32b_x64(tlane + ab * ACC_STRIDE, v);
            else if constexpr (W == 32) tmem_ld_32x32b_x32(tlane + ab * ACC_STRIDE, v);
            else tmem_ld_32x32b_x16(tlane + ab * ACC_STRIDE, v);
            tmem_wait_ld(v);
            // Every column this warp needs is in registers: hand the accumulator back. The
            // arrive is relaxed, so it never waits for this warp's output stores.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(ab ? acc_empty_leader1 : acc_empty_leader0);
            // The best value so far (its column bits zero) is one more input of the tree: it
            // wins every tie with this tile's keys, so the result differs from it only when a
            // key of this tile is strictly smaller, and an earlier tile keeps an equal value.
            const uint32_t mb = __float_as_uint(keys_min<W>(v, kmask, best_v));
            if (mb != __float_as_uint(best_v)) {
                best_m = mb;
                best_j = j;
            }
            best_v = __uint_as_float(mb & kmask);
            return true;
        };
        int local = 0;
        int b = t_begin / p.mtiles;          // batch element and pair tile of work item t,
        int mt = t_begin - b * p.mtiles;     // advanced incrementally
        for (int t = t_begin; t < t_end; ++t, ++local) {
            const int m0 = mt * (2 * BM) + static_cast<int>(rank) * BM;
            const int xb = local & 1;
            bool ok = true;
            float best_v = INFINITY;   // the best value (key without its column bits) so far
            uint32_t best_m = 0;       // its packed key
            int best_j = 0;            // and its tile
            if (nct_even) {
                // Tiles come in pairs, buffer 0 then buffer 1, so every item starts on buffer 0.
                for (int j = 0; j < p.nct; j += 2) {
                    if (!tile(0, j, xb, best_v, best_m, best_j) || !tile(1, j + 1, xb, best_v, best_m, best_j)) {
                        ok = false;
                        break;
                    }
                    aph ^= 1u;
                }
            } else {
                for (int j = 0; j < p.nct; ++j) {
                    if (!tile(abuf, j, xb, best_v, best_m, best_j)) { ok = false; break; }
                    abuf ^= 1;
                    if (abuf == 0) aph ^= 1u;
                }
            }
            int best_i = best_j * BN + cbase + static_cast<int>(best_m & IMASK);
            // Column quarter 0 merges the four quarters of each row and writes the result; the
            // reported distance adds back delta, the rounding of this row's two-piece ||x||^2/2.
            const int slot = local & 1;
            if (cq != 0) {
                mval[(slot * 3 + cq - 1) * BM + row] = best_v;
                midx[(slot * 3 + cq - 1) * BM + row] = best_i;
            }
            float delta = 0.f;
            if (cq == 0 && p.need_dist && ok) {
                const int ds = local & (DELTA_SLOTS - 1);
                if (mbar_wait_warp(DELTA_FULL(ds), (local / DELTA_SLOTS) & 1, abortp)) delta = dbuf[ds * BM + row];
            }
            // All four warps of a lane quarter reach this barrier once per work item, then
            // leave together if any of them saw a role give up.
            if (named_barrier_or(1 + q, 128, !ok || *abortp != 0)) break;
            if (cq == 0) {
#pragma unroll
                for (int o = 0; o < 3; ++o) {
                    // a quarter's best may come from any tile: equal values keep the lower index
                    const float ob = mval[(slot * 3 + o) * BM + row];
                    const int oi = midx[(slot * 3 + o) * BM + row];
                    if (ob < best_v || (ob == best_v && oi < best_i)) {
                        best_v = ob;
                        best_i = oi;
                    }
                }
                const int i = m0 + row;
                double contrib = 0.0;
                if (i < p.N) {
                    const size_t gi = static_cast<size_t>(b) * p.N + i;
                    p.ids[gi] = best_i;
                    if (p.need_dist) {
                        const float md = fmaxf(0.f, 2.f * (best_v + delta));
                        if (p.mind) p.mind[gi] = md;
                        const float wi = p.w ? p.w[static_cast<int64_t>(b) * p.wld + i] : 1.f;
                        contrib = static_cast<double>(wi) * static_cast<double>(md);
                    }
                }
                if (p.inertia) {
                    contrib = warp_sum(contrib);
                    if (lane == 0) atomicAdd(p.inertia + b, contrib);
                }
                // the histogram the update's sort starts from (a reduction without return)
                if (p.counts && i < p.N) atomicAdd(p.counts + static_cast<size_t>(b) * p.K + best_i, 1);
            }
            if (++mt == p.mtiles) {
                mt = 0;
                ++b;
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
