// km_lib.cu -- the C ABI of libkmeans_b200.so (declared in include/kmeans_b200.h).
//
// Argument validation, workspace carving, kernel selection and stream-ordered launches. All
// kernels live in the km_*.cuh headers of this directory and are compiled in this single
// translation unit. The library never allocates device memory: every scratch buffer is carved
// from the caller's workspace, whose size km_workspace_size computes with the same layout code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "kmeans_b200.h"
#include "km_assign_simt.cuh"
#include "km_assign_tc.cuh"
#include "km_centroids.cuh"
#include "km_codebook1d.cuh"
#include "km_common.cuh"
#include "km_emeans.cuh"
#include "km_fit1d.cuh"
#include "km_fit_small.cuh"
#include "km_update.cuh"

namespace {

using km::Cvt;

constexpr size_t kAlign = 256;
constexpr int64_t kMaxIndex = (int64_t{1} << 31) - 1;
constexpr int64_t kMaxD = int64_t{1} << 20;
constexpr int kMaxGridY = 65535;

inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool valid_dtype(km_dtype dt) { return dt == KM_F32 || dt == KM_F16 || dt == KM_BF16; }
inline size_t dtype_size(km_dtype dt) { return dt == KM_F32 ? 4 : 2; }

inline bool sizes_ok(int64_t B, int64_t N, int64_t K, int64_t d) {
    return B >= 1 && N >= 1 && K >= 1 && d >= 1 && B <= kMaxIndex && N <= kMaxIndex &&
           K <= kMaxIndex && d <= kMaxD && B * N <= (int64_t{1} << 40) &&
           B * K <= (int64_t{1} << 40);
}

// ---------------------------------------------------------------- workspace layouts

struct Carver {
    uint8_t *base;
    size_t off = 0;
    explicit Carver(void *b) : base(static_cast<uint8_t *>(b)) {}
    template <typename P> P *take(size_t bytes) {
        P *p = base ? reinterpret_cast<P *>(base + off) : nullptr;
        off += align_up(bytes);
        return p;
    }
};

inline bool tc_shape_ok(km_dtype dt, int64_t d) {
    return dt != KM_F32 && d % 8 == 0 && d >= 8 && d <= 256;
}
// Centroids per SM-pair tile: the smallest of 64/128/256 that covers K, narrowed while the
// point tile plus two ring stages would not fit in shared memory (large d).
inline int tc_bn(int64_t K, int64_t d) {
    int bn = K > 128 ? 256 : (K > 64 ? 128 : 64);
    const int nkc = static_cast<int>(ceil_div(d, km::tc::KC));
    while (bn > 64 && km::tc::pick_stages(nkc, bn) == 0) bn /= 2;
    return bn;
}
inline int64_t tc_kp(int64_t K, int64_t d) { return ceil_div(K, tc_bn(K, d)) * tc_bn(K, d); }

inline size_t ws_assign(int64_t B, int64_t K, int64_t d, km_dtype dt) {
    return tc_shape_ok(dt, d) ? align_up(static_cast<size_t>(B * tc_kp(K, d)) * 32) : 0;
}

struct UpdateWs {
    int32_t *offsets, *cursor, *perm;
    float *sums, *wsum;
};
inline UpdateWs carve_update(Carver &c, int64_t B, int64_t N, int64_t K, int64_t d) {
    UpdateWs u;
    u.offsets = c.take<int32_t>(static_cast<size_t>(B * (K + 1)) * 4);
    u.cursor = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    u.perm = c.take<int32_t>(static_cast<size_t>(B * N) * 4);
    u.sums = c.take<float>(static_cast<size_t>(B * K * d) * 4);
    u.wsum = c.take<float>(static_cast<size_t>(B * K) * 4);
    return u;
}

// The fused reduce-and-divide form: the sort scratch, arrival counters and the per-range partial
// slots of split segments (ranges per batch element are at most kFinalWarpsMax / B + 1).
constexpr int64_t kFinalWarpsMax = 2048;
struct FinalWs {
    int32_t *offsets, *cursor, *perm, *arrive, *rseg;
    float *slots, *wslots;
};
inline int64_t final_rpb_max(int64_t B) { return std::max<int64_t>(1, kFinalWarpsMax / B) + 1; }
inline FinalWs carve_final(Carver &c, int64_t B, int64_t N, int64_t K, int64_t d) {
    FinalWs f;
    f.offsets = c.take<int32_t>(static_cast<size_t>(B * (K + 1)) * 4);
    f.cursor = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    f.perm = c.take<int32_t>(static_cast<size_t>(B * N) * 4);
    f.arrive = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    f.rseg = c.take<int32_t>(static_cast<size_t>(B * final_rpb_max(B)) * 4);
    const int64_t nslots = B * final_rpb_max(B) * 2;
    f.slots = c.take<float>(static_cast<size_t>(nslots * d) * 4);
    f.wslots = c.take<float>(static_cast<size_t>(nslots) * 4);
    return f;
}
// bytes that cover both update forms (the caller's workspace serves whichever runs)
inline size_t ws_update(int64_t B, int64_t N, int64_t K, int64_t d) {
    Carver a(nullptr), f(nullptr);
    carve_update(a, B, N, K, d);
    carve_final(f, B, N, K, d);
    return std::max(a.off, f.off);
}

inline bool fit1d_ok(int64_t N, int64_t K, int64_t d) {
    return d == 1 && K <= km::fit1d::KMAX && N <= km::fit1d::NMAX;
}
// the warp-per-row form: one centroid per lane
inline bool fit1d_rows_ok(int64_t N, int64_t K, int64_t d) {
    return fit1d_ok(N, K, d) && K <= km::fit1d::ITER_KMAX;
}

// Warp-per-row 1-D fit: sorted values and original indices, prefix sums of w, w*x, w*x^2.
struct Fit1dWs {
    float *xs;
    int32_t *is;
    double *P0, *P1, *P2;
};
inline Fit1dWs carve_fit1d(Carver &c, int64_t B, int64_t N) {
    Fit1dWs g;
    g.xs = c.take<float>(static_cast<size_t>(B * N) * 4);
    g.is = c.take<int32_t>(static_cast<size_t>(B * N) * 4);
    g.P0 = c.take<double>(static_cast<size_t>(B * (N + 1)) * 8);
    g.P1 = c.take<double>(static_cast<size_t>(B * (N + 1)) * 8);
    g.P2 = c.take<double>(static_cast<size_t>(B * (N + 1)) * 8);
    return g;
}

// Whole-fit single launch for small problems (km_fit_small.cuh): shapes it may take. The launch
// itself is used only when every CTA can be resident at once (checked at run time).
constexpr int64_t kSmallMaxCtas = 2048;
inline bool fit_small_shape_ok(int64_t B, int64_t N, int64_t K, int64_t d) {
    return d >= 1 && d <= 64 && K * d <= 4096 && B * ceil_div(N, km::fs::kPts) <= kSmallMaxCtas &&
           B * N * K * d <= (int64_t{1} << 27);
}
// One block, zeroed before each launch: three accumulators [3, B, K, d + 2] fp32, three inertia
// slots [3, B] fp64, the barrier words.
struct SmallWs {
    float *acc;
    double *iacc;
    unsigned int *bar;
    size_t bytes;
};
inline SmallWs carve_small(Carver &c, int64_t B, int64_t K, int64_t d) {
    const size_t abytes = static_cast<size_t>(3 * B * K * (d + 2)) * 4;
    const size_t ibytes = static_cast<size_t>(3 * B) * 8;
    SmallWs s;
    s.bytes = align_up(abytes) + align_up(ibytes) + 16;
    uint8_t *base = c.take<uint8_t>(s.bytes);
    s.acc = reinterpret_cast<float *>(base);
    s.iacc = base ? reinterpret_cast<double *>(base + align_up(abytes)) : nullptr;
    s.bar = base ? reinterpret_cast<unsigned int *>(base + align_up(abytes) + align_up(ibytes)) : nullptr;
    return s;
}

struct FitWs {
    void *Cx;
    float *cn;
    int32_t *ids, *counts;
    double *inertia;
    void *rest;
};
inline FitWs carve_fit(Carver &c, int64_t B, int64_t N, int64_t K, int64_t d, km_dtype dt) {
    FitWs f;
    f.Cx = c.take<uint8_t>(static_cast<size_t>(B * K * d) * dtype_size(dt));
    f.cn = c.take<float>(static_cast<size_t>(B * K) * 4);
    f.ids = c.take<int32_t>(static_cast<size_t>(B * N) * 4);
    f.counts = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    f.inertia = c.take<double>(static_cast<size_t>(B) * 8);
    f.rest = c.base ? c.base + c.off : nullptr;
    Carver g(nullptr);
    if (fit1d_rows_ok(N, K, d)) carve_fit1d(g, B, N);
    Carver h(nullptr);
    if (fit_small_shape_ok(B, N, K, d)) carve_small(h, B, K, d);
    c.off += std::max({ws_update(B, N, K, d), ws_assign(B, K, d, dt), g.off, h.off});
    return f;
}

struct HostWs {
    void *X;
    float *w, *C;
    int32_t *ids;
    double *inertia;
    void *fit;
};
inline HostWs carve_host(Carver &c, int64_t B, int64_t N, int64_t K, int64_t d, km_dtype dt,
                         bool weighted, int iters) {
    HostWs h;
    h.X = c.take<uint8_t>(static_cast<size_t>(B * N * d) * dtype_size(dt));
    h.w = weighted ? c.take<float>(static_cast<size_t>(B * N) * 4) : nullptr;
    h.C = c.take<float>(static_cast<size_t>(B * K * d) * 4);
    h.ids = c.take<int32_t>(static_cast<size_t>(B * N) * 4);
    h.inertia = c.take<double>(static_cast<size_t>(std::max(iters, 1)) * B * 8);
    h.fit = c.base ? c.base + c.off : nullptr;
    carve_fit(c, B, N, K, d, dt);
    return h;
}

// Streamed fit: two device buffers of `chunk` points per batch element (X and weights), the
// running per-cluster statistics, one chunk's sort and assignment scratch.
struct StreamWs {
    void *xbuf[2];
    float *wbuf[2];
    void *Cx;
    float *cn;
    int32_t *ids, *counts, *chunk_counts;
    void *rest;   // UpdateWs for one chunk, then (reusing it) the assignment scratch
};
inline StreamWs carve_stream(Carver &c, int64_t B, int64_t K, int64_t d, km_dtype dt, bool weighted,
                             int64_t chunk) {
    StreamWs s;
    for (int i = 0; i < 2; ++i) {
        s.xbuf[i] = c.take<uint8_t>(static_cast<size_t>(B * chunk * d) * dtype_size(dt));
        s.wbuf[i] = weighted ? c.take<float>(static_cast<size_t>(B * chunk) * 4) : nullptr;
    }
    s.Cx = c.take<uint8_t>(static_cast<size_t>(B * K * d) * dtype_size(dt));
    s.cn = c.take<float>(static_cast<size_t>(B * K) * 4);
    s.ids = c.take<int32_t>(static_cast<size_t>(B * chunk) * 4);
    s.counts = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    s.chunk_counts = c.take<int32_t>(static_cast<size_t>(B * K) * 4);
    s.rest = c.base ? c.base + c.off : nullptr;
    Carver u(nullptr);
    carve_update(u, B, chunk, K, d);
    c.off += u.off;   // the running sums/wsum live in this UpdateWs; the assignment scratch follows
    c.off += align_up(ws_assign(B, K, d, dt));
    return s;
}

// ---------------------------------------------------------------- device queries

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

inline km_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? KM_OK : KM_ERR_CUDA;
}

// ---------------------------------------------------------------- kernel launchers

template <typename T>
km_status run_prep(const float *C, int64_t rows, int64_t d, void *Cx, float *cn, cudaStream_t st) {
    const int64_t blocks = ceil_div(rows, 8);
    km::prep_kernel<T><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        C, rows, static_cast<int>(d), static_cast<T *>(Cx), cn);
    return launch_status();
}

km_status prep_dispatch(const float *C, km_dtype dt, int64_t rows, int64_t d, void *Cx, float *cn,
                        cudaStream_t st) {
    switch (dt) {
        case KM_F32: return run_prep<float>(C, rows, d, Cx, cn, st);
        case KM_F16: return run_prep<__half>(C, rows, d, Cx, cn, st);
        default: return run_prep<__nv_bfloat16>(C, rows, d, Cx, cn, st);
    }
}

template <typename T>
km_status run_finalize(const float *sums, const float *wsum, const int32_t *counts,
                       const float *C_prev, int64_t rows, int64_t d, float *C_new, void *Cx,
                       float *cn, cudaStream_t st) {
    km::finalize_kernel<T><<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, st>>>(
        sums, wsum, counts, C_prev, rows, static_cast<int>(d), C_new, static_cast<T *>(Cx), cn);
    return launch_status();
}

km_status finalize_dispatch(const float *sums, const float *wsum, const int32_t *counts,
                            const float *C_prev, int64_t rows, int64_t d, float *C_new, km_dtype dt,
                            void *Cx, float *cn, cudaStream_t st) {
    switch (dt) {
        case KM_F16: return run_finalize<__half>(sums, wsum, counts, C_prev, rows, d, C_new, Cx, cn, st);
        case KM_BF16:
            return run_finalize<__nv_bfloat16>(sums, wsum, counts, C_prev, rows, d, C_new, Cx, cn, st);
        default: return run_finalize<float>(sums, wsum, counts, C_prev, rows, d, C_new, Cx, cn, st);
    }
}

template <typename T>
km_status run_assign_simt(const void *X, const void *Cx, const float *w, int64_t B, int64_t N,
                          int64_t K, int64_t d, int32_t *ids, float *mind, double *inertia,
                          int32_t *counts, int64_t xld, cudaStream_t st) {
    const T *Xt = static_cast<const T *>(X);
    const T *Ct = static_cast<const T *>(Cx);
    for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {
        const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
        dim3 grid(static_cast<unsigned>(ceil_div(N, km::kSimtPts)), static_cast<unsigned>(nb));
        km::assign_simt_kernel<T><<<grid, km::kSimtPts, 0, st>>>(
            Xt + b0 * xld * d, Ct + b0 * K * d, w ? w + b0 * xld : nullptr, static_cast<int>(N),
            static_cast<int>(K), static_cast<int>(d), ids + b0 * N, mind ? mind + b0 * N : nullptr,
            inertia ? inertia + b0 : nullptr, counts ? counts + b0 * K : nullptr, xld);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
    }
    return KM_OK;
}

template <typename T, int BN, int NKC>
km_status launch_assign_tc(const CUtensorMap &tmX, const CUtensorMap &tmC, const CUtensorMap &tmA,
                           km::tc::Params &p, int64_t items, cudaStream_t st) {
    using namespace km::tc;
    // Keep every centroid tile of a batch element resident when the ring can hold them all
    // (one reload per batch element instead of one per work item); else stream them.
    if (p.nct >= 2 && p.nct <= MAX_STAGES && make_layout(NKC, BN, p.nct).total + 1024u <= SMEM_ATTR) {
        p.stages = p.nct;
        p.resident = 1;
    } else {
        p.stages = pick_stages(NKC, BN);
        p.resident = 0;
    }
    if (p.stages < 2) return KM_ERR_UNSUPPORTED;
    const Layout L = make_layout(NKC, BN, p.stages);
    // More than half of the shared memory per block keeps one CTA per SM, so no second CTA
    // ever waits in tcgen05.alloc for the 512 TMEM columns the first one holds.
    const size_t smem = std::max<size_t>(L.total + 1024, SMEM_LIMIT / 2 + 1024);
    // The attribute is an upper bound for every later launch, so it is always set to the
    // kernel's largest request, never to this call's size.
    if (smem > SMEM_ATTR ||
        cudaFuncSetAttribute(assign_tc_kernel<T, BN, NKC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SMEM_ATTR)) != cudaSuccess)
        return KM_ERR_CUDA;
    // Persistent clusters (SM pairs): as many as can be resident at once (a pair needs two SMs
    // of one GPC, so this can be below half the SM count), never more than the work items.
    static int resident[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int max_clusters = (dev >= 0 && dev < 64) ? resident[dev] : 0;
    if (max_clusters <= 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(2 * std::max(1, num_sms() / 2)));
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = SMEM_ATTR;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, assign_tc_kernel<T, BN, NKC>, &cfg) != cudaSuccess ||
            max_clusters <= 0) {
            cudaGetLastError();
            max_clusters = std::max(1, num_sms() / 2);
        }
        if (dev >= 0 && dev < 64) resident[dev] = max_clusters;
    }
    const int64_t clusters = std::min<int64_t>(items, max_clusters);
    const unsigned grid = static_cast<unsigned>(2 * clusters);
    assign_tc_kernel<T, BN, NKC><<<grid, NUM_THREADS, smem, st>>>(tmX, tmC, tmA, p);
    return launch_status();
}

// `caug` (workspace) holds B * tc_kp(K) rows of 16 bf16: the centroid side of the extra
// reduction step that adds ||c||^2 / 2 (see km_assign_tc.cuh).
template <typename T>
km_status run_assign_tc(const void *X, km_dtype dt, const void *Cx, const float *cn,
                        const float *w, int64_t B, int64_t N, int64_t K, int64_t d, int32_t *ids,
                        float *mind, double *inertia, int32_t *counts, void *caug, int64_t xld,
                        cudaStream_t st, int32_t *zero_counts = nullptr,
                        double *zero_inertia = nullptr) {
    using namespace km::tc;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return KM_ERR_CUDA;
    const int bn = tc_bn(K, d);
    const int64_t Kp = tc_kp(K, d);
    const int nkc = static_cast<int>(ceil_div(d, KC));
    if (cn && aligned(caug, 16))
        km::caug_rows_kernel<<<static_cast<unsigned>(ceil_div(B * Kp, 256)), 256, 0, st>>>(
            cn, static_cast<int>(B), static_cast<int>(K), static_cast<int>(Kp),
            static_cast<__nv_bfloat16 *>(caug), zero_counts, zero_inertia);
    else
        km::caug_kernel<T><<<static_cast<unsigned>(ceil_div(B * Kp, 8)), 256, 0, st>>>(
            static_cast<const T *>(Cx), cn, static_cast<int>(B), static_cast<int>(K),
            static_cast<int>(Kp), static_cast<int>(d), static_cast<__nv_bfloat16 *>(caug));
    if (launch_status() != KM_OK) return KM_ERR_CUDA;

    const CUtensorMapDataType tdt =
        dt == KM_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap tmX, tmC, tmA;
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                    static_cast<cuuint64_t>(B)};
        // batch elements xld rows apart (a mini-batch of each problem is a strided view)
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(xld * d * 2)};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(KC), static_cast<cuuint32_t>(BM), 1};
        if (enc(&tmX, tdt, 3, const_cast<void *>(X), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return KM_ERR_CUDA;
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(K),
                                    static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(K * d * 2)};
        // each CTA of a pair stages half of every centroid tile
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(KC), static_cast<cuuint32_t>(bn / 2), 1};
        if (enc(&tmC, tdt, 3, const_cast<void *>(Cx), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return KM_ERR_CUDA;
    }
    {
        const cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(Kp), static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[2] = {32, static_cast<cuuint64_t>(Kp * 32)};
        const cuuint32_t box[3] = {16, static_cast<cuuint32_t>(bn / 2), 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, caug, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return KM_ERR_CUDA;
    }
    Params p;
    p.B = static_cast<int>(B);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.d = static_cast<int>(d);
    p.nkc = nkc;
    p.nct = static_cast<int>(Kp / bn);
    p.mtiles = static_cast<int>(ceil_div(N, 2 * BM));   // 256-point items, one per SM pair
    p.stages = 2;
    p.resident = 0;
    p.need_dist = (mind || inertia) ? 1 : 0;
    // M = 256 across the pair; main step with A (the points) negated, so the accumulator
    // collects -<x, c>
    p.idesc_main =
        km::mma_idesc_f16(dt == KM_BF16 ? 1u : 0u, 2 * BM, static_cast<uint32_t>(bn)) | (1u << 13);
    p.idesc_aug = km::mma_idesc_f16(1u, 2 * BM, static_cast<uint32_t>(bn));
    p.w = w;
    p.wld = xld;
    p.ids = ids;
    p.mind = mind;
    p.inertia = inertia;
    p.counts = counts;
    const int64_t items = B * p.mtiles;
    if (items > kMaxIndex) return KM_ERR_UNSUPPORTED;
    // (bn, chunks of 64 along d); bn = 256 with d > 192 never fits (tc_bn narrows it)
#define KM_TC_CASE(BN_, NKC_) \
    if (bn == BN_ && nkc == NKC_) return launch_assign_tc<T, BN_, NKC_>(tmX, tmC, tmA, p, items, st);
    KM_TC_CASE(64, 1) KM_TC_CASE(64, 2) KM_TC_CASE(64, 3) KM_TC_CASE(64, 4)
    KM_TC_CASE(128, 1) KM_TC_CASE(128, 2) KM_TC_CASE(128, 3) KM_TC_CASE(128, 4)
    KM_TC_CASE(256, 1) KM_TC_CASE(256, 2) KM_TC_CASE(256, 3)
#undef KM_TC_CASE
    return KM_ERR_UNSUPPORTED;
}

// Validated-argument assignment; `caug` must hold ws_assign(B, K, d) bytes when the tensor-core
// path can run.
// With accumulate_inertia the objective is added to `inertia` instead of overwriting it (the
// streamed fit sums it over chunks of points).
// counts (optional) receive the per-cluster point counts of the assignment (overwritten).
// X (and w) hold the B batch elements xld >= N rows apart (0: xld = N); ids, mind, counts are
// compact [B, N] / [B, K].
km_status do_assign(const void *X, km_dtype dt, const void *Cx, const float *cn, const float *w,
                    int64_t B, int64_t N, int64_t K, int64_t d, int32_t *ids, float *mind,
                    double *inertia, void *caug, cudaStream_t st, bool accumulate_inertia = false,
                    int32_t *counts = nullptr, int64_t xld = 0) {
    if (xld == 0) xld = N;
    const bool tc = tc_shape_ok(dt, d) && aligned(X, 16) && aligned(Cx, 16) && caug != nullptr &&
                    B * ceil_div(N, 128) <= kMaxIndex;
    double *zero_inertia = inertia && !accumulate_inertia ? inertia : nullptr;
    // the tensor-core path's augmentation kernel clears the counts and the objective itself
    const bool folded = tc && cn && aligned(caug, 16);
    if (!folded) {
        if (zero_inertia && cudaMemsetAsync(zero_inertia, 0, static_cast<size_t>(B) * 8, st) != cudaSuccess)
            return KM_ERR_CUDA;
        if (counts && cudaMemsetAsync(counts, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess)
            return KM_ERR_CUDA;
    }
    if (tc) {
        int32_t *zc = folded ? counts : nullptr;
        double *zi = folded ? zero_inertia : nullptr;
        if (dt == KM_F16)
            return run_assign_tc<__half>(X, dt, Cx, cn, w, B, N, K, d, ids, mind, inertia, counts, caug,
                                         xld, st, zc, zi);
        return run_assign_tc<__nv_bfloat16>(X, dt, Cx, cn, w, B, N, K, d, ids, mind, inertia, counts,
                                            caug, xld, st, zc, zi);
    }
    switch (dt) {
        case KM_F32: return run_assign_simt<float>(X, Cx, w, B, N, K, d, ids, mind, inertia, counts, xld, st);
        case KM_F16: return run_assign_simt<__half>(X, Cx, w, B, N, K, d, ids, mind, inertia, counts, xld, st);
        default:
            return run_assign_simt<__nv_bfloat16>(X, Cx, w, B, N, K, d, ids, mind, inertia, counts, xld, st);
    }
}

template <typename T, int VEC, int G>
km_status run_segreduce_t(const void *X, const float *w, const int32_t *perm,
                          const int32_t *offsets, int64_t B, int64_t N, int64_t K, int64_t d,
                          float *sums, float *wsum, cudaStream_t st) {
    // One wave: as many (warp, range) pairs as warps that can be resident at once, split
    // evenly over the batch elements (each warp walks one contiguous range of sorted positions).
    const int64_t ycols = ceil_div(d, static_cast<int64_t>(G) * VEC);
    static int blocks_per_sm[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int bps = (dev >= 0 && dev < 64) ? blocks_per_sm[dev] : 0;
    if (bps <= 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, km::upd::segreduce_kernel<T, VEC, G>,
                                                          km::upd::SEG_THREADS, 0) != cudaSuccess ||
            bps <= 0) {
            cudaGetLastError();
            bps = 1;
        }
        if (dev >= 0 && dev < 64) blocks_per_sm[dev] = bps;
    }
    const int64_t resident_warps = static_cast<int64_t>(num_sms()) * bps * (km::upd::SEG_THREADS / 32);
    const int64_t want = std::max<int64_t>(1, resident_warps / ycols);
    const int64_t rpb0 = std::max<int64_t>(1, want / B);
    int64_t range = ceil_div(N, rpb0);
    range = std::max<int64_t>(64, ceil_div(range, 32) * 32);
    const int64_t rpb = ceil_div(N, range);
    const int64_t warps = B * rpb;
    dim3 grid(static_cast<unsigned>(ceil_div(warps, km::upd::SEG_THREADS / 32)),
              static_cast<unsigned>(ycols));
    if (ycols > kMaxGridY) return KM_ERR_UNSUPPORTED;
    km::upd::segreduce_kernel<T, VEC, G><<<grid, km::upd::SEG_THREADS, 0, st>>>(
        static_cast<const T *>(X), w, perm, offsets, static_cast<int>(B), static_cast<int>(N),
        static_cast<int>(K), static_cast<int>(d), static_cast<int>(range), static_cast<int>(rpb),
        sums, wsum);
    return launch_status();
}

// The row-per-warp form (d = 32 * V): one wave of (warp, range) pairs, split evenly over the
// batch elements.
template <typename T, int V, bool WEIGHTED>
km_status run_segreduce_rows_w(const void *X, const float *w, const int32_t *perm,
                             const int32_t *offsets, int64_t B, int64_t N, int64_t K,
                             float *sums, float *wsum, cudaStream_t st) {
    using namespace km::upd;
    static int blocks_per_sm[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int bps = (dev >= 0 && dev < 64) ? blocks_per_sm[dev] : 0;
    if (bps <= 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, segreduce_rows_kernel<T, V, WEIGHTED>, ROWS_THREADS, 0) !=
                cudaSuccess ||
            bps <= 0) {
            cudaGetLastError();
            bps = 1;
        }
        if (dev >= 0 && dev < 64) blocks_per_sm[dev] = bps;
    }
    const int64_t resident_warps = static_cast<int64_t>(num_sms()) * bps * (ROWS_THREADS / 32);
    const int64_t rpb0 = std::max<int64_t>(1, resident_warps / B);
    const int64_t range = std::max<int64_t>(64, ceil_div(ceil_div(N, rpb0), 32) * 32);
    const int64_t rpb = ceil_div(N, range);
    const int64_t warps = B * rpb;
    segreduce_rows_kernel<T, V, WEIGHTED><<<static_cast<unsigned>(ceil_div(warps, ROWS_THREADS / 32)), ROWS_THREADS, 0, st>>>(
        static_cast<const T *>(X), w, perm, offsets, static_cast<int>(B), static_cast<int>(N),
        static_cast<int>(K), static_cast<int>(range), static_cast<int>(rpb), sums, wsum);
    return launch_status();
}
template <typename T, int V>
km_status run_segreduce_rows(const void *X, const float *w, const int32_t *perm,
                             const int32_t *offsets, int64_t B, int64_t N, int64_t K,
                             float *sums, float *wsum, cudaStream_t st) {
    // the weight sums are produced exactly when weights are given
    if (w) return run_segreduce_rows_w<T, V, true>(X, w, perm, offsets, B, N, K, sums, wsum, st);
    return run_segreduce_rows_w<T, V, false>(X, w, perm, offsets, B, N, K, sums, wsum, st);
}

template <typename T, int VEC>
km_status segreduce_g(int G, const void *X, const float *w, const int32_t *perm,
                      const int32_t *offsets, int64_t B, int64_t N, int64_t K, int64_t d,
                      float *sums, float *wsum, cudaStream_t st) {
    switch (G) {
        case 1: return run_segreduce_t<T, VEC, 1>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
        case 2: return run_segreduce_t<T, VEC, 2>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
        case 4: return run_segreduce_t<T, VEC, 4>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
        case 8: return run_segreduce_t<T, VEC, 8>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
        case 16: return run_segreduce_t<T, VEC, 16>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
        default: return run_segreduce_t<T, VEC, 32>(X, w, perm, offsets, B, N, K, d, sums, wsum, st);
    }
}

template <typename T>
km_status segreduce_dispatch(const void *X, const float *w, const int32_t *perm,
                             const int32_t *offsets, int64_t B, int64_t N, int64_t K, int64_t d,
                             float *sums, float *wsum, cudaStream_t st) {
    constexpr int VV = 16 / sizeof(T);
    const bool vec = (d % VV == 0) && aligned(X, 16) && aligned(sums, 16);
    const int vw = vec ? VV : 1;
    int64_t lanes = ceil_div(d, vw);
    int G = 1;
    while (G < lanes && G < 32) G <<= 1;
    // row-per-warp form: lane l owns columns [l * V, l * V + V), V = d / 32, with V * sizeof(T)
    // of 4, 8 or 16 bytes (aligned loads and, for 16 bytes of fp32, vector atomics)
    if (d % 32 == 0 && aligned(X, 16) && aligned(sums, 16)) {
        const int64_t vb = (d / 32) * static_cast<int64_t>(sizeof(T));
        if (vb == 4) return run_segreduce_rows<T, 4 / sizeof(T)>(X, w, perm, offsets, B, N, K, sums, wsum, st);
        if (vb == 8) return run_segreduce_rows<T, 8 / sizeof(T)>(X, w, perm, offsets, B, N, K, sums, wsum, st);
        if (vb == 16) return run_segreduce_rows<T, 16 / sizeof(T)>(X, w, perm, offsets, B, N, K, sums, wsum, st);
    }
    if (vec) return segreduce_g<T, VV>(G, X, w, perm, offsets, B, N, K, d, sums, wsum, st);
    return segreduce_g<T, 1>(G, X, w, perm, offsets, B, N, K, d, sums, wsum, st);
}

// sums[B,K,d], counts[B,K] and (when non-null) wsum[B,K] are overwritten.
// Accumulating form (sort_counts != nullptr): sums, wsum and counts are added to, not
// overwritten; the sort of this call's points uses `sort_counts` (B*K int32 scratch), which is
// then added into `counts`.
km_status do_update_partial(const void *X, km_dtype dt, const int32_t *ids, const float *w,
                            int64_t B, int64_t N, int64_t K, int64_t d, float *sums, float *wsum,
                            int32_t *counts, const UpdateWs &u, cudaStream_t st,
                            int32_t *sort_counts = nullptr) {
    int32_t *total_counts = counts;
    if (sort_counts) {
        counts = sort_counts;
        if (cudaMemsetAsync(counts, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess)
            return KM_ERR_CUDA;
    } else if (cudaMemsetAsync(counts, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess ||
               cudaMemsetAsync(sums, 0, static_cast<size_t>(B * K * d) * 4, st) != cudaSuccess ||
               (wsum && cudaMemsetAsync(wsum, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess)) {
        return KM_ERR_CUDA;
    }
    using namespace km::upd;
    const bool smem_bins = K <= SMEM_K_MAX;
    const int64_t ntiles = ceil_div(N, TILE);
    // Attributes are upper bounds for all later launches: always the kernels' largest request.
    if (cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_K_MAX * 4) != cudaSuccess ||
        cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (SMEM_K_MAX + TILE) * 4) != cudaSuccess)
        return KM_ERR_CUDA;
    for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {
        const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
        dim3 grid(static_cast<unsigned>(ntiles), static_cast<unsigned>(nb));
        hist_kernel<<<grid, TILE_THREADS, smem_bins ? K * 4 : 0, st>>>(
            ids + b0 * N, static_cast<int>(N), static_cast<int>(K), counts + b0 * K, smem_bins);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
    }
    scan_kernel<<<static_cast<unsigned>(B), SCAN_THREADS, 0, st>>>(counts, static_cast<int>(K),
                                                                      u.offsets, u.cursor);
    if (launch_status() != KM_OK) return KM_ERR_CUDA;
    const size_t scatter_smem = smem_bins ? static_cast<size_t>(K + TILE) * 4 : 0;
    for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {
        const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
        dim3 grid(static_cast<unsigned>(ntiles), static_cast<unsigned>(nb));
        scatter_kernel<<<grid, TILE_THREADS, scatter_smem, st>>>(
            ids + b0 * N, static_cast<int>(N), static_cast<int>(K), u.cursor + b0 * K,
            u.perm + b0 * N, smem_bins, TILE);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
    }
    km_status s;
    switch (dt) {
        case KM_F32: s = segreduce_dispatch<float>(X, w, u.perm, u.offsets, B, N, K, d, sums, wsum, st); break;
        case KM_F16: s = segreduce_dispatch<__half>(X, w, u.perm, u.offsets, B, N, K, d, sums, wsum, st); break;
        default: s = segreduce_dispatch<__nv_bfloat16>(X, w, u.perm, u.offsets, B, N, K, d, sums, wsum, st);
    }
    if (s != KM_OK || !sort_counts) return s;
    add_i32_kernel<<<static_cast<unsigned>(ceil_div(B * K, 256)), 256, 0, st>>>(total_counts, sort_counts, B * K);
    return launch_status();
}

// ---------------------------------------------------------------- fused update (reduce + divide)

// Rows of d = 32 * V elements of 128, 256 or 512 bytes, 16-byte aligned X, and B * N rows that
// fit the tensor map's 32-bit row coordinate.
inline bool final_ok(km_dtype dt, const void *X, int64_t B, int64_t N, int64_t d) {
    if (d % 32 != 0 || !aligned(X, 16) || B * N >= (int64_t{1} << 31)) return false;
    const int64_t rb = d * static_cast<int64_t>(dtype_size(dt));
    return rb == 128 || rb == 256 || rb == 512;
}

// Ranges of sorted positions for the fused reduce: one CTA per SM of `nw` warps, every warp one
// range of one batch element (ranges need not be whole chunks of 32 positions, so every warp
// gets one), but no range shorter than one chunk: below that a warp's fixed costs outweigh its
// rows. Returns (range, ranges per batch element).
inline void final_ranges(int64_t B, int64_t N, int nw, int64_t &range, int64_t &rpb) {
    const int64_t total = static_cast<int64_t>(std::min(num_sms(), static_cast<int>(kFinalWarpsMax / nw))) * nw;
    const int64_t rpb0 = std::max<int64_t>(1, total / B);
    range = std::max<int64_t>(32, ceil_div(N, rpb0));
    rpb = ceil_div(N, range);   // <= rpb0 < final_rpb_max(B)
}

template <typename T, int V, bool WEIGHTED, bool EMA>
km_status launch_final(const CUtensorMap &tm, km::upd::FinalParams &p, int64_t B, int64_t N,
                       cudaStream_t st) {
    using namespace km::upd;
    constexpr int RB = 32 * V * static_cast<int>(sizeof(T));
    constexpr int NW = fz_warps(RB);
    if (cudaFuncSetAttribute(segreduce_final_kernel<T, V, WEIGHTED, EMA>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, fz_smem(RB)) != cudaSuccess)
        return KM_ERR_CUDA;
    (void)N;
    const int64_t warps = B * p.rpb;
    segreduce_final_kernel<T, V, WEIGHTED, EMA>
        <<<static_cast<unsigned>(ceil_div(warps, NW)), NW * 32, fz_smem(RB), st>>>(tm, p);
    return launch_status();
}

template <typename T, int V>
km_status final_weighted(const CUtensorMap &tm, km::upd::FinalParams &p, int64_t B, int64_t N,
                         cudaStream_t st) {
    if (p.Nc)
        return p.w ? launch_final<T, V, true, true>(tm, p, B, N, st)
                   : launch_final<T, V, false, true>(tm, p, B, N, st);
    return p.w ? launch_final<T, V, true, false>(tm, p, B, N, st)
               : launch_final<T, V, false, false>(tm, p, B, N, st);
}

// The moving-average form of the fused update (e-means) and the view of a mini-batch: batch
// element b's points are rows b * xld + x0 + [0, N) of X (and the same offsets into w).
struct EmaArgs {
    float alpha;
    float *Nc, *eS, *eW;
    int32_t *eCnt;
};

// One sort-inverse update that writes the new centroids directly (no per-cluster sums array):
// counts (overwritten), then C_new and, when given, Cx (X's dtype), cn and wsum. Requires
// final_ok(); `ws` holds carve_final's layout.
template <typename T>
km_status run_update_final(const void *X, km_dtype dt, const int32_t *ids, const float *w,
                           int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                           float *C_new, void *Cx, float *cn, int32_t *counts, bool have_counts,
                           float *wsum, void *ws, cudaStream_t st, int64_t xld = 0, int64_t x0 = 0,
                           const EmaArgs *ema = nullptr) {
    if (xld == 0) xld = N;
    using namespace km::upd;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return KM_ERR_CUDA;
    Carver c(ws);
    const FinalWs f = carve_final(c, B, N, K, d);
    if (!have_counts && cudaMemsetAsync(counts, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess)
        return KM_ERR_CUDA;
    const bool smem_bins = K <= SMEM_K_MAX;
    const int64_t ntiles = ceil_div(N, TILE);
    if (cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_K_MAX * 4) != cudaSuccess ||
        cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (SMEM_K_MAX + TILE) * 4) != cudaSuccess)
        return KM_ERR_CUDA;
    for (int64_t b0 = 0; b0 < B && !have_counts; b0 += kMaxGridY) {
        const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
        dim3 grid(static_cast<unsigned>(ntiles), static_cast<unsigned>(nb));
        hist_kernel<<<grid, TILE_THREADS, smem_bins ? K * 4 : 0, st>>>(
            ids + b0 * N, static_cast<int>(N), static_cast<int>(K), counts + b0 * K, smem_bins);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
    }
    // the reduce's ranges, decided now so the scatter can tabulate where each one starts
    int64_t range = 0, rpb = 0;
    final_ranges(B, N, fz_warps(static_cast<int>(d * sizeof(T))), range, rpb);
    if (rpb > final_rpb_max(B)) return KM_ERR_UNSUPPORTED;   // never (see final_ranges)
    // scatter tiles: halved (down to 1024 points) until every SM has at least one block, so a
    // small problem (an e-means mini-batch) is not sorted by a handful of blocks
    int64_t stile = TILE;
    while (stile > 1024 && B * ceil_div(N, stile) < num_sms()) stile /= 2;
    const int64_t sntiles = ceil_div(N, stile);
    if (smem_bins) {
        // the scan folded into the scatter: slot reservations on a zeroed fill counter
        const size_t smem = static_cast<size_t>(K <= SCATTER_SORT_K_MAX ? ((2 * K + 1 + 3) & ~3) + K + stile
                                                                        : 2 * K + 1) * 4;
        if (cudaMemsetAsync(f.cursor, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess ||
            cudaFuncSetAttribute(scatter_final_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (2 * SMEM_K_MAX + 1) * 4) != cudaSuccess)
            return KM_ERR_CUDA;
        for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {
            const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
            dim3 grid(static_cast<unsigned>(sntiles), static_cast<unsigned>(nb));
            scatter_final_kernel<T><<<grid, TILE_THREADS, smem, st>>>(
                ids + b0 * N, counts + b0 * K, static_cast<int>(N), static_cast<int>(K),
                static_cast<int>(d), static_cast<int>(stile), f.cursor + b0 * K,
                f.offsets + b0 * (K + 1), f.perm + b0 * N, f.arrive + b0 * K, C_prev + b0 * K * d,
                C_new + b0 * K * d, Cx ? static_cast<T *>(Cx) + b0 * K * d : nullptr,
                cn ? cn + b0 * K : nullptr, wsum ? wsum + b0 * K : nullptr,
                ema ? ema->Nc + b0 * K : nullptr, ema ? ema->alpha : 0.f, static_cast<int>(range),
                static_cast<int>(rpb), f.rseg + b0 * rpb);
            if (launch_status() != KM_OK) return KM_ERR_CUDA;
        }
    } else {
        scan_final_kernel<T><<<static_cast<unsigned>(B), SCAN_THREADS, 0, st>>>(
            counts, static_cast<int>(K), static_cast<int>(d), f.offsets, f.cursor, f.arrive, C_prev,
            C_new, static_cast<T *>(Cx), cn, wsum, ema ? ema->Nc : nullptr, ema ? ema->alpha : 0.f);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
        for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {
            const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
            dim3 grid(static_cast<unsigned>(sntiles), static_cast<unsigned>(nb));
            scatter_kernel<<<grid, TILE_THREADS, 0, st>>>(
                ids + b0 * N, static_cast<int>(N), static_cast<int>(K), f.cursor + b0 * K,
                f.perm + b0 * N, 0, static_cast<int>(stile));
            if (launch_status() != KM_OK) return KM_ERR_CUDA;
        }
    }
    // X as [B*xld rows, d] with one-row boxes for the four-row gathers
    CUtensorMap tm;
    const CUtensorMapDataType tdt = dt == KM_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                    : dt == KM_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(B * xld)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * dtype_size(dt)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(d), 1};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, tdt, 2, const_cast<void *>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return KM_ERR_CUDA;
    FinalParams p;
    p.B = static_cast<int>(B);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.range = static_cast<int>(range);
    p.rpb = static_cast<int>(rpb);
    p.rseg = smem_bins ? f.rseg : nullptr;
    p.xld = static_cast<int>(xld);
    p.x0 = static_cast<int>(x0);
    p.perm = f.perm;
    p.offsets = f.offsets;
    p.w = w;
    p.C_prev = C_prev;
    p.C_new = C_new;
    p.Cx = Cx;
    p.cn = cn;
    p.wsum = wsum;
    p.slots = f.slots;
    p.wslots = f.wslots;
    p.arrive = f.arrive;
    p.alpha = ema ? ema->alpha : 0.f;
    p.Nc = ema ? ema->Nc : nullptr;
    p.eS = ema ? ema->eS : nullptr;
    p.eW = ema ? ema->eW : nullptr;
    p.eCnt = ema ? ema->eCnt : nullptr;
    constexpr int VV = static_cast<int>(16 / sizeof(T));   // 16-byte rows per lane at most
    const int64_t V = d / 32;
    if (V == VV) return final_weighted<T, VV>(tm, p, B, N, st);
    if (V == VV / 2) return final_weighted<T, VV / 2>(tm, p, B, N, st);
    if (V == VV / 4) return final_weighted<T, VV / 4>(tm, p, B, N, st);
    return KM_ERR_UNSUPPORTED;
}

km_status update_final_dispatch(const void *X, km_dtype dt, const int32_t *ids, const float *w,
                                int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                                float *C_new, void *Cx, float *cn, int32_t *counts, bool have_counts,
                                float *wsum, void *ws, cudaStream_t st) {
    switch (dt) {
        case KM_F32:
            return run_update_final<float>(X, dt, ids, w, B, N, K, d, C_prev, C_new, Cx, cn, counts,
                                           have_counts, wsum, ws, st);
        case KM_F16:
            return run_update_final<__half>(X, dt, ids, w, B, N, K, d, C_prev, C_new, Cx, cn, counts,
                                            have_counts, wsum, ws, st);
        default:
            return run_update_final<__nv_bfloat16>(X, dt, ids, w, B, N, K, d, C_prev, C_new, Cx, cn,
                                                   counts, have_counts, wsum, ws, st);
    }
}

// The whole update: the fused form where it applies, else the sums array and finalize_kernel.
// `ws` holds ws_update() bytes. wsum (optional) receives the per-cluster weight sums. With
// have_counts the counts already hold the histogram of ids (the assignment wrote it) and the
// fused form skips its own histogram pass.
km_status do_update(const void *X, km_dtype dt, const int32_t *ids, const float *w, int64_t B,
                    int64_t N, int64_t K, int64_t d, const float *C_prev, float *C_new,
                    km_dtype cx_dt, void *Cx, float *cn, int32_t *counts, float *wsum, void *ws,
                    cudaStream_t st, bool have_counts = false) {
    if (final_ok(dt, X, B, N, d) && (!Cx || cx_dt == dt))
        return update_final_dispatch(X, dt, ids, w, B, N, K, d, C_prev, C_new, Cx, cn, counts,
                                     have_counts, wsum, ws, st);
    Carver r(ws);
    UpdateWs u = carve_update(r, B, N, K, d);
    float *ws_w = wsum ? wsum : (w ? u.wsum : nullptr);
    km_status s = do_update_partial(X, dt, ids, w, B, N, K, d, u.sums, ws_w, counts, u, st);
    if (s != KM_OK) return s;
    return finalize_dispatch(u.sums, w ? ws_w : nullptr, counts, C_prev, B * K, d, C_new,
                             Cx ? cx_dt : KM_F32, Cx, cn, st);
}

template <typename T>
km_status run_fit1d(const void *X, const float *w, int64_t B, int64_t N, int64_t K, float *C,
                    int iters, int32_t *ids, double *inertia_hist, float *C_hist, void *ws,
                    cudaStream_t st) {
    int NP = 2;
    while (NP < N) NP <<= 1;
    if (fit1d_rows_ok(N, K, 1)) {
        using namespace km::fit1d;
        Carver r(ws);
        const Fit1dWs g = carve_fit1d(r, B, N);
        // the radix sort splits the row into RADIX_WARPS segments of whole 32-position rounds
        const int NR = static_cast<int>(ceil_div(N, RADIX_WARPS * 32) * RADIX_WARPS * 32);
        const size_t per = 2 * (sizeof(typename SortKey<T>::Word) + 2);   // key and index, twice
        if (cudaFuncSetAttribute(fit1d_sort_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(NMAX * per)) != cudaSuccess)
            return KM_ERR_CUDA;
        fit1d_sort_kernel<T><<<static_cast<unsigned>(B), THREADS, static_cast<size_t>(NR) * per, st>>>(
            static_cast<const T *>(X), w, static_cast<int>(N), NR, g.xs, g.is, g.P0, g.P1,
            inertia_hist ? g.P2 : nullptr);
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
        auto iter = [&](auto kt) {
            fit1d_iter_kernel<T, decltype(kt)::value><<<static_cast<unsigned>(ceil_div(B, ITER_WARPS)),
                                                       ITER_WARPS * 32, 0, st>>>(
                g.xs, g.is, g.P0, g.P1, inertia_hist ? g.P2 : nullptr, static_cast<int>(B),
                static_cast<int>(N), static_cast<int>(K), iters, C, ids, inertia_hist, C_hist);
        };
        if (K <= 4) iter(std::integral_constant<int, 4>{});
        else if (K <= 8) iter(std::integral_constant<int, 8>{});
        else if (K <= 16) iter(std::integral_constant<int, 16>{});
        else iter(std::integral_constant<int, 32>{});
        return launch_status();
    }
    const size_t smem = static_cast<size_t>(NP) * 12;
    if (cudaFuncSetAttribute(km::fit1d::fit1d_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             km::fit1d::NMAX * 12) != cudaSuccess)
        return KM_ERR_CUDA;
    km::fit1d::fit1d_kernel<T><<<static_cast<unsigned>(B), km::fit1d::THREADS, smem, st>>>(
        static_cast<const T *>(X), w, static_cast<int>(B), static_cast<int>(N), NP,
        static_cast<int>(K), iters, C, ids, inertia_hist, C_hist);
    return launch_status();
}

// The whole fit in one cooperative launch (km_fit_small.cuh). Returns KM_ERR_UNSUPPORTED, with
// nothing enqueued, when the CTAs could not all be resident at once.
template <typename T, int DM>
km_status run_fit_small(const void *X, const float *w, int64_t B, int64_t N, int64_t K, int64_t d,
                        float *C, int iters, int32_t *ids, double *inertia_hist, float *C_hist,
                        void *rest, cudaStream_t st) {
    Carver c(rest);
    SmallWs sw = carve_small(c, B, K, d);
    km::fs::Params p;
    p.B = static_cast<int>(B);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.d = static_cast<int>(d);
    p.P = static_cast<int>(ceil_div(N, km::fs::kPts));
    p.iters = iters;
    p.w = w;
    p.C = C;
    p.ids = ids;
    p.inertia_hist = inertia_hist;
    p.C_hist = C_hist;
    p.acc = sw.acc;
    p.iacc = sw.iacc;
    p.bar = sw.bar;
    const size_t smem = static_cast<size_t>(2 * K * d + km::fs::kPts * (d + 3) + K + 1) * 4;
    if (cudaFuncSetAttribute(km::fs::fit_small_kernel<T, DM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return KM_ERR_CUDA;
    const int ctas = static_cast<int>(B) * p.P;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, km::fs::fit_small_kernel<T, DM>,
                                                      km::fs::kThreads, smem) != cudaSuccess)
        return KM_ERR_CUDA;
    if (static_cast<int64_t>(per_sm) * num_sms() < ctas) return KM_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(sw.acc, 0, sw.bytes, st) != cudaSuccess) return KM_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    cfg.blockDim = dim3(km::fs::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the grid barrier needs it
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, km::fs::fit_small_kernel<T, DM>, static_cast<const T *>(X), p) != cudaSuccess)
        return KM_ERR_CUDA;
    return launch_status();
}

template <typename T>
km_status fit_small_dispatch(const void *X, const float *w, int64_t B, int64_t N, int64_t K, int64_t d,
                             float *C, int iters, int32_t *ids, double *inertia_hist, float *C_hist,
                             void *rest, cudaStream_t st) {
    if (d <= 16) return run_fit_small<T, 16>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, rest, st);
    if (d <= 32) return run_fit_small<T, 32>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, rest, st);
    return run_fit_small<T, 64>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, rest, st);
}

km_status do_fit(const void *X, km_dtype dt, const float *w, int64_t B, int64_t N, int64_t K,
                 int64_t d, float *C, int iters, int32_t *ids, double *inertia_hist, float *C_hist,
                 void *ws, cudaStream_t st) {
    Carver c(ws);
    FitWs f = carve_fit(c, B, N, K, d, dt);
    if (fit1d_ok(N, K, d)) {
        switch (dt) {
            case KM_F32: return run_fit1d<float>(X, w, B, N, K, C, iters, ids, inertia_hist, C_hist, f.rest, st);
            case KM_F16: return run_fit1d<__half>(X, w, B, N, K, C, iters, ids, inertia_hist, C_hist, f.rest, st);
            default:
                return run_fit1d<__nv_bfloat16>(X, w, B, N, K, C, iters, ids, inertia_hist, C_hist, f.rest, st);
        }
    }
    if (fit_small_shape_ok(B, N, K, d) && iters > 0 && aligned(X, dtype_size(dt))) {
        km_status s = KM_ERR_UNSUPPORTED;
        switch (dt) {
            case KM_F32: s = fit_small_dispatch<float>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, f.rest, st); break;
            case KM_F16: s = fit_small_dispatch<__half>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, f.rest, st); break;
            default: s = fit_small_dispatch<__nv_bfloat16>(X, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, f.rest, st);
        }
        if (s != KM_ERR_UNSUPPORTED) return s;   // else: the step-by-step fit below
    }
    void *caug = f.rest;  // assignment scratch shares the update region (used one after the other)
    const bool fused = final_ok(dt, X, B, N, d);
    const size_t cbytes = static_cast<size_t>(B * K * d) * 4;
    km_status s = prep_dispatch(C, dt, B * K, d, f.Cx, f.cn, st);
    if (s != KM_OK) return s;
    for (int t = 0; t < iters; ++t) {
        if (C_hist && cudaMemcpyAsync(C_hist + static_cast<int64_t>(t) * B * K * d, C, cbytes,
                                      cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return KM_ERR_CUDA;
        double *in = inertia_hist ? inertia_hist + static_cast<int64_t>(t) * B : nullptr;
        // the assignment writes the counts only where the fused update will use them
        s = do_assign(X, dt, f.Cx, f.cn, w, B, N, K, d, f.ids, nullptr, in, caug, st, false,
                      fused ? f.counts : nullptr);
        if (s != KM_OK) return s;
        s = do_update(X, dt, f.ids, w, B, N, K, d, C, C, dt, f.Cx, f.cn, f.counts, nullptr, f.rest, st,
                      fused);
        if (s != KM_OK) return s;
    }
    if (C_hist && cudaMemcpyAsync(C_hist + static_cast<int64_t>(iters) * B * K * d, C, cbytes,
                                  cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return KM_ERR_CUDA;
    if (ids) return do_assign(X, dt, f.Cx, f.cn, w, B, N, K, d, ids, nullptr, nullptr, caug, st);
    return KM_OK;
}

inline bool elem_aligned(const void *p, km_dtype dt) { return aligned(p, dtype_size(dt)); }

// Out-of-core Lloyd: every iteration streams X (and w) from host memory through two device
// buffers of `chunk` points per batch element. Copies run on their own stream; chunk c's
// assignment and accumulation wait for its copy, and the copy into a buffer waits until the
// chunk that last used it has been processed, so copy c+1 overlaps compute c.
km_status do_fit_stream(const void *Xh, km_dtype dt, const float *wh, int64_t B, int64_t N,
                        int64_t K, int64_t d, float *C, int iters, int64_t chunk,
                        double *inertia_hist, void *ws, cudaStream_t st) {
    Carver c(ws);
    StreamWs sw = carve_stream(c, B, K, d, dt, wh != nullptr, chunk);
    Carver r(sw.rest);
    UpdateWs u = carve_update(r, B, chunk, K, d);
    void *caug = r.base + r.off;
    const size_t esz = dtype_size(dt);
    const int64_t nch = ceil_div(N, chunk);
    cudaStream_t cp = nullptr;
    cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
    km_status s = KM_OK;
    auto cleanup = [&]() {   // resources are released once the enqueued work has finished
        for (int i = 0; i < 2; ++i) {
            if (ready[i]) cudaEventDestroy(ready[i]);
            if (freed[i]) cudaEventDestroy(freed[i]);
        }
        if (cp) cudaStreamDestroy(cp);
    };
    if (cudaStreamCreateWithFlags(&cp, cudaStreamNonBlocking) != cudaSuccess) { cleanup(); return KM_ERR_CUDA; }
    for (int i = 0; i < 2; ++i)
        if (cudaEventCreateWithFlags(&ready[i], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&freed[i], cudaEventDisableTiming) != cudaSuccess) {
            cleanup();
            return KM_ERR_CUDA;
        }
    // the copy stream starts after everything the caller enqueued before this call
    if (cudaEventRecord(freed[0], st) != cudaSuccess || cudaStreamWaitEvent(cp, freed[0], 0) != cudaSuccess) {
        cleanup();
        return KM_ERR_CUDA;
    }
    s = prep_dispatch(C, dt, B * K, d, sw.Cx, sw.cn, st);
    bool used[2] = {false, false};
    for (int t = 0; t < iters && s == KM_OK; ++t) {
        double *in = inertia_hist ? inertia_hist + static_cast<int64_t>(t) * B : nullptr;
        if (cudaMemsetAsync(sw.counts, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess ||
            cudaMemsetAsync(u.sums, 0, static_cast<size_t>(B * K * d) * 4, st) != cudaSuccess ||
            (wh && cudaMemsetAsync(u.wsum, 0, static_cast<size_t>(B * K) * 4, st) != cudaSuccess) ||
            (in && cudaMemsetAsync(in, 0, static_cast<size_t>(B) * 8, st) != cudaSuccess)) {
            s = KM_ERR_CUDA;
            break;
        }
        for (int64_t ch = 0; ch < nch && s == KM_OK; ++ch) {
            const int i = static_cast<int>(ch & 1);
            const int64_t n0 = ch * chunk, n = std::min(chunk, N - n0);
            if (used[i] && cudaStreamWaitEvent(cp, freed[i], 0) != cudaSuccess) { s = KM_ERR_CUDA; break; }
            // rows n0..n0+n of every batch element: one 2-D copy (B rows of n * d elements)
            if (cudaMemcpy2DAsync(sw.xbuf[i], static_cast<size_t>(n * d) * esz,
                                  static_cast<const uint8_t *>(Xh) + static_cast<size_t>(n0 * d) * esz,
                                  static_cast<size_t>(N * d) * esz, static_cast<size_t>(n * d) * esz,
                                  static_cast<size_t>(B), cudaMemcpyHostToDevice, cp) != cudaSuccess ||
                (wh && cudaMemcpy2DAsync(sw.wbuf[i], static_cast<size_t>(n) * 4, wh + n0,
                                         static_cast<size_t>(N) * 4, static_cast<size_t>(n) * 4,
                                         static_cast<size_t>(B), cudaMemcpyHostToDevice, cp) != cudaSuccess) ||
                cudaEventRecord(ready[i], cp) != cudaSuccess || cudaStreamWaitEvent(st, ready[i], 0) != cudaSuccess) {
                s = KM_ERR_CUDA;
                break;
            }
            s = do_assign(sw.xbuf[i], dt, sw.Cx, sw.cn, sw.wbuf[i], B, n, K, d, sw.ids, nullptr, in,
                          caug, st, true);
            if (s != KM_OK) break;
            s = do_update_partial(sw.xbuf[i], dt, sw.ids, sw.wbuf[i], B, n, K, d, u.sums,
                                  wh ? u.wsum : nullptr, sw.counts, u, st, sw.chunk_counts);
            if (s != KM_OK) break;
            if (cudaEventRecord(freed[i], st) != cudaSuccess) { s = KM_ERR_CUDA; break; }
            used[i] = true;
        }
        if (s == KM_OK)
            s = finalize_dispatch(u.sums, wh ? u.wsum : nullptr, sw.counts, C, B * K, d, C, dt, sw.Cx,
                                  sw.cn, st);
    }
    cleanup();
    return s;
}

// e-means: state, epoch totals, one mini-batch's statistics and one problem's batch scratch.
struct EmeansWs {
    void *Cx;
    float *cn, *S, *Nc, *eS, *eW, *bsum, *bw, *sizes;
    int32_t *ids, *eCnt, *bcnt;
    UpdateWs u;
    void *caug;
};
inline EmeansWs carve_emeans(Carver &c, int64_t B, int64_t K, int64_t d, km_dtype dt, int64_t batch) {
    EmeansWs e;
    const size_t kd = static_cast<size_t>(B * K * d), bk = static_cast<size_t>(B * K);
    e.Cx = c.take<uint8_t>(kd * dtype_size(dt));
    e.cn = c.take<float>(bk * 4);
    e.S = c.take<float>(kd * 4);
    e.Nc = c.take<float>(bk * 4);
    e.eS = c.take<float>(kd * 4);
    e.eW = c.take<float>(bk * 4);
    e.bsum = c.take<float>(kd * 4);
    e.bw = c.take<float>(bk * 4);
    e.sizes = c.take<float>(bk * 4);
    e.ids = c.take<int32_t>(static_cast<size_t>(batch) * 4);
    e.eCnt = c.take<int32_t>(bk * 4);
    e.bcnt = c.take<int32_t>(bk * 4);
    e.u = carve_update(c, 1, batch, K, d);
    e.caug = c.base ? c.base + c.off : nullptr;
    c.off += align_up(ws_assign(1, K, d, dt));
    return e;
}

template <typename T>
km_status run_ema(const float *s, const int32_t *cnt, const float *wsum, float alpha, int64_t rows,
                  int64_t d, float *S, float *Nc, float *C, void *Cx, float *cn, float *eS,
                  int32_t *eCnt, float *eW, cudaStream_t st) {
    constexpr int WPB = 8;
    km::em::ema_kernel<T><<<static_cast<unsigned>(ceil_div(rows, WPB)), WPB * 32, 0, st>>>(
        s, cnt, wsum, alpha, rows, static_cast<int>(d), S, Nc, C, static_cast<T *>(Cx), cn, eS,
        eCnt, eW);
    return launch_status();
}

km_status ema_dispatch(km_dtype dt, const float *s, const int32_t *cnt, const float *wsum,
                       float alpha, int64_t rows, int64_t d, float *S, float *Nc, float *C,
                       void *Cx, float *cn, float *eS, int32_t *eCnt, float *eW, cudaStream_t st) {
    switch (dt) {
        case KM_F16: return run_ema<__half>(s, cnt, wsum, alpha, rows, d, S, Nc, C, Cx, cn, eS, eCnt, eW, st);
        case KM_BF16:
            return run_ema<__nv_bfloat16>(s, cnt, wsum, alpha, rows, d, S, Nc, C, Cx, cn, eS, eCnt, eW, st);
        default: return run_ema<float>(s, cnt, wsum, alpha, rows, d, S, Nc, C, Cx, cn, eS, eCnt, eW, st);
    }
}

km_status run_split(float *sizes, const float *u, float eps, int64_t B, int64_t K, int64_t d,
                    float *C, float *Nc, float *S, int32_t *donors, cudaStream_t st) {
    km::em::split_kernel<<<static_cast<unsigned>(B), km::em::SPLIT_THREADS, 0, st>>>(
        sizes, u, eps, static_cast<int>(K), static_cast<int>(d), C, Nc, S, donors);
    return launch_status();
}

// Step size of step t of T: cosine decay from alpha0 towards 0.1 alpha0 (evaluated in fp64).
inline float emeans_alpha(float alpha0, int64_t t, int64_t T) {
    const double pi = 3.14159265358979323846;
    return static_cast<float>(static_cast<double>(alpha0) *
                              (0.1 + 0.9 * (1.0 + std::cos(pi * static_cast<double>(t) /
                                                           static_cast<double>(T))) / 2.0));
}

// The e-means run: consecutive mini-batches of `batch` points per problem, each assigned against
// the current centroids and folded into the moving averages; dead clusters (no point in an
// epoch) split between epochs when uniforms are given; at the end the centroids move to the mean
// of the points the last epoch assigned to them.
km_status do_emeans(const void *X, km_dtype dt, const float *w, int64_t B, int64_t N, int64_t K,
                    int64_t d, float *C, int64_t batch, int epochs, float alpha0,
                    const float *split_u, float eps, double *sse_hist, void *ws, cudaStream_t st) {
    Carver c(ws);
    EmeansWs e = carve_emeans(c, B, K, d, dt, batch);
    const size_t esz = dtype_size(dt);
    const int64_t rows = B * K;
    const size_t kd4 = static_cast<size_t>(rows * d) * 4;
    if (cudaMemcpyAsync(e.S, C, kd4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return KM_ERR_CUDA;
    km::em::fill_f32_kernel<<<static_cast<unsigned>(ceil_div(rows, 256)), 256, 0, st>>>(e.Nc, 1.f, rows);
    if (launch_status() != KM_OK) return KM_ERR_CUDA;
    km_status s = prep_dispatch(C, dt, rows, d, e.Cx, e.cn, st);
    if (s != KM_OK) return s;
    const int64_t steps = ceil_div(N, batch), T = static_cast<int64_t>(epochs) * steps;
    for (int ep = 0; ep < epochs; ++ep) {
        double *sse = sse_hist ? sse_hist + static_cast<int64_t>(ep) * B : nullptr;
        if (cudaMemsetAsync(e.eS, 0, kd4, st) != cudaSuccess ||
            cudaMemsetAsync(e.eCnt, 0, static_cast<size_t>(rows) * 4, st) != cudaSuccess ||
            cudaMemsetAsync(e.eW, 0, static_cast<size_t>(rows) * 4, st) != cudaSuccess ||
            (sse && cudaMemsetAsync(sse, 0, static_cast<size_t>(B) * 8, st) != cudaSuccess))
            return KM_ERR_CUDA;
        for (int64_t stp = 0; stp < steps; ++stp) {
            const int64_t n0 = stp * batch, n = std::min(batch, N - n0);
            for (int64_t b = 0; b < B; ++b) {
                const void *Xb = static_cast<const uint8_t *>(X) + static_cast<size_t>((b * N + n0) * d) * esz;
                const float *wb = w ? w + b * N + n0 : nullptr;
                const void *Cxb = static_cast<const uint8_t *>(e.Cx) + static_cast<size_t>(b * K * d) * esz;
                s = do_assign(Xb, dt, Cxb, e.cn + b * K, wb, 1, n, K, d, e.ids, nullptr,
                              sse ? sse + b : nullptr, e.caug, st, true);
                if (s != KM_OK) return s;
                s = do_update_partial(Xb, dt, e.ids, wb, 1, n, K, d, e.bsum + b * K * d,
                                      w ? e.bw + b * K : nullptr, e.bcnt + b * K, e.u, st);
                if (s != KM_OK) return s;
            }
            s = ema_dispatch(dt, e.bsum, e.bcnt, w ? e.bw : nullptr,
                             emeans_alpha(alpha0, static_cast<int64_t>(ep) * steps + stp, T), rows, d,
                             e.S, e.Nc, C, e.Cx, e.cn, e.eS, e.eCnt, w ? e.eW : nullptr, st);
            if (s != KM_OK) return s;
        }
        if (split_u && ep + 1 < epochs) {
            // sizes = the epoch's point counts (weight sums when weighted)
            if (w) {
                if (cudaMemcpyAsync(e.sizes, e.eW, static_cast<size_t>(rows) * 4,
                                    cudaMemcpyDeviceToDevice, st) != cudaSuccess)
                    return KM_ERR_CUDA;
            } else {
                km::em::i32_to_f32_kernel<<<static_cast<unsigned>(ceil_div(rows, 256)), 256, 0, st>>>(
                    e.eCnt, e.sizes, rows);
                if (launch_status() != KM_OK) return KM_ERR_CUDA;
            }
            s = run_split(e.sizes, split_u + static_cast<int64_t>(ep) * rows, eps, B, K, d, C, e.Nc,
                          e.S, nullptr, st);
            if (s != KM_OK) return s;
            s = prep_dispatch(C, dt, rows, d, e.Cx, e.cn, st);
            if (s != KM_OK) return s;
        }
    }
    if (epochs > 0)
        return finalize_dispatch(e.eS, w ? e.eW : nullptr, e.eCnt, C, rows, d, C, dt, e.Cx, e.cn, st);
    return KM_OK;
}


// e-means with the fused update (rows of 128, 256 or 512 bytes): the state is (C, Nc) with
// S = C * Nc, every mini-batch of all B problems is one strided view of X, and per mini-batch
// there is one assignment (labels, batch counts, the objective added to the epoch's) and one
// sort-inverse update whose finalize applies the moving average.
struct EmeansFz {
    void *Cx;
    float *cn, *Nc, *eS, *eW, *sizes;
    int32_t *ids, *eCnt, *bcnt;
    void *fin;    // the fused update's scratch, then the assignment's (used one after the other)
};
inline EmeansFz carve_emeans_fused(Carver &c, int64_t B, int64_t K, int64_t d, km_dtype dt, int64_t batch) {
    EmeansFz e;
    const size_t kd = static_cast<size_t>(B * K * d), bk = static_cast<size_t>(B * K);
    e.Cx = c.take<uint8_t>(kd * dtype_size(dt));
    e.cn = c.take<float>(bk * 4);
    e.Nc = c.take<float>(bk * 4);
    e.eS = c.take<float>(kd * 4);
    e.eW = c.take<float>(bk * 4);
    e.sizes = c.take<float>(bk * 4);
    e.ids = c.take<int32_t>(static_cast<size_t>(B * batch) * 4);
    e.eCnt = c.take<int32_t>(bk * 4);
    e.bcnt = c.take<int32_t>(bk * 4);
    e.fin = c.base ? c.base + c.off : nullptr;
    Carver f(nullptr);
    carve_final(f, B, batch, K, d);
    c.off += std::max(f.off, align_up(ws_assign(B, K, d, dt)));
    return e;
}

template <typename T>
km_status run_emeans_fused(const void *X, km_dtype dt, const float *w, int64_t B, int64_t N,
                           int64_t K, int64_t d, float *C, int64_t batch, int epochs, float alpha0,
                           const float *split_u, float eps, double *sse_hist, void *ws,
                           cudaStream_t st) {
    Carver c(ws);
    EmeansFz e = carve_emeans_fused(c, B, K, d, dt, batch);
    const size_t esz = dtype_size(dt);
    const int64_t rows = B * K;
    km::em::fill_f32_kernel<<<static_cast<unsigned>(ceil_div(rows, 256)), 256, 0, st>>>(e.Nc, 1.f, rows);
    if (launch_status() != KM_OK) return KM_ERR_CUDA;
    km_status s = prep_dispatch(C, dt, rows, d, e.Cx, e.cn, st);
    if (s != KM_OK) return s;
    const int64_t steps = ceil_div(N, batch), T_all = static_cast<int64_t>(epochs) * steps;
    for (int ep = 0; ep < epochs; ++ep) {
        const bool last = ep + 1 == epochs;
        double *sse = sse_hist ? sse_hist + static_cast<int64_t>(ep) * B : nullptr;
        // the epoch's sums are needed only for the final shift, so only the last epoch keeps them
        if (cudaMemsetAsync(e.eCnt, 0, static_cast<size_t>(rows) * 4, st) != cudaSuccess ||
            (w && cudaMemsetAsync(e.eW, 0, static_cast<size_t>(rows) * 4, st) != cudaSuccess) ||
            (last && cudaMemsetAsync(e.eS, 0, static_cast<size_t>(rows * d) * 4, st) != cudaSuccess) ||
            (sse && cudaMemsetAsync(sse, 0, static_cast<size_t>(B) * 8, st) != cudaSuccess))
            return KM_ERR_CUDA;
        for (int64_t stp = 0; stp < steps; ++stp) {
            const int64_t n0 = stp * batch, n = std::min(batch, N - n0);
            const void *Xv = static_cast<const uint8_t *>(X) + static_cast<size_t>(n0 * d) * esz;
            s = do_assign(Xv, dt, e.Cx, e.cn, w ? w + n0 : nullptr, B, n, K, d, e.ids, nullptr, sse,
                          e.fin, st, true, e.bcnt, N);
            if (s != KM_OK) return s;
            const EmaArgs ea{emeans_alpha(alpha0, static_cast<int64_t>(ep) * steps + stp, T_all), e.Nc,
                             last ? e.eS : nullptr, w ? e.eW : nullptr, e.eCnt};
            s = run_update_final<T>(X, dt, e.ids, w, B, n, K, d, C, C, e.Cx, e.cn, e.bcnt, true, nullptr,
                                    e.fin, st, N, n0, &ea);
            if (s != KM_OK) return s;
        }
        if (split_u && !last) {
            // sizes = the epoch's point counts (weight sums when weighted)
            if (w) {
                if (cudaMemcpyAsync(e.sizes, e.eW, static_cast<size_t>(rows) * 4, cudaMemcpyDeviceToDevice,
                                    st) != cudaSuccess)
                    return KM_ERR_CUDA;
            } else {
                km::em::i32_to_f32_kernel<<<static_cast<unsigned>(ceil_div(rows, 256)), 256, 0, st>>>(
                    e.eCnt, e.sizes, rows);
                if (launch_status() != KM_OK) return KM_ERR_CUDA;
            }
            s = run_split(e.sizes, split_u + static_cast<int64_t>(ep) * rows, eps, B, K, d, C, e.Nc,
                          nullptr, nullptr, st);
            if (s != KM_OK) return s;
            s = prep_dispatch(C, dt, rows, d, e.Cx, e.cn, st);
            if (s != KM_OK) return s;
        }
    }
    if (epochs > 0)
        return finalize_dispatch(e.eS, w ? e.eW : nullptr, e.eCnt, C, rows, d, C, dt, e.Cx, e.cn, st);
    return KM_OK;
}

template <typename T> struct TypeTag { using type = T; };

inline bool emeans_fused_ok(km_dtype dt, const void *X, int64_t B, int64_t N, int64_t d) {
    return final_ok(dt, X, B, N, d);
}

template <typename T, int LOGP>
void launch_encode1d(const void *X, int64_t N, const float *C, int K, uint8_t *codes, dim3 grid,
                     bool vec, cudaStream_t st) {
    using namespace km::cb;
    const T *x = static_cast<const T *>(X);
    if (vec) encode1d_kernel<T, LOGP, true><<<grid, ENC_THREADS, 0, st>>>(x, N, C, K, codes);
    else encode1d_kernel<T, LOGP, false><<<grid, ENC_THREADS, 0, st>>>(x, N, C, K, codes);
}

template <typename T, int... L>
void encode1d_by_logp(int logp, const void *X, int64_t N, const float *C, int K, uint8_t *codes,
                      dim3 grid, bool vec, cudaStream_t st, std::integer_sequence<int, L...>) {
    ((logp == L + 1 ? launch_encode1d<T, L + 1>(X, N, C, K, codes, grid, vec, st) : void()), ...);
}

}  // namespace

// =================================================================== exported C ABI

extern "C" {

const char *km_status_string(km_status s) {
    switch (s) {
        case KM_OK: return "KM_OK";
        case KM_ERR_INVALID_ARG: return "KM_ERR_INVALID_ARG";
        case KM_ERR_UNSUPPORTED: return "KM_ERR_UNSUPPORTED";
        case KM_ERR_WORKSPACE: return "KM_ERR_WORKSPACE";
        case KM_ERR_CUDA: return "KM_ERR_CUDA";
        case KM_ERR_DEVICE_TIMEOUT: return "KM_ERR_DEVICE_TIMEOUT";
    }
    return "KM_ERR_UNKNOWN";
}

int km_abi_version(void) { return 2; }

int km_assign_uses_tensor_cores(km_dtype dtype, int64_t d, const void *X, const void *Cx) {
    return valid_dtype(dtype) && tc_shape_ok(dtype, d) && aligned(X, 16) && aligned(Cx, 16) ? 1 : 0;
}

size_t km_workspace_size(km_op op, int64_t B, int64_t N, int64_t K, int64_t d, km_dtype dtype,
                         int weighted, int iters) {
    if (!sizes_ok(B, N, K, d) || !valid_dtype(dtype) || iters < 0) return 0;
    Carver c(nullptr);
    switch (op) {
        case KM_OP_ASSIGN: return ws_assign(B, K, d, dtype);
        case KM_OP_UPDATE: return ws_update(B, N, K, d);
        case KM_OP_FIT: carve_fit(c, B, N, K, d, dtype); return c.off;
        case KM_OP_FIT_HOST: carve_host(c, B, N, K, d, dtype, weighted != 0, iters); return c.off;
    }
    return 0;
}

km_status km_prep(const float *C, km_dtype dtype, int64_t B, int64_t K, int64_t d, void *Cx,
                  float *cn, void *stream) {
    if (!C || (!Cx && !cn) || !valid_dtype(dtype) || !sizes_ok(B, 1, K, d) || !aligned(C, 4) ||
        (Cx && !elem_aligned(Cx, dtype)) || (cn && !aligned(cn, 4)))
        return KM_ERR_INVALID_ARG;
    return prep_dispatch(C, dtype, B * K, d, Cx, cn, S(stream));
}

km_status km_assign(const void *X, km_dtype dtype, const void *Cx, const float *cn, const float *w,
                    int64_t B, int64_t N, int64_t K, int64_t d, int32_t *ids, float *mind,
                    double *inertia, int32_t *counts, void *ws, size_t ws_bytes, void *stream) {
    if (!X || !Cx || !ids || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) ||
        !elem_aligned(X, dtype) || !elem_aligned(Cx, dtype) || !aligned(ids, 4) ||
        (w && !aligned(w, 4)) || (cn && !aligned(cn, 4)) || (mind && !aligned(mind, 4)) ||
        (inertia && !aligned(inertia, 8)) || (counts && !aligned(counts, 4)))
        return KM_ERR_INVALID_ARG;
    const size_t need = ws_assign(B, K, d, dtype);
    if (need && (!ws || ws_bytes < need || !aligned(ws, kAlign))) return KM_ERR_WORKSPACE;
    return do_assign(X, dtype, Cx, cn, w, B, N, K, d, ids, mind, inertia, need ? ws : nullptr,
                     S(stream), false, counts);
}

km_status km_update_partial(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                            int64_t B, int64_t N, int64_t K, int64_t d, float *sums, float *wsum,
                            int32_t *counts, void *ws, size_t ws_bytes, void *stream) {
    if (!X || !ids || !sums || !counts || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) ||
        !elem_aligned(X, dtype) || !aligned(ids, 4) || !aligned(sums, 4) || !aligned(counts, 4) ||
        (w && !aligned(w, 4)) || (wsum && !aligned(wsum, 4)) || (w && !wsum))
        return KM_ERR_INVALID_ARG;
    Carver c(nullptr);
    carve_update(c, B, N, K, d);
    if (!ws || ws_bytes < c.off || !aligned(ws, kAlign)) return KM_ERR_WORKSPACE;
    Carver r(ws);
    UpdateWs u = carve_update(r, B, N, K, d);
    return do_update_partial(X, dtype, ids, w, B, N, K, d, sums, wsum, counts, u, S(stream));
}

km_status km_finalize(const float *sums, const float *wsum, const int32_t *counts,
                      const float *C_prev, int64_t B, int64_t K, int64_t d, float *C_new,
                      km_dtype cx_dtype, void *Cx, float *cn, void *stream) {
    if (!sums || !counts || !C_prev || !C_new || !sizes_ok(B, 1, K, d) || !valid_dtype(cx_dtype) ||
        (Cx && !elem_aligned(Cx, cx_dtype)))
        return KM_ERR_INVALID_ARG;
    return finalize_dispatch(sums, wsum, counts, C_prev, B * K, d, C_new, Cx ? cx_dtype : KM_F32,
                             Cx, cn, S(stream));
}

km_status km_update(const void *X, km_dtype dtype, const int32_t *ids, const float *w, int64_t B,
                    int64_t N, int64_t K, int64_t d, const float *C_prev, float *C_new,
                    int32_t *counts, float *wsum, void *ws, size_t ws_bytes, void *stream) {
    if (!X || !ids || !C_prev || !C_new || !counts || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) ||
        !elem_aligned(X, dtype) || !aligned(ids, 4) || !aligned(counts, 4) || !aligned(C_prev, 4) ||
        !aligned(C_new, 4) || (w && !aligned(w, 4)) || (wsum && !aligned(wsum, 4)))
        return KM_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ws_update(B, N, K, d) || !aligned(ws, kAlign)) return KM_ERR_WORKSPACE;
    return do_update(X, dtype, ids, w, B, N, K, d, C_prev, C_new, KM_F32, nullptr, nullptr, counts,
                     wsum, ws, S(stream));
}

km_status km_update_next(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                         int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                         float *C_new, void *Cx, float *cn, int32_t *counts, int counts_ready,
                         float *wsum, void *ws, size_t ws_bytes, void *stream) {
    if (!X || !ids || !C_prev || !C_new || !Cx || !cn || !counts || !valid_dtype(dtype) ||
        !sizes_ok(B, N, K, d) || !elem_aligned(X, dtype) || !aligned(ids, 4) || !aligned(counts, 4) ||
        !aligned(C_prev, 4) || !aligned(C_new, 4) || !elem_aligned(Cx, dtype) || !aligned(cn, 4) ||
        (w && !aligned(w, 4)) || (wsum && !aligned(wsum, 4)))
        return KM_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ws_update(B, N, K, d) || !aligned(ws, kAlign)) return KM_ERR_WORKSPACE;
    return do_update(X, dtype, ids, w, B, N, K, d, C_prev, C_new, dtype, Cx, cn, counts, wsum, ws,
                     S(stream), counts_ready != 0);
}

km_status km_init_grid1d(const void *X, km_dtype dtype, int64_t B, int64_t N, int64_t K, float *C,
                         void *stream) {
    if (!X || !C || !valid_dtype(dtype) || !sizes_ok(B, N, K, 1) || !elem_aligned(X, dtype) ||
        !aligned(C, 4))
        return KM_ERR_INVALID_ARG;
    const unsigned grid = static_cast<unsigned>(B);
    switch (dtype) {
        case KM_F32:
            km::fit1d::grid_init_kernel<float><<<grid, 256, 0, S(stream)>>>(
                static_cast<const float *>(X), static_cast<int>(N), static_cast<int>(K), C);
            break;
        case KM_F16:
            km::fit1d::grid_init_kernel<__half><<<grid, 256, 0, S(stream)>>>(
                static_cast<const __half *>(X), static_cast<int>(N), static_cast<int>(K), C);
            break;
        default:
            km::fit1d::grid_init_kernel<__nv_bfloat16><<<grid, 256, 0, S(stream)>>>(
                static_cast<const __nv_bfloat16 *>(X), static_cast<int>(N), static_cast<int>(K), C);
    }
    return launch_status();
}

km_status km_fit(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N, int64_t K,
                 int64_t d, float *C, int iters, int32_t *ids, double *inertia_hist, float *C_hist,
                 void *ws, size_t ws_bytes, void *stream) {
    if (!X || !C || iters < 0 || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) ||
        !elem_aligned(X, dtype) || !aligned(C, 4) || (w && !aligned(w, 4)) ||
        (ids && !aligned(ids, 4)) || (inertia_hist && !aligned(inertia_hist, 8)) ||
        (C_hist && !aligned(C_hist, 4)))
        return KM_ERR_INVALID_ARG;
    if (!fit1d_ok(N, K, d) || fit1d_rows_ok(N, K, d)) {   // the fused per-row kernel needs none
        Carver c(nullptr);
        carve_fit(c, B, N, K, d, dtype);
        if (!ws || ws_bytes < c.off || !aligned(ws, kAlign)) return KM_ERR_WORKSPACE;
    }
    return do_fit(X, dtype, w, B, N, K, d, C, iters, ids, inertia_hist, C_hist, ws, S(stream));
}

size_t km_stream_workspace_size(int64_t B, int64_t K, int64_t d, km_dtype dtype, int weighted,
                                int64_t chunk) {
    if (!sizes_ok(B, chunk, K, d) || !valid_dtype(dtype)) return 0;
    Carver c(nullptr);
    carve_stream(c, B, K, d, dtype, weighted != 0, chunk);
    return c.off;
}

km_status km_fit_stream(const void *X_host, km_dtype dtype, const float *w_host, int64_t B,
                        int64_t N, int64_t K, int64_t d, float *C, int iters, int64_t chunk,
                        double *inertia_hist, void *ws, size_t ws_bytes, void *stream) {
    if (!X_host || !C || iters < 0 || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) || chunk < 1 ||
        !aligned(C, 4) || (inertia_hist && !aligned(inertia_hist, 8)) ||
        !aligned(X_host, dtype_size(dtype)) || (w_host && !aligned(w_host, 4)))
        return KM_ERR_INVALID_ARG;
    chunk = std::min(chunk, N);
    if (!ws || ws_bytes < km_stream_workspace_size(B, K, d, dtype, w_host != nullptr, chunk) ||
        !aligned(ws, kAlign))
        return KM_ERR_WORKSPACE;
    return do_fit_stream(X_host, dtype, w_host, B, N, K, d, C, iters, chunk, inertia_hist, ws, S(stream));
}

size_t km_emeans_workspace_size(int64_t B, int64_t K, int64_t d, km_dtype dtype, int weighted,
                                int64_t batch) {
    (void)weighted;   // the weight-sum arrays are always carved
    if (!sizes_ok(B, batch, K, d) || !valid_dtype(dtype)) return 0;
    Carver c(nullptr), f(nullptr);
    carve_emeans(c, B, K, d, dtype, batch);
    carve_emeans_fused(f, B, K, d, dtype, batch);
    return std::max(c.off, f.off);   // covers whichever form runs
}

km_status km_emeans_fit(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N,
                        int64_t K, int64_t d, float *C, int64_t batch, int epochs, float alpha0,
                        const float *split_u, float split_eps, double *sse_hist, void *ws,
                        size_t ws_bytes, void *stream) {
    if (!X || !C || epochs < 0 || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) || batch < 1 ||
        !(alpha0 > 0.f && alpha0 <= 1.f) || !(split_eps >= 0.f && split_eps < 1.f) ||
        !elem_aligned(X, dtype) || !aligned(C, 4) || (w && !aligned(w, 4)) ||
        (split_u && !aligned(split_u, 4)) || (sse_hist && !aligned(sse_hist, 8)))
        return KM_ERR_INVALID_ARG;
    batch = std::min(batch, N);
    if (!ws || ws_bytes < km_emeans_workspace_size(B, K, d, dtype, w != nullptr, batch) ||
        !aligned(ws, kAlign))
        return KM_ERR_WORKSPACE;
    if (emeans_fused_ok(dtype, X, B, N, d)) {
        switch (dtype) {
            case KM_F32:
                return run_emeans_fused<float>(X, dtype, w, B, N, K, d, C, batch, epochs, alpha0, split_u,
                                               split_eps, sse_hist, ws, S(stream));
            case KM_F16:
                return run_emeans_fused<__half>(X, dtype, w, B, N, K, d, C, batch, epochs, alpha0, split_u,
                                                split_eps, sse_hist, ws, S(stream));
            default:
                return run_emeans_fused<__nv_bfloat16>(X, dtype, w, B, N, K, d, C, batch, epochs, alpha0,
                                                       split_u, split_eps, sse_hist, ws, S(stream));
        }
    }
    return do_emeans(X, dtype, w, B, N, K, d, C, batch, epochs, alpha0, split_u, split_eps,
                     sse_hist, ws, S(stream));
}

km_status km_split_dead(float *C, float *sizes, const float *u, float eps, int64_t B, int64_t K,
                        int64_t d, float *Nc, float *S_sums, int32_t *donors, void *stream) {
    if (!C || !sizes || !u || !sizes_ok(B, 1, K, d) || !(eps >= 0.f && eps < 1.f) ||
        !aligned(C, 4) || !aligned(sizes, 4) || !aligned(u, 4) || (Nc && !aligned(Nc, 4)) ||
        (S_sums && !aligned(S_sums, 4)) || (donors && !aligned(donors, 4)))
        return KM_ERR_INVALID_ARG;
    return run_split(sizes, u, eps, B, K, d, C, Nc, S_sums, donors, S(stream));
}

km_status km_encode1d(const void *X, km_dtype dtype, int64_t B, int64_t N, const float *C,
                      int64_t K, uint8_t *codes, void *stream) {
    using namespace km::cb;
    if (!X || !C || !codes || !valid_dtype(dtype) || !sizes_ok(B, N, K, 1) || K > ENC_KMAX ||
        !elem_aligned(X, dtype) || !aligned(C, 4))
        return KM_ERR_INVALID_ARG;
    cudaStream_t st = S(stream);
    const size_t esz = dtype_size(dtype);
    const int k = static_cast<int>(K);
    const int logp = enc_logp(k);   // 1 .. 9 for K = 1 .. 256
    // the vector form: whole 16-value groups, every row starting on a 16-byte boundary
    const bool vec = N % ENC_VPT == 0 && aligned(X, 16) && aligned(codes, 16);
    using Seq = std::make_integer_sequence<int, 9>;
    for (int64_t b0 = 0; b0 < B; b0 += kMaxGridY) {   // rows in slices of the grid's y extent
        const int64_t nb = std::min<int64_t>(kMaxGridY, B - b0);
        const dim3 grid(static_cast<unsigned>(ceil_div(N, ENC_THREADS * ENC_VPT)), static_cast<unsigned>(nb));
        const void *Xs = static_cast<const uint8_t *>(X) + static_cast<size_t>(b0 * N) * esz;
        const float *Cs = C + b0 * K;
        uint8_t *out = codes + b0 * N;
        switch (dtype) {
            case KM_F32: encode1d_by_logp<float>(logp, Xs, N, Cs, k, out, grid, vec, st, Seq{}); break;
            case KM_F16: encode1d_by_logp<__half>(logp, Xs, N, Cs, k, out, grid, vec, st, Seq{}); break;
            default: encode1d_by_logp<__nv_bfloat16>(logp, Xs, N, Cs, k, out, grid, vec, st, Seq{});
        }
        if (launch_status() != KM_OK) return KM_ERR_CUDA;
    }
    return KM_OK;
}

km_status km_init_kmeanspp1d(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N,
                             int64_t K, const float *u, float *C, int32_t *chosen, void *stream) {
    using namespace km::cb;
    if (!X || !u || !C || !valid_dtype(dtype) || !sizes_ok(B, N, K, 1) ||
        !elem_aligned(X, dtype) || (w && !aligned(w, 4)) || !aligned(u, 4) || !aligned(C, 4) ||
        (chosen && !aligned(chosen, 4)))
        return KM_ERR_INVALID_ARG;
    if (N > PP_NMAX) return KM_ERR_UNSUPPORTED;
    cudaStream_t st = S(stream);
    const unsigned grid = static_cast<unsigned>(B);
    const int n = static_cast<int>(N), k = static_cast<int>(K);
    // rows of up to 4096 values: 8 points per thread (two blocks per SM), else 16
    auto run = [&](auto tag, auto per) {
        using T = typename decltype(tag)::type;
        kmeanspp1d_kernel<T, decltype(per)::value><<<grid, PP_THREADS, 0, st>>>(
            static_cast<const T *>(X), w, n, k, u, C, chosen);
    };
    const bool small = N <= PP_THREADS * 8;
    switch (dtype) {
        case KM_F32:
            if (small) run(TypeTag<float>{}, std::integral_constant<int, 8>{});
            else run(TypeTag<float>{}, std::integral_constant<int, PP_PER>{});
            break;
        case KM_F16:
            if (small) run(TypeTag<__half>{}, std::integral_constant<int, 8>{});
            else run(TypeTag<__half>{}, std::integral_constant<int, PP_PER>{});
            break;
        default:
            if (small) run(TypeTag<__nv_bfloat16>{}, std::integral_constant<int, 8>{});
            else run(TypeTag<__nv_bfloat16>{}, std::integral_constant<int, PP_PER>{});
    }
    return launch_status();
}

km_status km_fit_host(const void *X_host, km_dtype dtype, const float *w_host, int64_t B,
                      int64_t N, int64_t K, int64_t d, float *C_host, int iters, int32_t *ids_host,
                      double *inertia_host, void *ws, size_t ws_bytes, void *stream) {
    if (!X_host || !C_host || iters < 0 || !valid_dtype(dtype) || !sizes_ok(B, N, K, d))
        return KM_ERR_INVALID_ARG;
    Carver c(nullptr);
    carve_host(c, B, N, K, d, dtype, w_host != nullptr, iters);
    if (!ws || ws_bytes < c.off || !aligned(ws, kAlign)) return KM_ERR_WORKSPACE;
    Carver r(ws);
    HostWs h = carve_host(r, B, N, K, d, dtype, w_host != nullptr, iters);
    cudaStream_t st = S(stream);
    const size_t xb = static_cast<size_t>(B * N * d) * dtype_size(dtype);
    const size_t cb = static_cast<size_t>(B * K * d) * 4;
    // One iteration without labels: X is needed once, so it is streamed in 16 chunks (the
    // out-of-core fit) and each chunk's assignment and accumulation overlap the next chunk's
    // copy; the X staging area serves as that fit's workspace.
    if (iters == 1 && !ids_host && xb >= (size_t{64} << 20)) {
        const int64_t chunk = std::max<int64_t>(256, (ceil_div(N, 16) + 255) / 256 * 256);
        const size_t need = km_stream_workspace_size(B, K, d, dtype, w_host != nullptr, chunk);
        if (chunk < N && need > 0 && need <= xb) {
            if (cudaMemcpyAsync(h.C, C_host, cb, cudaMemcpyHostToDevice, st) != cudaSuccess)
                return KM_ERR_CUDA;
            km_status s = do_fit_stream(X_host, dtype, w_host, B, N, K, d, h.C, 1, chunk,
                                        inertia_host ? h.inertia : nullptr, h.X, st);
            if (s != KM_OK) return s;
            if (cudaMemcpyAsync(C_host, h.C, cb, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
                (inertia_host && cudaMemcpyAsync(inertia_host, h.inertia, static_cast<size_t>(B) * 8,
                                                 cudaMemcpyDeviceToHost, st) != cudaSuccess))
                return KM_ERR_CUDA;
            return cudaStreamSynchronize(st) == cudaSuccess ? KM_OK : KM_ERR_CUDA;
        }
    }
    if (cudaMemcpyAsync(h.X, X_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        (w_host && cudaMemcpyAsync(h.w, w_host, static_cast<size_t>(B * N) * 4,
                                   cudaMemcpyHostToDevice, st) != cudaSuccess) ||
        cudaMemcpyAsync(h.C, C_host, cb, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return KM_ERR_CUDA;
    km_status s = do_fit(h.X, dtype, w_host ? h.w : nullptr, B, N, K, d, h.C, iters,
                         ids_host ? h.ids : nullptr, (inertia_host && iters) ? h.inertia : nullptr,
                         nullptr, h.fit, st);
    if (s != KM_OK) return s;
    if (cudaMemcpyAsync(C_host, h.C, cb, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        (ids_host && cudaMemcpyAsync(ids_host, h.ids, static_cast<size_t>(B * N) * 4,
                                     cudaMemcpyDeviceToHost, st) != cudaSuccess) ||
        (inertia_host && iters &&
         cudaMemcpyAsync(inertia_host, h.inertia, static_cast<size_t>(iters) * B * 8,
                         cudaMemcpyDeviceToHost, st) != cudaSuccess))
        return KM_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? KM_OK : KM_ERR_CUDA;
}

km_status km_device_error(void *stream, int *code) {
    if (!code) return KM_ERR_INVALID_ARG;
    *code = 0;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return KM_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, km::g_km_dev_error, sizeof(v)) != cudaSuccess ||
        cudaMemcpyToSymbol(km::g_km_dev_error, &zero, sizeof(zero)) != cudaSuccess)
        return KM_ERR_CUDA;
    *code = static_cast<int>(v);
    return v ? KM_ERR_DEVICE_TIMEOUT : KM_OK;
}

km_status km_debug_wait_limit(unsigned long long limit_ns, unsigned long long *previous_ns) {
    if (limit_ns == 0) return KM_ERR_INVALID_ARG;
    unsigned long long old = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(&old, km::g_km_wait_limit_ns, sizeof(old)) != cudaSuccess ||
        cudaMemcpyToSymbol(km::g_km_wait_limit_ns, &limit_ns, sizeof(limit_ns)) != cudaSuccess)
        return KM_ERR_CUDA;
    if (previous_ns) *previous_ns = old;
    return KM_OK;
}

km_status km_debug_inject(int mode) {
    if (mode < 0 || mode > 2) return KM_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyToSymbol(km::g_km_inject, &mode, sizeof(mode)) != cudaSuccess)
        return KM_ERR_CUDA;
    return KM_OK;
}

}  // extern "C"

// =================================================================== allocation-free update
//
// Scratch for km_update_noalloc: one file-scope device array, present on every device that
// loads the library until the process exits. Host code must not hand the array's name to a
// kernel (on the host it only names a stand-in); its device address comes from
// cudaGetSymbolAddress, looked up with the device current once per context (normally once per
// device).
static __device__ __align__(256) uint8_t g_km_noalloc_scratch[KM_NOALLOC_SCRATCH_BYTES];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        tried = true;
    }
    return fn;
}

// Device address of the scratch array in the current context. The address belongs to the
// context the module was loaded in, so it is cached per (device, context) and looked up again
// when the current context changes (e.g. after cudaDeviceReset). The lookup happens with the
// device current and allocates nothing; a mutex covers first calls from several host threads.
void *noalloc_scratch_device_ptr() {
    static std::mutex mu;
    static CUcontext ctx_of[64] = {nullptr};
    static void *addr_of[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    CtxGetCurrentFn get = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    // null when the runtime has not yet made its context current on this thread
    if (get && get(&ctx) == CUDA_SUCCESS && ctx && addr_of[dev] && ctx_of[dev] == ctx)
        return addr_of[dev];
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_km_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    // the lookup made the device's context current: remember the address for that context
    ctx = nullptr;
    if (get && get(&ctx) == CUDA_SUCCESS && ctx) {
        ctx_of[dev] = ctx;
        addr_of[dev] = p;
    }
    return p;
}

}  // namespace

extern "C" {

size_t km_noalloc_scratch_needed(int64_t B, int64_t N, int64_t K, int64_t d) {
    if (!sizes_ok(B, N, K, d)) return 0;
    Carver c(nullptr);
    carve_update(c, B, N, K, d);
    return c.off;
}

km_status km_update_noalloc(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                            int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                            float *C_new, int32_t *counts, float *wsum, void *stream) {
    if (!X || !ids || !C_prev || !C_new || !counts || !valid_dtype(dtype) || !sizes_ok(B, N, K, d) ||
        !elem_aligned(X, dtype) || !aligned(ids, 4) || !aligned(counts, 4) || !aligned(C_prev, 4) ||
        !aligned(C_new, 4) || (w && !aligned(w, 4)) || (wsum && !aligned(wsum, 4)))
        return KM_ERR_INVALID_ARG;
    if (km_noalloc_scratch_needed(B, N, K, d) > KM_NOALLOC_SCRATCH_BYTES) return KM_ERR_WORKSPACE;
    void *scratch = noalloc_scratch_device_ptr();
    if (!scratch) return KM_ERR_CUDA;
    Carver r(scratch);
    UpdateWs u = carve_update(r, B, N, K, d);
    float *ws_w = wsum ? wsum : (w ? u.wsum : nullptr);
    // do_update_partial clears counts, sums and wsum first, so the previous call's contents of
    // the shared array never leak into this one.
    km_status s = do_update_partial(X, dtype, ids, w, B, N, K, d, u.sums, ws_w, counts, u, S(stream));
    if (s != KM_OK) return s;
    return finalize_dispatch(u.sums, w ? ws_w : nullptr, counts, C_prev, B * K, d, C_new, KM_F32,
                             nullptr, nullptr, S(stream));
}

}  // extern "C"
