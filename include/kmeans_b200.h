/*
 * kmeans_b200.h -- C ABI of libkmeans_b200.so: exact Lloyd k-means on NVIDIA B200 (sm_100a).
 *
 * One Lloyd iteration has two stages (technologypulse.uk "Flash-KMeans" article, section
 * "Flash-KMeans: same maths, new dataflow"; wispaper.ai Flash-KMeans blog, Background):
 *   assignment  ids[i] = argmin_k ||x_i - c_k||^2
 *   update      c_k    = (sum_{i: ids[i]=k} w_i x_i) / (sum_{i: ids[i]=k} w_i)
 * The assignment never materialises the N x K distance matrix (FlashAssign, same article,
 * "Bottleneck 1"; wispaper blog "1. FlashAssign"). The update sorts the assignment vector so
 * that each cluster's points form one contiguous segment and reduces segment by segment, with
 * one atomic merge per segment instead of one per point (Sort-Inverse Update, same article,
 * "Bottleneck 2"; wispaper blog "2. Sort-Inverse Update"). Per-point sample weights and the
 * uniform-grid initialisation linspace(min, max, K) come from the per-row 1-D codebook fitting
 * of the LeanQuant issue "1D k-means" (kmeans_fit with sample_weight).
 * Beyond one resident Lloyd iteration: an out-of-core fit that streams X from host memory
 * (km_fit_stream), e-means mini-batch training with moving averages and the proportional
 * splitting of dead clusters (km_emeans_fit, km_split_dead; steinslab e-means daily), and 1-D
 * codebook seeding and encoding (km_init_kmeanspp1d, km_encode1d).
 *
 * Conventions for every entry point:
 *   - Layout: row-major, innermost index last. X[B,N,d], C[B,K,d], w[B,N], ids[B,N],
 *     cn[B,K], counts[B,K]. B independent problems ("batches") share nothing.
 *   - Pointers are DEVICE pointers owned by the caller, except the host buffers of km_fit_host
 *     and km_fit_stream (see there). The library allocates no device memory: scratch comes from
 *     the caller's workspace, sized by km_workspace_size (km_stream_workspace_size,
 *     km_emeans_workspace_size). Nothing is retained between calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only enqueues work
 *     on that stream and returns; KM_OK means "validated and enqueued". km_fit_host is the one
 *     synchronous call.
 *   - Argument errors are reported synchronously, before anything is enqueued:
 *     KM_ERR_INVALID_ARG (null required pointer, a size <= 0, N or K >= 2^31, misaligned
 *     pointer), KM_ERR_UNSUPPORTED (dtype/shape combination not provided), KM_ERR_WORKSPACE
 *     (workspace smaller than km_workspace_size). A failed launch returns KM_ERR_CUDA.
 *   - Device-side waits in the kernels are bounded; a wait that runs out records an error word
 *     on the device and the kernel exits. km_device_error() reads and clears it.
 *   - Numerics: fp16/bf16/fp32 inputs, fp32 accumulation, fp32 master centroids. The
 *     assignment compares distances to the centroids rounded (round-to-nearest-even) to X's
 *     dtype, with ||c||^2 computed from the rounded values; ties go to the lowest index.
 *     Inputs containing NaN or Inf give undefined results.
 *   - Empty clusters (count 0 or total weight 0) keep their previous centroid.
 */
#ifndef KMEANS_B200_H
#define KMEANS_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum km_status {
    KM_OK = 0,
    KM_ERR_INVALID_ARG = 1,
    KM_ERR_UNSUPPORTED = 2,
    KM_ERR_WORKSPACE = 3,
    KM_ERR_CUDA = 4,
    KM_ERR_DEVICE_TIMEOUT = 5
} km_status;

typedef enum km_dtype { KM_F32 = 0, KM_F16 = 1, KM_BF16 = 2 } km_dtype;

typedef enum km_op { KM_OP_ASSIGN = 0, KM_OP_UPDATE = 1, KM_OP_FIT = 2, KM_OP_FIT_HOST = 3 } km_op;

/* Human-readable name of a status code (static string, never NULL). */
const char *km_status_string(km_status s);

/* ABI version of this library (incremented on any signature change). */
int km_abi_version(void);

/*
 * Bytes of device workspace the entry point `op` needs for these sizes (0 on invalid sizes, and
 * 0 for KM_OP_ASSIGN when the CUDA-core path needs none). `weighted` != 0 when a weight array
 * will be passed and `iters` the iteration count. Both matter for KM_OP_FIT_HOST only: that
 * workspace also holds the device copies of the caller's host buffers, i.e. the weights
 * (B*N fp32, only when weighted) and the inertia history (iters*B fp64); the other ops keep
 * those in caller memory, so there they are ignored.
 * The workspace must be 256-byte aligned; its contents need not be initialised.
 */
size_t km_workspace_size(km_op op, int64_t B, int64_t N, int64_t K, int64_t d, km_dtype dtype,
                         int weighted, int iters);

/*
 * Centroid preparation for the assignment: Cx[b,k,:] = C[b,k,:] rounded to `dtype` (RNE), and
 * cn[b,k] = sum_j Cx[b,k,j]^2 in fp32 from the rounded values (the ||c||^2 term of the expanded
 * distance ||x||^2 - 2<x,c> + ||c||^2 used by FlashAssign; technologypulse.uk Flash-KMeans
 * article, "Bottleneck 1"). C[B,K,d] fp32 in; Cx[B,K,d] in `dtype`, cn[B,K] fp32 out.
 */
km_status km_prep(const float *C, km_dtype dtype, int64_t B, int64_t K, int64_t d, void *Cx,
                  float *cn, void *stream);

/*
 * Assignment stage (FlashAssign): ids[b,i] = argmin_k ||X[b,i,:] - Cx[b,k,:]||^2, lowest k on
 * ties, computed tile by tile with a running (min, argmin) per point so that no N x K matrix is
 * written (technologypulse.uk Flash-KMeans article, "Bottleneck 1"; wispaper blog
 * "1. FlashAssign", online argmin).
 *   X[B,N,d] in `dtype`; Cx[B,K,d] in the same dtype (see km_prep);
 *   cn[B,K] fp32 = ||Cx[b,k]||^2, or NULL (then computed into the workspace);
 *   w[B,N] fp32 per-point weights for the inertia, or NULL (all ones);
 *   ids[B,N] int32 out (required); mind[B,N] fp32 out or NULL: the squared distance to the
 *   chosen centroid, max(0, .); inertia[B] fp64 out or NULL: sum_i w_i * mind_i;
 *   counts[B,K] int32 out or NULL: the number of points assigned to each cluster (the
 *   histogram the Sort-Inverse Update starts from; written by the kernel that writes the ids,
 *   one atomic per distinct cluster per warp, so the update need not read the ids for it).
 * fp16/bf16 with d % 8 == 0, 8 <= d <= 256 and 16-byte aligned X/Cx run on the tcgen05 tensor
 * cores (fp32 accumulation of <x,c>); every other case runs an exact-fp32 CUDA-core kernel that
 * evaluates sum_j (x_j - c_j)^2 directly. On the tensor-core path mind is formed as
 * ||x||^2 + (||c||^2 - 2<x,c>) in fp32, so its absolute error is a small multiple of
 * 2^-24 (||x||^2 + ||c||^2); for points almost on their centroid that can exceed 1e-4 of the
 * distance itself (the assignment is unaffected except at near-ties). The tensor-core path also
 * compares distances as packed (value, index) keys whose lowest 4-6 mantissa bits hold the
 * column: distances closer than 2^-17 relative are resolved by index, and the reported mind is
 * truncated by less than 2^-17 relative.
 */
km_status km_assign(const void *X, km_dtype dtype, const void *Cx, const float *cn,
                    const float *w, int64_t B, int64_t N, int64_t K, int64_t d, int32_t *ids,
                    float *mind, double *inertia, int32_t *counts, void *ws, size_t ws_bytes,
                    void *stream);

/*
 * 1 when km_assign with these arguments runs on the tcgen05 tensor cores, 0 when it runs the
 * exact-fp32 CUDA-core kernel (no launch, no validation beyond the eligibility rule).
 */
int km_assign_uses_tensor_cores(km_dtype dtype, int64_t d, const void *X, const void *Cx);

/*
 * Update stage (Sort-Inverse Update), fed an assignment ids[B,N] (values in [0,K)):
 *   counts[b,k] = #{i : ids[b,i] = k}                                        (int32, required)
 *   wsum[b,k]   = sum of w over those points (fp32; NULL allowed)
 *   C_new[b,k]  = sum_i w_i X[b,i,:] / wsum[b,k], or C_prev[b,k] when the cluster is empty.
 * The ids are argsorted per batch by a device counting sort into contiguous per-cluster
 * segments; X is read in sorted order by index (never permuted in memory) and each range of
 * sorted positions reduces its runs on chip (technologypulse.uk Flash-KMeans article,
 * "Bottleneck 2"; wispaper blog "2. Sort-Inverse Update"). For d = 32 * V with rows of 128, 256
 * or 512 bytes and a 16-byte aligned X, rows are gathered four at a time by the tensor-memory
 * engine and the divide is fused into the reduction: a run that is a whole cluster is divided
 * where it was summed, a cluster split over ranges combines its per-range partials in range
 * order (one merge per segment, no atomics on the sums). Other shapes merge each run into a
 * sums array with one vector atomic per coordinate block and divide in a second kernel.
 * C_new may alias C_prev. Points whose id lies outside [0,K) are ignored (neither counted nor
 * summed). Workspace: km_workspace_size(KM_OP_UPDATE, ...) bytes.
 */
km_status km_update(const void *X, km_dtype dtype, const int32_t *ids, const float *w, int64_t B,
                    int64_t N, int64_t K, int64_t d, const float *C_prev, float *C_new,
                    int32_t *counts, float *wsum, void *ws, size_t ws_bytes, void *stream);

/*
 * km_update followed by km_prep of the new centroids, in the same pass: besides C_new, counts
 * and wsum (as km_update) it writes Cx[B,K,d] = C_new rounded to X's dtype and cn[B,K] =
 * ||Cx||^2 (fp32), the inputs of the next km_assign. This is the update of one Lloyd iteration
 * as km_fit runs it. Cx and cn are required; C_new may alias C_prev. Same workspace as
 * km_update. counts_ready != 0 says that counts already holds the histogram of ids (as
 * km_assign writes it) and the histogram pass is skipped; otherwise counts is written here.
 */
km_status km_update_next(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                         int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                         float *C_new, void *Cx, float *cn, int32_t *counts, int counts_ready,
                         float *wsum, void *ws, size_t ws_bytes, void *stream);

/*
 * First half of km_update, for callers that combine partial sums across devices (points
 * split over GPUs, centroids replicated): writes this device's sums[B,K,d] (fp32,
 * sum_i w_i x_i), wsum[B,K] (fp32, may be NULL when w is NULL) and counts[B,K] (int32), all
 * overwritten (not accumulated). Same sort-inverse reduction as km_update. Uses the
 * KM_OP_UPDATE workspace.
 */
km_status km_update_partial(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                            int64_t B, int64_t N, int64_t K, int64_t d, float *sums, float *wsum,
                            int32_t *counts, void *ws, size_t ws_bytes, void *stream);

/*
 * Second half of km_update: C_new[b,k] = sums[b,k] / wsum[b,k] (wsum NULL: counts) when
 * counts[b,k] > 0 and the divisor is > 0, else C_prev[b,k] (the mean S_j / N_j of the e-means
 * daily's Lloyd recap, steinslab, first section). Optionally also writes Cx (C_new rounded to
 * `cx_dtype`) and cn = ||Cx||^2 for the next assignment (pass NULL to skip). C_new may alias
 * C_prev.
 */
km_status km_finalize(const float *sums, const float *wsum, const int32_t *counts,
                      const float *C_prev, int64_t B, int64_t K, int64_t d, float *C_new,
                      km_dtype cx_dtype, void *Cx, float *cn, void *stream);

/*
 * Uniform-grid initialisation of 1-D rows (LeanQuant issue "1D k-means": the sklearn init
 * np.linspace(row.min(), row.max(), K)): with lo/hi the min/max of X[b,:,0],
 * C[b,k] = k * ((hi - lo) / (K - 1)) + lo evaluated in fp64 exactly as numpy's linspace does,
 * C[b,K-1] = hi, K == 1 gives lo; then rounded to fp32. X[B,N,1] in `dtype`, C[B,K] fp32 out.
 */
km_status km_init_grid1d(const void *X, km_dtype dtype, int64_t B, int64_t N, int64_t K, float *C,
                         void *stream);

/*
 * `iters` Lloyd iterations from the centroids in C[B,K,d] (fp32, in/out), then (only when ids is
 * non-NULL) one final assignment against the final centroids written to ids[B,N].
 *   inertia_hist[iters,B] fp64 out or NULL: inertia of iteration t's assignment;
 *   C_hist[iters+1,B,K,d] fp32 out or NULL: the centroids entering each iteration and the final
 *   ones (C_hist[0] = the input C).
 * d == 1 with N <= 8192 (the per-row codebook setting of the LeanQuant issue): for K <= 32 one
 * kernel sorts every row once and stores the sorted values, indices and fp64 prefix sums of w,
 * w*x, w*x^2 in the workspace (32 bytes per point), then one kernel runs all iterations with a
 * warp per row; for 32 < K <= 64 one fused kernel per row keeps the row on chip (no workspace
 * needed). Small problems (K * d <= 4096, d <= 64, B * ceil(N / 64) <= 2048 CTAs that can all
 * be resident, B * N * K * d <= 2^27, iters > 0) run the whole fit in one cooperative launch:
 * each CTA keeps 64 points in registers (four threads per point) and assigns them with the same
 * fp32 direct-form arithmetic as the CUDA-core assignment; each CTA adds its per-cluster partial
 * sums into the iteration's totals with atomics, and a grid barrier whose waits are bounded like
 * every other wait of the library separates the iterations. Everything else
 * chains km_prep / km_assign / km_update on the stream. `ws` must hold
 * km_workspace_size(KM_OP_FIT, ...) bytes (else KM_ERR_WORKSPACE).
 */
km_status km_fit(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N, int64_t K,
                 int64_t d, float *C, int iters, int32_t *ids, double *inertia_hist,
                 float *C_hist, void *ws, size_t ws_bytes, void *stream);

/*
 * km_fit on HOST buffers: copies X_host (and w_host, C_host) to the device staging area inside
 * the workspace (one cudaMemcpyAsync per array), runs km_fit, copies C back into C_host and,
 * when non-NULL, ids into ids_host[B,N] and the inertia history into inertia_host[iters,B],
 * then synchronises `stream`. Host buffers should be pinned for full PCIe bandwidth. The
 * workspace (device memory) is sized by km_workspace_size(KM_OP_FIT_HOST, ..., weighted, iters).
 * With iters == 1, ids_host NULL and X of 64 MiB or more, X is needed only once: the call then
 * streams X in 16 chunks of points (each a slice of every problem, as km_fit_stream does),
 * with its buffers inside the X staging area, so the copy of one chunk overlaps the assignment
 * and accumulation of the previous one. The labels are the same
 * as km_fit's; the sums are accumulated chunk by chunk, so C and the inertia match km_fit's to
 * fp32 (fp64 for the inertia) rounding, not bit for bit.
 */
km_status km_fit_host(const void *X_host, km_dtype dtype, const float *w_host, int64_t B,
                      int64_t N, int64_t K, int64_t d, float *C_host, int iters, int32_t *ids_host,
                      double *inertia_host, void *ws, size_t ws_bytes, void *stream);

/* Out-of-core exact Lloyd (technologypulse.uk Flash-KMeans article, the out-of-core line of the
 * measurements and the chunked stream overlap that hides PCIe transfers; wispaper blog
 * "Performance", the scalability point): points that do not fit in device memory stay in
 * host memory and are streamed through the GPU every iteration in chunks; each chunk is
 * assigned as it arrives and its per-cluster sums and counts are accumulated, so the result is
 * the exact Lloyd iteration of the whole set (up to fp32 summation order).
 *   X_host[B,N,d] in host memory (pinned memory lets the copies overlap the kernels; pageable
 *   memory works but the copies then block the calling thread), w_host[B,N] or NULL;
 *   C[B,K,d] fp32 DEVICE memory: initial centroids in, final centroids out;
 *   iters >= 0; chunk >= 1 points per batch element per copy (clamped to N);
 *   inertia_hist[iters,B] fp64 DEVICE memory or NULL: the objective of each iteration's
 *   assignment. Two device buffers of `chunk` points per batch element; copies run on a stream
 *   the call creates and releases, ordered after the work already enqueued on `stream`.
 *   Asynchronous on `stream` like km_fit; X_host and w_host must stay valid and unchanged until
 *   the stream has completed the call's work.
 * Errors: KM_ERR_INVALID_ARG (null pointers, sizes, chunk < 1, misaligned), KM_ERR_WORKSPACE
 * (ws smaller than km_stream_workspace_size), KM_ERR_CUDA.
 */
size_t km_stream_workspace_size(int64_t B, int64_t K, int64_t d, km_dtype dtype, int weighted,
                                int64_t chunk);
km_status km_fit_stream(const void *X_host, km_dtype dtype, const float *w_host, int64_t B,
                        int64_t N, int64_t K, int64_t d, float *C, int iters, int64_t chunk,
                        double *inertia_hist, void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the current device.
 * *code = 0 when no kernel recorded an error; otherwise a bit mask (1 = a bounded wait ran out).
 * Returns KM_ERR_DEVICE_TIMEOUT when *code != 0, KM_ERR_CUDA when the synchronisation failed.
 */
km_status km_device_error(void *stream, int *code);

/*
 * Test hooks for the failure path (no page text has a counterpart). Every wait inside the
 * kernels is bounded; km_debug_wait_limit sets that bound for the current device (default 4 s;
 * *previous_ns receives the old value when non-NULL) so a test can make a wait run out quickly.
 * km_debug_inject(1) makes the next tensor-core assignments withhold the first point tile of the
 * first SM pair: the waits on it run out, every role of that pair leaves its loop, copies in
 * flight land, the issued MMAs drain, tensor memory is freed and the kernel returns with bit 0
 * of the device error word set (km_device_error reports KM_ERR_DEVICE_TIMEOUT); its labels
 * are left unwritten. km_debug_inject(2) makes the first CTA of the next single-launch small fits
 * (km_fit on shapes with K * d <= 4096, d <= 64 and at most 2048 CTAs of 256 points) skip its
 * first grid-barrier arrival: the other CTAs' waits run out, set bit 0 and an abort word, and
 * every CTA leaves. km_debug_inject(0) (the default) turns both off. Both calls synchronise the
 * device first. No fault, trap or endless loop is involved.
 */
km_status km_debug_wait_limit(unsigned long long limit_ns, unsigned long long *previous_ns);
km_status km_debug_inject(int mode);

/*
 * km_update for callers that cannot allocate device memory: the same computation and outputs
 * as km_update, but the scratch (offsets, cursors, permutation, partial sums) lives in one
 * array of the library itself, KM_NOALLOC_SCRATCH_BYTES (32 MiB) per device. No page text has a
 * counterpart: this is an interface convenience, not part of the method.
 * Meant for code that must not call cudaMalloc/cudaFree at that point (the allocation calls
 * can synchronise the device and stall other streams, and some embeddings hand the library no
 * allocator at all), so there is no workspace to pass.
 *   - The array is reserved when the library's CUDA module is first loaded in a context on a
 *     device, i.e. at the first call of ANY entry point of this library there (CUDA loads
 *     modules lazily), and it is held until the context is destroyed (normally process exit).
 *     Callers that never use km_update_noalloc pay for it too.
 *   - Sizes whose scratch exceeds the array (see km_noalloc_scratch_needed) are rejected with
 *     KM_ERR_WORKSPACE before anything is enqueued.
 *   - The array's device address is looked up with cudaGetSymbolAddress on the first call in
 *     each context (normally once per device, with that device current) and cached per context;
 *     after cudaDeviceReset the next call looks it up again in the new context. Make the first
 *     call on a device before any stream capture.
 *   - Every call uses the same array and it keeps the last call's contents (each call clears
 *     what must start at zero): calls that can overlap on the GPU (different streams, or
 *     several host threads) race with each other and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define KM_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
km_status km_update_noalloc(const void *X, km_dtype dtype, const int32_t *ids, const float *w,
                            int64_t B, int64_t N, int64_t K, int64_t d, const float *C_prev,
                            float *C_new, int32_t *counts, float *wsum, void *stream);

/* Bytes of the static scratch km_update_noalloc needs for these sizes (0 on invalid sizes). */
size_t km_noalloc_scratch_needed(int64_t B, int64_t N, int64_t K, int64_t d);

/*
 * e-means: mini-batch k-means with moving averages (steinslab daily "Beating 25 Lloyd
 * Iterations in 2 Epochs", sections "Breaking 70 Years of Full-Batch Inertia...", "Mini-Batch
 * Stochastic Noise Escapes Local Optima", "Matching 25 Iterations of Error in Just 2 Epochs" and
 * "Proportional Splitting Resurrects Thousands of Dead Centers").
 * Each problem's points are visited `epochs` times in consecutive mini-batches of `batch` points
 * (in the order given; shuffle beforehand). Every mini-batch is assigned against the current
 * centroids (the same exact argmin as km_assign), its per-cluster sums s and sizes n (counts, or
 * weight sums) enter the state
 *     S <- (1 - a_t) S + a_t s,   N <- (1 - a_t) N + a_t n,   C = S / N (kept where N == 0),
 * with S = C, N = 1 at the start and a_t = alpha0 (0.1 + 0.9 (1 + cos(pi t / T)) / 2) at step t
 * of T = epochs * ceil(N_points / batch). Between epochs, when split_u is given, every cluster
 * that received no point during the epoch is revived as in km_split_dead (sizes = the epoch's
 * counts or weight sums, uniforms split_u[epoch][B][K]). After the last epoch C moves to the
 * mean of the points that epoch assigned to each cluster (clusters it left empty keep theirs).
 *   X[B,N,d] in `dtype`, w[B,N] fp32 or NULL, C[B,K,d] fp32 in/out (device);
 *   split_u: NULL (no splitting) or [epochs,B,K] fp32 uniforms in [0,1) (device);
 *   sse_hist: NULL or [epochs,B] fp64 out: per epoch, the sum of w * squared distance of every
 *   point to the centroid it was assigned to when its mini-batch was processed;
 *   ws: km_emeans_workspace_size(B, K, d, dtype, weighted, batch) bytes (device, 256-B aligned).
 * Asynchronous on `stream`. Errors: KM_ERR_INVALID_ARG (null X or C, sizes, batch < 1,
 * alpha0 outside (0,1], split_eps outside [0,1), misaligned), KM_ERR_WORKSPACE, KM_ERR_CUDA.
 */
size_t km_emeans_workspace_size(int64_t B, int64_t K, int64_t d, km_dtype dtype, int weighted,
                                int64_t batch);
km_status km_emeans_fit(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N,
                        int64_t K, int64_t d, float *C, int64_t batch, int epochs, float alpha0,
                        const float *split_u, float split_eps, double *sse_hist, void *ws,
                        size_t ws_bytes, void *stream);

/*
 * Proportional splitting of dead clusters (steinslab e-means daily, section "Proportional
 * Splitting Resurrects Thousands of Dead Centers"; usable after a Lloyd update with sizes = the
 * update's counts). Per problem, the clusters with sizes == 0 are revived in index order: dead
 * cluster i takes as donor the first cluster j whose running size sum exceeds u[i] * (total
 * size) (fp64), then per coordinate k (s_k = +1 for even k, -1 for odd k)
 *     C[i][k] = C[j][k] (1 + eps s_k),   C[j][k] <- C[j][k] (1 - eps s_k),
 * sizes[i] = sizes[j] / 2, sizes[j] -= sizes[i]; when given, Nc is halved the same way and
 * S_sums[i], S_sums[j] = C * Nc. Nothing happens when every size is 0.
 *   C[B,K,d], sizes[B,K], u[B,K] fp32; Nc[B,K], S_sums[B,K,d] fp32 or NULL; donors[B,K] int32
 *   out or NULL (donor of each revived cluster, -1 elsewhere). All device memory.
 * Asynchronous on `stream`. One block of 1024 threads per problem; each revival rescans the K
 * sizes. Errors: KM_ERR_INVALID_ARG (null C/sizes/u, sizes, eps outside [0,1), misaligned),
 * KM_ERR_CUDA.
 */
km_status km_split_dead(float *C, float *sizes, const float *u, float eps, int64_t B, int64_t K,
                        int64_t d, float *Nc, float *S_sums, int32_t *donors, void *stream);

/*
 * 1-D codebook encoding (the weight-clustering proposal reposted on wpnews.pro, "Cache-Aware
 * Weight Clustering ...": values stored as 8-bit indices of shared cluster values). Each value
 * X[b,i] becomes the index of its nearest centroid C[b,k] (centroids rounded to `dtype`, fp32
 * squared distance, lowest index on ties: the same decision as km_assign with d = 1), found by
 * binary search in the per-row sorted codebook. Unlike the other calls, infinite values are
 * defined here: every centroid is then at infinite distance, so the value gets index 0 (NaN
 * values still get an unspecified index below K). Rows of N a multiple of 16 with X and codes
 * 16-byte aligned are read and written with 16-byte vector accesses.
 *   X[B,N] in `dtype`, C[B,K] fp32 (any order), codes[B,N] uint8 out; all device memory.
 * K <= 256. Asynchronous on `stream`. Errors: KM_ERR_INVALID_ARG, KM_ERR_CUDA.
 */
km_status km_encode1d(const void *X, km_dtype dtype, int64_t B, int64_t N, const float *C,
                      int64_t K, uint8_t *codes, void *stream);

/*
 * k-means++ seeding of per-row 1-D codebooks (the LeanQuant issue "1D k-means": rows with more
 * than 8 clusters are seeded by k-means++). Per row, centre 0 is drawn with probability
 * proportional to w, every next one proportional to w * (squared distance to the nearest centre
 * so far), distances and masses in fp64; draw k takes the first point whose running mass exceeds
 * u[b,k] * (total mass), point 0 when no mass is left.
 *   X[B,N] in `dtype`, w[B,N] fp32 or NULL (unit weights), u[B,K] fp32 uniforms in [0,1),
 *   C[B,K] fp32 out (the chosen values), chosen[B,K] int32 out or NULL (their indices).
 * N <= 8192 (else KM_ERR_UNSUPPORTED). One block per row. Asynchronous on `stream`.
 * Errors: KM_ERR_INVALID_ARG, KM_ERR_UNSUPPORTED, KM_ERR_CUDA.
 */
km_status km_init_kmeanspp1d(const void *X, km_dtype dtype, const float *w, int64_t B, int64_t N,
                             int64_t K, const float *u, float *C, int32_t *chosen, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KMEANS_B200_H */
