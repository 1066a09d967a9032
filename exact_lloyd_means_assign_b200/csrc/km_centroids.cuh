// km_centroids.cuh -- per-centroid kernels: preparation for the assignment and the final divide.
//
// prep:     Cx = C rounded to the points' dtype, cn = ||Cx||^2 (fp32), one warp per centroid.
// finalize: C_new = sums / wsum for non-empty clusters, else C_prev (the mean S_j / N_j of the
//           Lloyd recap in the steinslab e-means daily); optionally also Cx and cn for the next
//           assignment, so a multi-iteration fit never runs prep twice.
// caug:     the extra reduction step the tensor-core assignment appends to every centroid tile:
//           per centroid 16 bf16 values [1, a, b, c, 0...] with a + b + c = ||c||^2 / 2 (a
//           three-piece bf16 split, exact to about 2^-27 relative), padded to whole tiles with
//           [0, 1e30, 0...] rows so padding columns can never win the argmin.
#pragma once

#include "km_common.cuh"

namespace km {

template <typename T>
__global__ void prep_kernel(const float *__restrict__ C, int64_t rows, int d, T *__restrict__ Cx,
                            float *__restrict__ cn) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float *c = C + row * d;
    float s = 0.f;
    for (int j = lane; j < d; j += 32) {
        const T v = Cvt<T>::from_f(c[j]);
        if (Cx) Cx[row * d + j] = v;
        const float f = Cvt<T>::to_f(v);
        s = fmaf(f, f, s);
    }
    s = warp_sum(s);
    if (lane == 0 && cn) cn[row] = s;
}

// C_prev and C_new may alias (each element is read and then written by the same thread).
template <typename T>
__global__ void finalize_kernel(const float *__restrict__ sums, const float *__restrict__ wsum,
                                const int32_t *__restrict__ counts, const float *C_prev,
                                int64_t rows, int d, float *C_new, T *__restrict__ Cx,
                                float *__restrict__ cn) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int cnt = counts[row];
    const float div = wsum ? wsum[row] : static_cast<float>(cnt);
    const bool upd = cnt > 0 && div > 0.f;
    float s = 0.f;
    for (int j = lane; j < d; j += 32) {
        const int64_t e = row * d + j;
        const float v = upd ? sums[e] / div : C_prev[e];
        C_new[e] = v;
        if (Cx) {
            const T t = Cvt<T>::from_f(v);
            Cx[e] = t;
            const float f = Cvt<T>::to_f(t);
            s = fmaf(f, f, s);
        }
    }
    if (cn) {
        s = warp_sum(s);
        if (lane == 0) cn[row] = s;
    }
}

// caug[b, k, 0..15] (bf16) for k < Kp, one warp per (b, k). ||Cx[b,k]||^2 comes from `cn` when
// given, else it is computed from Cx.
template <typename T>
__global__ void caug_kernel(const T *__restrict__ Cx, const float *__restrict__ cn, int B, int K,
                            int Kp, int d, __nv_bfloat16 *__restrict__ caug) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= static_cast<int64_t>(B) * Kp) return;
    const int b = static_cast<int>(row / Kp), k = static_cast<int>(row % Kp);
    float v = 0.f;
    if (k < K) {
        if (cn) {
            v = cn[static_cast<int64_t>(b) * K + k];
        } else {
            const T *c = Cx + (static_cast<int64_t>(b) * K + k) * d;
            float s = 0.f;
            for (int j = lane; j < d; j += 32) {
                const float f = Cvt<T>::to_f(c[j]);
                s = fmaf(f, f, s);
            }
            v = warp_sum(s);
        }
    }
    // Row layout [1, 1, a, b, c, 0 x 11]: the point side is [x1, x2, 1, 1, 1, 0 x 11], so the
    // extra reduction step adds x1 + x2 + a + b + c = ||x||^2/2 (split) + ||c||^2/2.
    if (lane < 16) {
        float e = 0.f;
        if (k >= K) {
            e = (lane == 2) ? 1e30f : 0.f;
        } else {
            const float h = 0.5f * v;
            const float a = __bfloat162float(__float2bfloat16_rn(h));
            const float r1 = h - a;
            const float b2 = __bfloat162float(__float2bfloat16_rn(r1));
            const float c3 = r1 - b2;
            e = lane < 2 ? 1.f : lane == 2 ? a : lane == 3 ? b2 : lane == 4 ? c3 : 0.f;
        }
        caug[row * 16 + lane] = __float2bfloat16_rn(e);
    }
}

// The same rows from given norms, one thread per row (two 16-byte stores): the warp-per-row form
// above is only needed when the norms must be summed from Cx.
// It also clears the assignment's per-cluster counts and per-problem objective when given (the
// assignment that follows adds into them), saving two memset launches per assignment.
__global__ void caug_rows_kernel(const float *__restrict__ cn, int B, int K, int Kp,
                                 __nv_bfloat16 *__restrict__ caug, int32_t *__restrict__ zero_counts,
                                 double *__restrict__ zero_inertia) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (row >= static_cast<int64_t>(B) * Kp) return;
    const int b = static_cast<int>(row / Kp), k = static_cast<int>(row % Kp);
    if (zero_counts && k < K) zero_counts[static_cast<int64_t>(b) * K + k] = 0;
    if (zero_inertia && row < B) zero_inertia[row] = 0.0;
    __nv_bfloat16 e[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) e[j] = __float2bfloat16_rn(0.f);
    if (k >= K) {
        e[2] = __float2bfloat16_rn(1e30f);   // a padding column can never win
    } else {
        const float h = 0.5f * cn[static_cast<int64_t>(b) * K + k];
        const float a = __bfloat162float(__float2bfloat16_rn(h));
        const float r1 = h - a;
        const float b2 = __bfloat162float(__float2bfloat16_rn(r1));
        e[0] = e[1] = __float2bfloat16_rn(1.f);
        e[2] = __float2bfloat16_rn(a);
        e[3] = __float2bfloat16_rn(b2);
        e[4] = __float2bfloat16_rn(r1 - b2);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(caug + row * 16);
    dst[0] = *reinterpret_cast<const uint4 *>(&e[0]);
    dst[1] = *reinterpret_cast<const uint4 *>(&e[8]);
}

}  // namespace km
