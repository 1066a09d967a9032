// km_assign_simt.cuh -- exact-fp32 CUDA-core assignment (any dtype, any d).
//
// Used for fp32 inputs (no TF32 rounding of the points), for d that the tensor-core kernel does
// not take, and for misaligned pointers. Each thread owns one point; centroid tiles of 32 x 32
// and the matching point tile are staged in shared memory as fp32; the squared distance is
// accumulated in the direct form sum_j (x_j - c_j)^2, and a running (min, argmin) is kept in
// registers with the lowest index winning ties (FlashAssign's online argmin; technologypulse.uk
// Flash-KMeans article, "Bottleneck 1"; wispaper blog "1. FlashAssign"). No distance matrix is
// written.
#pragma once

#include "km_common.cuh"

namespace km {

constexpr int kSimtPts = 128;  // points per block
constexpr int kSimtKT = 32;    // centroids per tile
constexpr int kSimtDC = 32;    // coordinates per tile

template <typename T>
__global__ void __launch_bounds__(kSimtPts)
    assign_simt_kernel(const T *__restrict__ X, const T *__restrict__ Cx,
                       const float *__restrict__ w, int N, int K, int d, int32_t *__restrict__ ids,
                       float *__restrict__ mind, double *__restrict__ inertia,
                       int32_t *__restrict__ counts, int64_t xld) {
    __shared__ float xs[kSimtDC][kSimtPts + 1];
    __shared__ float cs[kSimtKT][kSimtDC];
    __shared__ double red[kSimtPts / 32];

    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kSimtPts;
    const int64_t i = i0 + tid;
    const bool valid = i < N;
    const T *Xb = X + static_cast<int64_t>(b) * xld * d;   // xld >= N rows per batch element
    const T *Cb = Cx + static_cast<int64_t>(b) * K * d;

    float best = INFINITY;
    int bi = 0;
    for (int k0 = 0; k0 < K; k0 += kSimtKT) {
        float acc[kSimtKT];
#pragma unroll
        for (int kk = 0; kk < kSimtKT; ++kk) acc[kk] = 0.f;
        for (int j0 = 0; j0 < d; j0 += kSimtDC) {
            __syncthreads();
            for (int e = tid; e < kSimtPts * kSimtDC; e += kSimtPts) {
                const int r = e / kSimtDC, c = e % kSimtDC;
                const int64_t ii = i0 + r;
                xs[c][r] = (ii < N && j0 + c < d) ? Cvt<T>::to_f(Xb[ii * d + j0 + c]) : 0.f;
            }
            for (int e = tid; e < kSimtKT * kSimtDC; e += kSimtPts) {
                const int r = e / kSimtDC, c = e % kSimtDC;
                cs[r][c] = (k0 + r < K && j0 + c < d)
                               ? Cvt<T>::to_f(Cb[static_cast<int64_t>(k0 + r) * d + j0 + c])
                               : 0.f;
            }
            __syncthreads();
            float xr[kSimtDC];
#pragma unroll
            for (int c = 0; c < kSimtDC; ++c) xr[c] = xs[c][tid];
#pragma unroll
            for (int kk = 0; kk < kSimtKT; ++kk) {
#pragma unroll
                for (int c = 0; c < kSimtDC; ++c) {
                    const float t = xr[c] - cs[kk][c];
                    acc[kk] = fmaf(t, t, acc[kk]);
                }
            }
        }
#pragma unroll
        for (int kk = 0; kk < kSimtKT; ++kk) {
            if (k0 + kk < K && acc[kk] < best) {
                best = acc[kk];
                bi = k0 + kk;
            }
        }
    }
    double contrib = 0.0;
    if (valid) {
        const int64_t gi = static_cast<int64_t>(b) * N + i;
        ids[gi] = bi;
        if (mind) mind[gi] = best;
        contrib = static_cast<double>(w ? w[static_cast<int64_t>(b) * xld + i] : 1.f) *
                  static_cast<double>(best);
    }
    if (counts && valid) atomicAdd(counts + static_cast<int64_t>(b) * K + bi, 1);   // histogram
    if (inertia) {
        contrib = warp_sum(contrib);
        if ((tid & 31) == 0) red[tid >> 5] = contrib;
        __syncthreads();
        if (tid == 0) {
            double s = 0.0;
            for (int k = 0; k < kSimtPts / 32; ++k) s += red[k];
            atomicAdd(inertia + b, s);
        }
    }
}

}  // namespace km
