// The moment check that picks the number of composed passes (the RHT-composition results
// quoted with the HARP pages: a linear-time check on the input's moments adapts at run time
// how many randomized Hadamard passes are applied; the page gives neither the statistic nor
// its thresholds).  Reading: per row, m2 = sum x^2, m3 = sum |x|^3, m4 = sum x^4, the
// peakedness kappa = m4 / m2^2 (1/d for a flat row, 1 for a one-hot row) and the passes: 1 if
// kappa <= tau1, 2 if kappa <= tau2, else 3.  One warp per row, 16-byte loads, double sums;
// a single pass over the rows in HBM.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void add_moments(float v, double& m2, double& m3, double& m4) {
    const double a = fabs((double)v);
    const double a2 = a * a;
    m2 += a2;
    m3 += a2 * a;
    m4 += a2 * a2;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void load8v(const float* p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
__device__ __forceinline__ void load8v(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        v[2 * q] = __uint_as_float(w[q] << 16);
        v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
    }
}
__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void __launch_bounds__(kThreads) moment_check_kernel(const T* __restrict__ x, int64_t rows, int64_t d,
                                                                int64_t ld, bool vec, double tau1, double tau2,
                                                                double* moments, int32_t* passes) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* row = x + r * ld;
        double m2 = 0.0, m3 = 0.0, m4 = 0.0;
        if (vec) {
            for (int64_t j = 8 * (int64_t)lane; j < d; j += 256) {
                float v[8];
                load8v(row + j, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) add_moments(v[e], m2, m3, m4);
            }
        } else {
            for (int64_t j = lane; j < d; j += 32) add_moments(load1(row + j), m2, m3, m4);
        }
        m2 = warp_sum(m2);
        m3 = warp_sum(m3);
        m4 = warp_sum(m4);
        if (lane == 0) {
            if (moments) {
                moments[3 * r] = m2;
                moments[3 * r + 1] = m3;
                moments[3 * r + 2] = m4;
            }
            if (passes) {
                const double kappa = m2 > 0.0 ? m4 / (m2 * m2) : 0.0;
                passes[r] = kappa <= tau1 ? 1 : kappa <= tau2 ? 2 : 3;
            }
        }
    }
}

}  // namespace

extern "C" harp_status harp_moment_check(const void* x, int64_t rows, int64_t d, int64_t ld, harp_dtype dtype,
                                         double tau1, double tau2, double* moments, int32_t* passes,
                                         void* stream_) {
    harp_clear_error();
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (rows < 0 || d <= 0) return harp_fail(HARP_ERR_INVALID_ARG, "rows >= 0 and d > 0");
    if (ld < d) return harp_fail(HARP_ERR_INVALID_ARG, "ld smaller than d");
    if (!(tau1 <= tau2)) return harp_fail(HARP_ERR_INVALID_ARG, "tau1 must not exceed tau2");
    if (rows == 0) return HARP_OK;
    if (!x || (!moments && !passes)) return harp_fail(HARP_ERR_INVALID_ARG, "x is NULL or no output given");
    const size_t es = dtype == HARP_F32 ? 4 : 2;
    const size_t xb = ((size_t)(rows - 1) * ld + d) * es;
    if ((moments && ranges_overlap(x, xb, moments, (size_t)rows * 3 * sizeof(double))) ||
        (passes && ranges_overlap(x, xb, passes, (size_t)rows * sizeof(int32_t))) ||
        (moments && passes &&
         ranges_overlap(moments, (size_t)rows * 3 * sizeof(double), passes, (size_t)rows * sizeof(int32_t))))
        return harp_fail(HARP_ERR_INVALID_ARG, "outputs overlap x or each other");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        sms = 148;
    }
    const bool vec = ((uintptr_t)x % 16 == 0) && (ld * es) % 16 == 0 && d % 8 == 0;
    const int64_t blocks = (rows + kThreads / 32 - 1) / (kThreads / 32);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(blocks, 16 * (int64_t)sms));
    cudaStream_t stream = (cudaStream_t)stream_;
    if (dtype == HARP_F32)
        moment_check_kernel<float><<<grid, kThreads, 0, stream>>>((const float*)x, rows, d, ld, vec, tau1, tau2,
                                                                 moments, passes);
    else
        moment_check_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>((const __nv_bfloat16*)x, rows, d, ld, vec,
                                                                         tau1, tau2, moments, passes);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("moment_check_kernel");
    return HARP_OK;
}
