// The fit's two evaluation terms on a Hessian proxy (HARP technical summary §2.3
// Optimization Objective: L_fit = L_diag + lambda_bd R_bd(Theta_V), described in words).
// Readings, the same as the oracle's:
//  * H' = T_V^T H T_V is the input-side Hessian proxy in the rotated basis (inputs rotate as
//    x' = T_V^T x); it is harp_apply_two_sided(planV, planV, H), so no kernel here.
//  * R_bd = the energy of H' outside its q x q diagonal blocks over its total energy:
//    harp_off_block_energy returns both sums.
//  * L_diag = sum_j H'_jj sum_r (W'_rj - Q(W')_rj)^2, W' = T_U^T W T_V the rotated weight and
//    Q the blockwise round-to-nearest int8 quantizer along its rows (scale = max|w| / 127 per
//    aligned block of qblock columns): harp_l_diag.
// Both are single passes over a matrix in HBM (4 or 2 bytes per element read, nothing
// written but two doubles), so the kernels are sized for bandwidth: 16-byte loads, a grid of
// a few CTAs per SM, double accumulators per thread, one atomic add per CTA.  The quantizer's
// decisions are taken in double, in the same operations as the float64 definition (s = a /
// 127, q = rint(w / s), target = q s), so its codes are the same as the definition's.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// 4 consecutive elements of a 16-byte-aligned row as float (fp32: one float4; bf16: 8 bytes)
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(a.x << 16), v[1] = __uint_as_float(a.x & 0xffff0000u);
    v[2] = __uint_as_float(a.y << 16), v[3] = __uint_as_float(a.y & 0xffff0000u);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sums of a CTA's per-thread values added to out[0..N): warp sums, then warp 0.
template <int N>
__device__ __forceinline__ void cta_add(const double (&v)[N], double* out) {
    __shared__ double part[kThreads / 32][N];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const double s = warp_sum(v[k]);
        if (lane == 0) part[warp][k] = s;
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int k = 0; k < N; ++k) {
            double s = lane < kThreads / 32 ? part[lane][k] : 0.0;
            s = warp_sum(s);
            if (lane == 0) atomicAdd(out + k, s);
        }
    }
}

// out[0] += sum of h_ij^2 over i / q != j / q, out[1] += sum of all h_ij^2.  Row i's columns
// split into the diagonal block [q (i / q), q (i / q) + q) and the rest, so the test is per
// run of four columns only where a run straddles the block's edges (q is a multiple of 4
// whenever the vector path is taken).
template <typename T>
__global__ void __launch_bounds__(kThreads) off_block_energy_kernel(const T* __restrict__ h, int64_t n,
                                                                    int64_t ld, int q, bool vec, double* out) {
    double off = 0.0, tot = 0.0;
    for (int64_t i = blockIdx.x; i < n; i += gridDim.x) {
        const T* row = h + i * ld;
        const int64_t b0 = (i / q) * q, b1 = b0 + q;   // the diagonal block's columns
        if (vec) {
            for (int64_t j = 4 * (int64_t)threadIdx.x; j < n; j += 4 * kThreads) {
                float v[4];
                load4(row + j, v);
                double s = 0.0;
#pragma unroll
                for (int e = 0; e < 4; ++e) s += (double)v[e] * (double)v[e];
                tot += s;
                if (j < b0 || j >= b1) off += s;
            }
        } else {
            for (int64_t j = threadIdx.x; j < n; j += kThreads) {
                const double v = (double)load1(row + j);
                const double s = v * v;
                tot += s;
                if (j < b0 || j >= b1) off += s;
            }
        }
    }
    const double v[2] = {off, tot};
    cta_add<2>(v, out);
}

// PER consecutive elements of a row as float: one vector load when `vec` (16-byte aligned rows,
// PER of 4 or 8), else scalar loads.
template <int PER>
__device__ __forceinline__ void load_run(const float* p, bool vec, float (&v)[PER]) {
    if constexpr (PER % 4 == 0) {
        if (vec) {
#pragma unroll
            for (int k = 0; k < PER / 4; ++k) {
                float t[4];
                load4(p + 4 * k, t);
#pragma unroll
                for (int e = 0; e < 4; ++e) v[4 * k + e] = t[e];
            }
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) v[e] = p[e];
}
template <int PER>
__device__ __forceinline__ void load_run(const __nv_bfloat16* p, bool vec, float (&v)[PER]) {
    if constexpr (PER % 4 == 0) {
        if (vec) {
#pragma unroll
            for (int k = 0; k < PER / 4; ++k) {
                float t[4];
                load4(p + 4 * k, t);
#pragma unroll
                for (int e = 0; e < 4; ++e) v[4 * k + e] = t[e];
            }
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) v[e] = __bfloat162float(p[e]);
}

// out[0] += sum_j hd_j sum_r (w_rj - q_rj s_rb)^2, hd_j = h[j ld_h + j].  Warp w takes quantizer
// block (column range) cb = w % nblk for the rows of slice w / nblk; its lanes hold qblock / 32
// consecutive columns each, so a lane reads its PER diagonal entries once and then one run of
// each of the slice's rows.
template <typename T, int PER>
__global__ void __launch_bounds__(kThreads) l_diag_kernel(const T* __restrict__ w, int64_t rows, int64_t cols,
                                                          int64_t ld, const float* __restrict__ h, int64_t ld_h,
                                                          bool vec, double* out) {
    constexpr int qblock = 32 * PER;
    const int lane = threadIdx.x & 31;
    const int64_t nblk = cols / qblock;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t slices = max((int64_t)1, warps / nblk);
    double acc = 0.0;
    for (int64_t it = wid; it < nblk * slices; it += warps) {
        const int64_t cb = it % nblk, slice = it / nblk;
        const int64_t r0 = rows * slice / slices, r1 = rows * (slice + 1) / slices;
        const int64_t c0 = cb * qblock + (int64_t)lane * PER;
        double hd[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) hd[e] = (double)h[(c0 + e) * ld_h + (c0 + e)];
        for (int64_t r = r0; r < r1; ++r) {
            float v[PER];
            load_run<PER>(w + r * ld + c0, vec, v);
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const double s = (double)a / 127.0;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                double target = 0.0;
                if (s > 0.0) {
                    const double qv = fmin(127.0, fmax(-127.0, rint((double)v[e] / s)));
                    target = qv * s;
                }
                const double err = (double)v[e] - target;
                acc += hd[e] * (err * err);
            }
        }
    }
    const double v[1] = {acc};
    cta_add<1>(v, out);
}

int grid_for(int64_t work_units) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        sms = 148;
    }
    return (int)std::max<int64_t>(1, std::min<int64_t>(work_units, 8 * (int64_t)sms));
}

}  // namespace

extern "C" harp_status harp_off_block_energy(const void* h, int64_t n, int64_t ld, harp_dtype dtype, int32_t q,
                                             double* out, void* stream_) {
    harp_clear_error();
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (n <= 0 || q <= 0 || n % q) return harp_fail(HARP_ERR_INVALID_ARG, "n > 0 and q > 0 dividing n");
    if (ld < n) return harp_fail(HARP_ERR_INVALID_ARG, "ld smaller than n");
    if (!h || !out) return harp_fail(HARP_ERR_INVALID_ARG, "h or out is NULL");
    const size_t es = dtype == HARP_F32 ? 4 : 2;
    if (ranges_overlap(h, ((size_t)(n - 1) * ld + n) * es, out, 2 * sizeof(double)))
        return harp_fail(HARP_ERR_INVALID_ARG, "out overlaps h");
    cudaStream_t stream = (cudaStream_t)stream_;
    cudaError_t e = cudaMemsetAsync(out, 0, 2 * sizeof(double), stream);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    const bool vec = ((uintptr_t)h % 16 == 0) && (ld * es) % 16 == 0 && n % 4 == 0 && q % 4 == 0;
    const int grid = grid_for(n);
    if (dtype == HARP_F32)
        off_block_energy_kernel<float><<<grid, kThreads, 0, stream>>>((const float*)h, n, ld, q, vec, out);
    else
        off_block_energy_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>((const __nv_bfloat16*)h, n, ld, q,
                                                                           vec, out);
    e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("off_block_energy_kernel");
    return HARP_OK;
}

extern "C" harp_status harp_l_diag(const void* w, int64_t rows, int64_t cols, int64_t ld_w, harp_dtype dtype,
                                   const float* h, int64_t ld_h, int32_t qblock, double* out, void* stream_) {
    harp_clear_error();
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (qblock != 32 && qblock != 64 && qblock != 128 && qblock != 256)
        return harp_fail(HARP_ERR_INVALID_ARG, "qblock must be 32, 64, 128 or 256");
    if (rows < 0 || cols <= 0 || cols % qblock) return harp_fail(HARP_ERR_INVALID_ARG, "qblock must divide cols");
    if (ld_w < cols || ld_h < cols) return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than cols");
    if (!out || !h || (rows > 0 && !w)) return harp_fail(HARP_ERR_INVALID_ARG, "NULL pointer");
    const size_t es = dtype == HARP_F32 ? 4 : 2;
    if ((rows > 0 && ranges_overlap(w, ((size_t)(rows - 1) * ld_w + cols) * es, out, sizeof(double))) ||
        ranges_overlap(h, ((size_t)(cols - 1) * ld_h + cols) * sizeof(float), out, sizeof(double)))
        return harp_fail(HARP_ERR_INVALID_ARG, "out overlaps w or h");
    cudaStream_t stream = (cudaStream_t)stream_;
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(double), stream);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    if (rows > 0) {
        const int grid = grid_for((rows * (cols / qblock) + kThreads / 32 - 1) / (kThreads / 32));
        const bool vec = ((uintptr_t)w % 16 == 0) && (ld_w * es) % 16 == 0;
#define HARP_LDIAG(T, PER)                                                                                 \
    l_diag_kernel<T, PER><<<grid, kThreads, 0, stream>>>((const T*)w, rows, cols, ld_w, h, ld_h, vec, out)
        const bool f = dtype == HARP_F32;
        switch (qblock) {
            case 32: if (f) HARP_LDIAG(float, 1); else HARP_LDIAG(__nv_bfloat16, 1); break;
            case 64: if (f) HARP_LDIAG(float, 2); else HARP_LDIAG(__nv_bfloat16, 2); break;
            case 128: if (f) HARP_LDIAG(float, 4); else HARP_LDIAG(__nv_bfloat16, 4); break;
            default: if (f) HARP_LDIAG(float, 8); else HARP_LDIAG(__nv_bfloat16, 8); break;
        }
#undef HARP_LDIAG
        e = cudaGetLastError();
        if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    harp_set_last_kernel("l_diag_kernel");
    return HARP_OK;
}
