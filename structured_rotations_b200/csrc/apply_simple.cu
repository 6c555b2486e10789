// General row kernel for the HARP transform (HARP technical summary §2.1 Core
// Architecture): one CTA owns a few rows, keeps them in shared memory as fp32
// across all m stages, and touches global memory once in and once out.  Stage t
// multiplies every group {lo + s_t(k + b_t hi)} by its block B_{t,c}
// (c = lo + s_t hi); the inverse walks the stages backwards with B^T.  Any
// schedule with radices in [2, 16] is accepted; the specialized kernels in
// apply_fast.cu take over for the shapes they cover.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

__device__ __forceinline__ float load_f32(const float* p) { return *p; }
__device__ __forceinline__ float load_f32(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_f32(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f32(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// y = B x (forward) or y = B^T x (inverse) for one group of B coordinates
// spaced s apart in shared memory, in place.
template <int B>
__device__ __forceinline__ void group_apply(float* __restrict__ row, int64_t base, int64_t s,
                                            const float* __restrict__ blk, bool transpose) {
    float xin[B];
#pragma unroll
    for (int l = 0; l < B; ++l) xin[l] = row[base + s * l];
    float yout[B];
#pragma unroll
    for (int k = 0; k < B; ++k) {
        float acc = 0.0f;
#pragma unroll
        for (int l = 0; l < B; ++l) {
            const float coef = transpose ? __ldg(blk + l * B + k) : __ldg(blk + k * B + l);
            acc = fmaf(coef, xin[l], acc);
        }
        yout[k] = acc;
    }
#pragma unroll
    for (int k = 0; k < B; ++k) row[base + s * k] = yout[k];
}

template <int B>
__device__ void stage_pass(float* sm, int nr, int64_t d, const StageDesc& sd,
                           const float* __restrict__ blocks, bool transpose) {
    const int64_t nb = sd.nblocks;
    const int64_t s = sd.s;
    for (int64_t task = threadIdx.x; task < (int64_t)nr * nb; task += blockDim.x) {
        const int64_t r = task / nb;
        const int64_t c = task - r * nb;
        const int64_t lo = c % s, hi = c / s;
        group_apply<B>(sm + r * d, lo + s * B * hi, s, blocks + sd.block_off + c * B * B, transpose);
    }
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) apply_simple_kernel(PlanDesc pd, const float* __restrict__ blocks,
                                                           const TIn* x, TOut* y,
                                                           int64_t rows, int64_t ld_x, int64_t ld_y,
                                                           int inverse, int rows_per_cta) {
    extern __shared__ float sm[];
    const int64_t d = pd.d;
    const int64_t row0 = (int64_t)blockIdx.x * rows_per_cta;
    const int nr = (int)min((int64_t)rows_per_cta, rows - row0);
    for (int64_t e = threadIdx.x; e < (int64_t)nr * d; e += blockDim.x) {
        const int64_t r = e / d, i = e - r * d;
        sm[e] = load_f32(x + (row0 + r) * ld_x + i);
    }
    __syncthreads();
    for (int step = 0; step < pd.m; ++step) {
        const int t = inverse ? pd.m - 1 - step : step;
        const StageDesc& sd = pd.st[t];
        switch (sd.b) {
#define HARP_CASE(R) case R: stage_pass<R>(sm, nr, d, sd, blocks, inverse != 0); break;
            HARP_CASE(2) HARP_CASE(3) HARP_CASE(4) HARP_CASE(5) HARP_CASE(6) HARP_CASE(7)
            HARP_CASE(8) HARP_CASE(9) HARP_CASE(10) HARP_CASE(11) HARP_CASE(12) HARP_CASE(13)
            HARP_CASE(14) HARP_CASE(15) HARP_CASE(16)
#undef HARP_CASE
            default: break;
        }
        __syncthreads();
    }
    for (int64_t e = threadIdx.x; e < (int64_t)nr * d; e += blockDim.x) {
        const int64_t r = e / d, i = e - r * d;
        store_f32(y + (row0 + r) * ld_y + i, sm[e]);
    }
}

template <typename TIn, typename TOut>
harp_status launch_typed(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                         int64_t ld_y, harp_dir dir, cudaStream_t stream) {
    const int64_t d = p->desc.d;
    const size_t row_bytes = sizeof(float) * d;
    // up to 8 rows per CTA within 96 KB, so two CTAs fit on one SM; one row if it is bigger
    int rpc = (int)std::max<int64_t>(1, std::min<int64_t>(8, (96 * 1024) / row_bytes));
    const size_t smem = row_bytes * rpc;
    auto kern = apply_simple_kernel<TIn, TOut>;
    if (smem > 48 * 1024) {
        cudaError_t e = (cudaError_t)harp_set_smem_limit((const void*)kern, (int)smem);
        if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    const int64_t grid = (rows + rpc - 1) / rpc;
    if (grid > 0x7fffffff) return harp_fail(HARP_ERR_INVALID_ARG, "too many rows for one launch");
    kern<<<(unsigned)grid, 256, smem, stream>>>(p->desc, p->d_blocks, (const TIn*)x, (TOut*)y, rows,
                                               ld_x, ld_y, dir == HARP_INVERSE ? 1 : 0, rpc);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("apply_simple_kernel");
    return HARP_OK;
}

}  // namespace

harp_status launch_apply_simple(const harp_plan_s* p, const void* x, void* y, int64_t rows,
                                int64_t ld_x, int64_t ld_y, harp_dtype in_dtype,
                                harp_dtype out_dtype, harp_dir dir, void* stream_) {
    cudaStream_t stream = (cudaStream_t)stream_;
    if (in_dtype == HARP_F32 && out_dtype == HARP_F32)
        return launch_typed<float, float>(p, x, y, rows, ld_x, ld_y, dir, stream);
    if (in_dtype == HARP_BF16 && out_dtype == HARP_BF16)
        return launch_typed<__nv_bfloat16, __nv_bfloat16>(p, x, y, rows, ld_x, ld_y, dir, stream);
    if (in_dtype == HARP_BF16 && out_dtype == HARP_F32)
        return launch_typed<__nv_bfloat16, float>(p, x, y, rows, ld_x, ld_y, dir, stream);
    return launch_typed<float, __nv_bfloat16>(p, x, y, rows, ld_x, ld_y, dir, stream);
}
