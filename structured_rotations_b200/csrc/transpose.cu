// Tiled out-of-place transpose used by the two-sided rotation (the columns of
// W are rotated as rows of W^T).  32x32 tiles staged through shared memory, with
// a padded row so the column reads hit 32 distinct banks.  Widens bf16 to fp32
// or rounds fp32 to bf16 (nearest even) on the way through.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

__device__ __forceinline__ float ld_f32(const float* p) { return *p; }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f32(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_f32(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) transpose_kernel(const TIn* __restrict__ src, TOut* __restrict__ dst,
                                                        int64_t rows, int64_t cols, int64_t ld_src,
                                                        int64_t ld_dst) {
    __shared__ float tile[32][33];
    const int64_t c0 = (int64_t)blockIdx.x * 32, r0 = (int64_t)blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        const int64_t r = r0 + ty + j, c = c0 + tx;
        if (r < rows && c < cols) tile[ty + j][tx] = ld_f32(src + r * ld_src + c);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        const int64_t c = c0 + ty + j, r = r0 + tx;   // dst[c][r] = src[r][c]
        if (r < rows && c < cols) st_f32(dst + c * ld_dst + r, tile[tx][ty + j]);
    }
}

template <typename TIn, typename TOut>
harp_status go(const void* src, void* dst, int64_t rows, int64_t cols, int64_t ld_src,
               int64_t ld_dst, cudaStream_t stream) {
    dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
    transpose_kernel<TIn, TOut><<<grid, 256, 0, stream>>>((const TIn*)src, (TOut*)dst, rows, cols,
                                                          ld_src, ld_dst);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HARP_OK : harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
}

}  // namespace

harp_status launch_transpose(const void* src, void* dst, int64_t rows, int64_t cols,
                             int64_t ld_src, int64_t ld_dst, harp_dtype in_dtype,
                             harp_dtype out_dtype, void* stream_) {
    cudaStream_t stream = (cudaStream_t)stream_;
    if (rows == 0 || cols == 0) return HARP_OK;
    if ((rows + 31) / 32 > 65535) return harp_fail(HARP_ERR_INVALID_ARG, "transpose: too many rows");
    if (in_dtype == HARP_F32 && out_dtype == HARP_F32) return go<float, float>(src, dst, rows, cols, ld_src, ld_dst, stream);
    if (in_dtype == HARP_BF16 && out_dtype == HARP_F32) return go<__nv_bfloat16, float>(src, dst, rows, cols, ld_src, ld_dst, stream);
    if (in_dtype == HARP_F32 && out_dtype == HARP_BF16) return go<float, __nv_bfloat16>(src, dst, rows, cols, ld_src, ld_dst, stream);
    return go<__nv_bfloat16, __nv_bfloat16>(src, dst, rows, cols, ld_src, ld_dst, stream);
}
