// Instantiations of the tiled row kernel for bf16 rows in, fp32 rows out (first pass of the two-sided rotation).
#include <cuda_bf16.h>

#include "apply_tiled.cuh"

cudaError_t harp_tiled_launch_bf16_f32(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                  size_t smem, int grid, cudaStream_t stream) {
    return harp_tiled::launch<__nv_bfloat16, float>(which, V, nt, cl, inverse, tp, smem, grid, stream);
}
