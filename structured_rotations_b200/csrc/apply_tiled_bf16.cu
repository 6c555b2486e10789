// Instantiations of the tiled row kernel for bf16 rows in and out.
#include <cuda_bf16.h>

#include "apply_tiled.cuh"

cudaError_t harp_tiled_launch_bf16(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                  size_t smem, int grid, cudaStream_t stream) {
    return harp_tiled::launch<__nv_bfloat16, __nv_bfloat16>(which, V, nt, cl, inverse, tp, smem, grid, stream);
}
