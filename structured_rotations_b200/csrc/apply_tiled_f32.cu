// Instantiations of the tiled row kernel for fp32 rows in and out.
#include <cuda_bf16.h>

#include "apply_tiled.cuh"

cudaError_t harp_tiled_launch_f32(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                  size_t smem, int grid, cudaStream_t stream) {
    return harp_tiled::launch<float, float>(which, V, nt, cl, inverse, tp, smem, grid, stream);
}
