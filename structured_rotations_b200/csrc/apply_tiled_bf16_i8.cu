// Instantiations of the tiled row kernel for bf16 rows in and int8 codes with per-block
// fp32 scales out (the fused quantizer epilogue).
#include <cuda_bf16.h>

#include "apply_tiled.cuh"

cudaError_t harp_tiled_launch_bf16_i8(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                      size_t smem, int grid, cudaStream_t stream) {
    return harp_tiled::launch<__nv_bfloat16, int8_t>(which, V, nt, cl, inverse, tp, smem, grid, stream);
}
