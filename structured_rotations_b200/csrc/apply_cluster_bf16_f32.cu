// Instantiations of the cluster row kernel for __nv_bfloat16 rows in, float rows out.
#include <cuda_bf16.h>

#include "apply_cluster.cuh"

cudaError_t harp_cluster_launch_bf16_f32(int which, int cl, bool inverse, const harp_cluster::ClusterParams& cp,
                                     size_t smem, int grid, cudaStream_t stream) {
    return harp_cluster::launch<__nv_bfloat16, float>(which, cl, inverse, cp, smem, grid, stream);
}
