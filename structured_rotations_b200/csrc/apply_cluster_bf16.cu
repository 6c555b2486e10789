// Instantiations of the cluster row kernel for bf16 rows in and out, and the cluster-occupancy
// query the host side uses to pick a cluster size.
#include <cuda_bf16.h>

#include "apply_cluster.cuh"

cudaError_t harp_cluster_launch_bf16(int which, int cl, bool inverse, const harp_cluster::ClusterParams& cp,
                                     size_t smem, int grid, cudaStream_t stream) {
    return harp_cluster::launch<__nv_bfloat16, __nv_bfloat16>(which, cl, inverse, cp, smem, grid, stream);
}

namespace {

template <int I>
const void* kernel_of(int which) {
    if constexpr (I < harp_tiled::kNumMasks) {
        if (which == I)
            return (const void*)harp_cluster::harp_cluster_kernel<__nv_bfloat16, __nv_bfloat16, false,
                                                                   harp_tiled::kMasks[I]>;
        return kernel_of<I + 1>(which);
    } else {
        return nullptr;
    }
}

}  // namespace

// Clusters of `cl` CTAs with `smem` bytes each that fit on the current device at once (0 if
// none does or the query fails).
int harp_cluster_max_active(int which, int cl, size_t smem) {
    const void* kern = kernel_of<0>(which);
    if (!kern) return 0;
    if (harp_set_smem_limit(kern, (int)smem) != (int)cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (cl > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cl);
    cfg.blockDim = dim3(harp_cluster::kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}
