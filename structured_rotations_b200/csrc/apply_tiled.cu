// Host launcher of the general tiled row kernel (kernel and layout in apply_tiled.cuh;
// HARP technical summary §2.1 Core Architecture).  Picks the rows per tile R from the
// shared-memory budget, the radix-set instantiation that covers the schedule, and one
// persistent CTA per SM.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "apply_tiled.cuh"
#include "harp_internal.h"

namespace {

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 1;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

harp_status launch_apply_tiled(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                               int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir,
                               void* stream) {
    using namespace harp_tiled;
    const int64_t d = p->desc.d;
    if (d % 8 != 0) return HARP_ERR_UNSUPPORTED;
    int mask = 0;
    for (int t = 0; t < p->desc.m; ++t) {
        if (p->desc.st[t].b > 8) return HARP_ERR_UNSUPPORTED;
        mask |= 1 << p->desc.st[t].b;
    }
    if (in_dtype == HARP_F32 && out_dtype == HARP_BF16) return HARP_ERR_UNSUPPORTED;
    const int64_t es_in = in_dtype == HARP_F32 ? 4 : 2, es_out = out_dtype == HARP_F32 ? 4 : 2;
    if (((uintptr_t)x & 15) || ((uintptr_t)y & 15) || ((ld_x * es_in) & 15) || ((ld_y * es_out) & 15))
        return HARP_ERR_UNSUPPORTED;
    int which = 0;
    while (which < kNumMasks && (kMasks[which] & mask) != mask) ++which;
    if (which == kNumMasks) return HARP_ERR_UNSUPPORTED;

    // Rows per tile: fp32 tile plus a staging area for the next tile's raw rows when two
    // or more rows fit that way, else the fp32 tile alone (loads then do not overlap).
    const int64_t per_row_staged = d * (4 + es_in);
    const int64_t per_row = d * 4;
    const int64_t budget = kSmemOptIn - 64;
    int64_t R = std::min<int64_t>(kMaxTileRows, budget / per_row_staged);
    int staged = 1;
    if (R < 2) {
        R = std::min<int64_t>(kMaxTileRows, budget / per_row);
        staged = 0;
    }
    if (R < 1) return HARP_ERR_UNSUPPORTED;
    R = std::min<int64_t>(R, rows);

    TiledParams tp;
    tp.pd = p->desc;
    tp.blocks = p->d_blocks;
    tp.x = x;
    tp.y = y;
    tp.rows = rows;
    tp.ld_x = ld_x;
    tp.ld_y = ld_y;
    tp.ntiles = (rows + R - 1) / R;
    tp.R = (int)R;
    tp.staged = staged;
    tp.swz = (d % 32 == 0) ? 0x18 : 0;
    tp.status = p->d_status;
    const size_t smem = (size_t)(staged ? per_row_staged : per_row) * R + 16;
    const int grid = (int)std::min<int64_t>(tp.ntiles, sm_count());
    cudaStream_t s = (cudaStream_t)stream;
    const bool inv = dir == HARP_INVERSE;
    cudaError_t e;
    if (in_dtype == HARP_BF16 && out_dtype == HARP_BF16)
        e = harp_tiled_launch_bf16(which, inv, tp, smem, grid, s);
    else if (in_dtype == HARP_F32)
        e = harp_tiled_launch_f32(which, inv, tp, smem, grid, s);
    else
        e = harp_tiled_launch_bf16_f32(which, inv, tp, smem, grid, s);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_tiled_kernel");
    return HARP_OK;
}
