// Composition of rotations: harp_plan_compose makes one plan whose transform is
// T_{k-1} ... T_1 T_0 for plans T_j of one dimension.  Independent randomized Hadamard
// transforms are composed to bring every input's coordinates closer to the Gaussian
// behaviour of a uniform random rotation (the RHT-composition results quoted with the HARP
// pages: two passes for scalar quantization, three for vector quantization).
//
// The composite's stage list is the plans' stages one after another (each plan's signs are
// already folded into its own first stage's blocks), with copies of their device blocks,
// so the row kernels run all k transforms while a tile stays in shared memory: one HBM
// pass instead of k.  The row kernels (specialized, tiled, simple) take any stride per
// stage; kernels that rely on s_t = prod_{j<t} b_j (the column passes, slab mode, the
// calibration backward) decline composites.
#include <cuda_runtime.h>

#include "harp_internal.h"

extern "C" harp_status harp_plan_compose(harp_plan_t* out, const harp_plan_t* plans, int32_t k, void* stream_) {
    harp_clear_error();
    if (!out) return harp_fail(HARP_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!plans || k < 1) return harp_fail(HARP_ERR_INVALID_ARG, "need at least one plan");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    int64_t d = -1;
    int m = 0;
    for (int j = 0; j < k; ++j) {
        harp_plan_s* p = plans[j];
        if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "a plan is NULL");
        const harp_status mst = harp_require_materialized(plans[j], stream_);   // int8 plans: implicitly
        if (mst != HARP_OK) return mst;
        if (p->device != dev) return harp_fail(HARP_ERR_WRONG_DEVICE, "plans must be materialized on the current device");
        if (d >= 0 && p->desc.d != d) return harp_fail(HARP_ERR_INVALID_ARG, "plans of different dimensions");
        d = p->desc.d;
        m += p->desc.m;
    }
    if (m > HARP_MAX_STAGES)
        return harp_fail(HARP_ERR_SCHEDULE, "more than " + std::to_string(HARP_MAX_STAGES) + " stages in all");

    harp_plan_s* c = new (std::nothrow) harp_plan_s();
    if (!c) return harp_fail(HARP_ERR_ALLOC, "host allocation of the plan");
    c->desc.d = d;
    c->desc.m = m;
    c->kind = HARP_THETA_F32;
    c->composite = true;
    c->device = dev;
    int T = 0;
    int64_t boff = 0, loff = 0, toff = 0;
    for (int j = 0; j < k; ++j) {
        const harp_plan_s* p = plans[j];
        for (int t = 0; t < p->desc.m; ++t, ++T) {
            c->desc.st[T] = p->desc.st[t];
            c->desc.st[T].block_off += boff;
            c->desc.st[T].theta_off += toff;
            c->lane_off[T] = p->lane_off[t] + loff;
        }
        boff += p->block_floats;
        loff += p->lane_floats;
        toff += p->theta_total;
    }
    c->block_floats = boff;
    c->lane_floats = loff;
    c->theta_total = toff;
    cudaStream_t stream = (cudaStream_t)stream_;
    auto fail = [&](harp_status s, const char* msg) {
        cudaGetLastError();
        harp_device_free(c);
        delete c;
        return harp_fail(s, msg);
    };
    if (cudaMalloc((void**)&c->d_blocks, sizeof(float) * boff) != cudaSuccess ||
        cudaMalloc((void**)&c->d_blocks_lanes, sizeof(float) * loff) != cudaSuccess ||
        cudaMalloc((void**)&c->d_status, 64) != cudaSuccess)
        return fail(HARP_ERR_ALLOC, "cudaMalloc of the composite's blocks failed");
    boff = loff = 0;
    cudaError_t e = cudaMemsetAsync(c->d_status, 0, 64, stream);
    for (int j = 0; j < k && e == cudaSuccess; ++j) {
        const harp_plan_s* p = plans[j];
        e = cudaMemcpyAsync(c->d_blocks + boff, p->d_blocks, sizeof(float) * p->block_floats,
                            cudaMemcpyDeviceToDevice, stream);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(c->d_blocks_lanes + loff, p->d_blocks_lanes, sizeof(float) * p->lane_floats,
                                cudaMemcpyDeviceToDevice, stream);
        boff += p->block_floats;
        loff += p->lane_floats;
    }
    if (e == cudaSuccess) {
        fast_prepare(c, stream);   // a composite of one (8,8,8,8) plan of d = 4096 takes the specialized kernel
        e = cudaGetLastError();
    }
    // wait for the copies, so that the source plans may be destroyed as soon as this returns
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    c->materialized = true;
    *out = c;
    return HARP_OK;
}
