// Two-sided rotation for callers that cannot allocate device memory.
//
// harp_apply_two_sided needs a caller-provided workspace of two fp32 copies of
// the weight.  Some callers cannot call cudaMalloc at the point where they rotate
// a weight: code running inside a memory pool or arena they do not own, graph
// capture regions, and embedded runtimes whose allocator is not exposed to
// plugins.  This entry point takes its workspace from a fixed array that lives in
// the library's device image instead, so it allocates nothing per call.
//
// The array is HARP_NOALLOC_SCRATCH_BYTES (32 MiB) of device memory on every GPU
// that loads the library, held until the process exits.  All calls share it:
// calls whose work overlaps on the GPU (two streams, or two host threads) race on
// it, so serialize them.  Nothing in it has to start at zero: every byte a call
// reads was written earlier by the same call.
#include <algorithm>
#include <mutex>
#include <string>

#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr size_t kScratchBytes = HARP_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_harp_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up once per device
// with that device current and kept for the life of the process; it does not survive
// cudaDeviceReset (the module may come back at another address), after which this
// entry point must not be called again in the same process.
harp_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (dev < 0 || dev >= kMaxDevices) return harp_fail(HARP_ERR_UNSUPPORTED, "device index too large");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_harp_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HARP_OK;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const char* pa = (const char*)a;
    const char* pb = (const char*)b;
    return pa < pb + nb && pb < pa + na;
}

}  // namespace

extern "C" size_t harp_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" harp_status harp_apply_two_sided_noalloc(harp_plan_t pu, harp_plan_t pv, const void* W,
                                                    void* W_out, int64_t n_out, int64_t n_in,
                                                    int64_t ld, harp_dtype dtype, void* stream) {
    harp_clear_error();
    if (!pu || !pv) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (n_out <= 0 || n_in <= 0) return harp_fail(HARP_ERR_INVALID_ARG, "empty weight");
    if (pu->desc.d != n_out) return harp_fail(HARP_ERR_INVALID_ARG, "planU dimension differs from n_out");
    if (pv->desc.d != n_in) return harp_fail(HARP_ERR_INVALID_ARG, "planV dimension differs from n_in");
    if (ld < n_in) return harp_fail(HARP_ERR_INVALID_ARG, "ld smaller than n_in");
    if (!W || !W_out) return harp_fail(HARP_ERR_INVALID_ARG, "NULL pointer");
    const size_t half = ((size_t)n_out * (size_t)n_in * sizeof(float) + 255) & ~(size_t)255;
    if (2 * half > kScratchBytes)
        return harp_fail(HARP_ERR_INVALID_ARG,
                         "weight too large for the static scratch: n_out * n_in must be at most " +
                             std::to_string(kScratchBytes / 8) + " elements");
    harp_status st;
    if ((st = harp_require_materialized(pu, stream)) != HARP_OK || (st = harp_require_materialized(pv, stream)) != HARP_OK)
        return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (pu->device != dev || pv->device != dev)
        return harp_fail(HARP_ERR_WRONG_DEVICE, "plans materialized on another device");
    const size_t es = dtype == HARP_F32 ? 4 : 2;
    const size_t wbytes = ((n_out - 1) * ld + n_in) * es;
    if (W != W_out && overlap(W, wbytes, W_out, wbytes))
        return harp_fail(HARP_ERR_INVALID_ARG, "W and W_out overlap without being equal");

    {
        // each row pass holds one whole fp32 row in shared memory: check the longer side against
        // the device's opt-in limit now, before anything is enqueued
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_CUDA, "cannot read the shared-memory limit");
        }
        if ((size_t)std::max(n_out, n_in) * sizeof(float) > (size_t)optin)
            return harp_fail(HARP_ERR_UNSUPPORTED, "a side of the weight is too long for one fp32 row in shared memory (" +
                                                       std::to_string(optin / 4) + " elements at most)");
    }
    void* scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != HARP_OK) return st;
    float* ws1 = (float*)scratch;
    float* ws2 = (float*)((char*)scratch + half);
    // rows of W: w_r <- T_V^T w_r, kept in fp32
    st = launch_apply_simple(pv, W, ws1, n_out, ld, n_in, dtype, HARP_F32, HARP_INVERSE, stream);
    if (st != HARP_OK) return st;
    if ((st = launch_transpose(ws1, ws2, n_out, n_in, n_in, n_out, HARP_F32, HARP_F32, stream)) != HARP_OK)
        return st;
    // columns of W: col <- T_U^T col, as rows of the transposed copy
    st = launch_apply_simple(pu, ws2, ws2, n_in, n_out, n_out, HARP_F32, HARP_F32, HARP_INVERSE, stream);
    if (st != HARP_OK) return st;
    return launch_transpose(ws2, W_out, n_in, n_out, n_out, ld, HARP_F32, dtype, stream);
}
