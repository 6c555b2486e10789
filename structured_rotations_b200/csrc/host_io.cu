// harp_apply_host: the row transform between host buffers, with the copies inside
// (HARP technical summary §2.1: rows in, rotated rows out).  Rows go through the GPU in
// chunks on three streams; on each stream a chunk's host-to-device copy, its row kernel
// and its device-to-host copy follow each other in order, and the three streams overlap,
// so the two copy directions (separate copy engines) and the kernels run at once.
#include <algorithm>
#include <mutex>
#include <string>

#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kSlots = 3;
constexpr size_t kChunkBytes = (size_t)32 << 20;   // rows per chunk: about 32 MiB of input

struct HostIo {
    int device = -1;
    size_t slot_bytes = 0;        // bytes of each device buffer
    cudaStream_t stream[kSlots] = {};
    void* din[kSlots] = {};
    void* dout[kSlots] = {};
};

void release(HostIo* h) {
    for (int k = 0; k < kSlots; ++k) {
        if (h->stream[k]) cudaStreamDestroy(h->stream[k]);
        cudaFree(h->din[k]);
        cudaFree(h->dout[k]);
        h->stream[k] = nullptr;
        h->din[k] = h->dout[k] = nullptr;
    }
    h->slot_bytes = 0;
}

harp_status ensure(harp_plan_s* p, size_t bytes) {
    HostIo* h = (HostIo*)p->host_io;
    if (!h) {
        h = new HostIo();
        p->host_io = h;
        h->device = p->device;
    }
    if (!h->stream[0]) {
        for (int k = 0; k < kSlots; ++k)
            if (cudaStreamCreateWithFlags(&h->stream[k], cudaStreamNonBlocking) != cudaSuccess) {
                cudaGetLastError();
                release(h);
                return harp_fail(HARP_ERR_CUDA, "cudaStreamCreate failed");
            }
    }
    if (h->slot_bytes < bytes) {
        for (int k = 0; k < kSlots; ++k) {
            cudaFree(h->din[k]);
            cudaFree(h->dout[k]);
            h->din[k] = h->dout[k] = nullptr;
        }
        h->slot_bytes = 0;
        for (int k = 0; k < kSlots; ++k)
            if (cudaMalloc(&h->din[k], bytes) != cudaSuccess || cudaMalloc(&h->dout[k], bytes) != cudaSuccess) {
                cudaGetLastError();
                release(h);
                return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the staging buffers failed");
            }
        h->slot_bytes = bytes;
    }
    return HARP_OK;
}

}  // namespace

void host_io_free(harp_plan_s* p) {
    HostIo* h = (HostIo*)p->host_io;
    if (!h) return;
    release(h);
    delete h;
    p->host_io = nullptr;
}

extern "C" harp_status harp_apply_host(harp_plan_t p, const void* x, void* y, int64_t rows, int64_t ld_x,
                                       int64_t ld_y, harp_dtype dtype, harp_dir dir) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (dir != HARP_FORWARD && dir != HARP_INVERSE) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown direction");
    if (rows < 0) return harp_fail(HARP_ERR_INVALID_ARG, "rows < 0");
    const int64_t d = p->desc.d;
    if (ld_x < d || ld_y < d) return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than d");
    if (rows == 0) return HARP_OK;
    if (!x || !y) return harp_fail(HARP_ERR_INVALID_ARG, "x or y is NULL");
    {
        // int8 plans materialize on their first call (on the legacy stream, synchronized)
        const harp_status mst = harp_require_materialized(p, nullptr);
        if (mst != HARP_OK) return mst;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (dev != p->device) return harp_fail(HARP_ERR_WRONG_DEVICE, "plan materialized on another device");
    const size_t es = dtype == HARP_F32 ? 4 : 2;
    const size_t row_bytes = (size_t)d * es;
    if (x != y) {
        const char* a = (const char*)x;
        const char* b = (const char*)y;
        const size_t na = ((size_t)(rows - 1) * ld_x + d) * es, nb = ((size_t)(rows - 1) * ld_y + d) * es;
        if (a < b + nb && b < a + na) return harp_fail(HARP_ERR_INVALID_ARG, "x and y overlap without being equal");
    } else if (ld_x != ld_y) {
        return harp_fail(HARP_ERR_INVALID_ARG, "in-place apply needs ld_x == ld_y");
    }
    const int64_t chunk = std::max<int64_t>(32, std::min<int64_t>(rows, (int64_t)(kChunkBytes / row_bytes)));
    std::lock_guard<std::mutex> lock(p->host_io_mu);   // the plan's streams and buffers serve one call at a time
    harp_status st = ensure(p, (size_t)chunk * row_bytes);
    if (st != HARP_OK) return st;
    HostIo* h = (HostIo*)p->host_io;
    // On an error after the first enqueue, the earlier chunks' copies may still be reading x
    // or writing y: wait for all three streams before returning, so the caller may free or
    // reuse its buffers at once.
    auto drain_and_fail = [&](harp_status s, const std::string& msg) {
        for (int i = 0; i < kSlots; ++i) cudaStreamSynchronize(h->stream[i]);
        cudaGetLastError();
        return harp_fail(s, msg);
    };
    const char* xs = (const char*)x;
    char* ys = (char*)y;
    int64_t k = 0;
    for (int64_t r0 = 0; r0 < rows; r0 += chunk, ++k) {
        const int slot = (int)(k % kSlots);
        cudaStream_t s = h->stream[slot];
        const int64_t n = std::min(chunk, rows - r0);
        cudaError_t e = cudaMemcpy2DAsync(h->din[slot], row_bytes, xs + (size_t)r0 * ld_x * es, (size_t)ld_x * es,
                                          row_bytes, (size_t)n, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return drain_and_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
        st = run_rows(p, h->din[slot], h->dout[slot], n, d, d, dtype, dtype, dir, s);
        if (st != HARP_OK) return drain_and_fail(st, harp_last_error());
        e = cudaMemcpy2DAsync(ys + (size_t)r0 * ld_y * es, (size_t)ld_y * es, h->dout[slot], row_bytes, row_bytes,
                              (size_t)n, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return drain_and_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    cudaError_t first = cudaSuccess;
    for (int i = 0; i < kSlots; ++i) {
        const cudaError_t e = cudaStreamSynchronize(h->stream[i]);
        if (e != cudaSuccess && first == cudaSuccess) first = e;
    }
    if (first != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(first));
    return HARP_OK;
}
