// C entry points that run device work: argument checks and dispatch between the
// specialized and the general row kernels, and the two-sided weight rotation
// (HARP abstract: a two-sided orthogonal processor; W_out = T_U^T W T_V).
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

size_t esize(harp_dtype t) { return t == HARP_F32 ? 4 : 2; }

harp_status check_device(const harp_plan_s* p) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (dev != p->device)
        return harp_fail(HARP_ERR_WRONG_DEVICE, "plan materialized on device " + std::to_string(p->device) +
                                                    ", current device is " + std::to_string(dev));
    return HARP_OK;
}

// HARP_KERNEL selects the row kernel: unset = the fastest one that covers the shape
// (specialized, then the cluster kernel for small batches, then tiled, then simple);
// "simple", "tiled", "cluster" or "fast" (specialized) force one and fail with
// HARP_ERR_UNSUPPORTED if it does not cover the shape.
enum { kAuto = 0, kSimple = 1, kFast = 2, kTiled = 3, kCluster = 4 };

int kernel_choice() {
    const char* v = std::getenv("HARP_KERNEL");
    if (!v) return kAuto;
    if (!std::strcmp(v, "simple")) return kSimple;
    if (!std::strcmp(v, "fast")) return kFast;
    if (!std::strcmp(v, "tiled")) return kTiled;
    if (!std::strcmp(v, "cluster")) return kCluster;
    return kAuto;
}

// Batches below this many rows take the cluster kernel when the plan has one: their cost is
// the blocks' reads, which the cluster spreads over its CTAs (measured on B200: 1 and 16 rows of
// d = 4096 / 5120 / 8192 faster on it, 256 rows of d = 4096 and 8192 faster on the tiled kernel).
constexpr int64_t kClusterRows = 65;

}  // namespace

int harp_set_smem_limit(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, int> done;   // (device, kernel) -> limit set
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find({dev, kernel});
    if (it != done.end() && it->second >= bytes) return (int)cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[{dev, kernel}] = bytes;
    return (int)e;
}

// The row kernels in order of preference.
harp_status run_rows(harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x, int64_t ld_y,
                     harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir, void* stream) {
    const int choice = kernel_choice();
    harp_status st;
    if (choice == kAuto || choice == kFast) {
        st = launch_apply_fast(p, x, y, rows, ld_x, ld_y, in_dtype, dir, stream, out_dtype);
        if (st != HARP_ERR_UNSUPPORTED || choice == kFast) return st;
        harp_clear_error();
    }
    if (choice == kCluster || (choice == kAuto && rows < kClusterRows)) {
        st = launch_apply_cluster(p, x, y, rows, ld_x, ld_y, in_dtype, out_dtype, dir, stream);
        if (st != HARP_ERR_UNSUPPORTED || choice == kCluster) return st;
        harp_clear_error();
    }
    if (choice == kAuto || choice == kTiled) {
        st = launch_apply_tiled(p, x, y, rows, ld_x, ld_y, in_dtype, out_dtype, dir, stream);
        if (st != HARP_ERR_UNSUPPORTED || choice == kTiled) return st;
        harp_clear_error();
    }
    return launch_apply_simple(p, x, y, rows, ld_x, ld_y, in_dtype, out_dtype, dir, stream);
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
    const char* pa = (const char*)a;
    const char* pb = (const char*)b;
    return pa < pb + nb && pb < pa + na;
}


namespace {

harp_status apply_checked(harp_plan_t p, const void* x, void* y, int64_t rows, int64_t ld_x, int64_t ld_y,
                          harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir, void* stream) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if ((in_dtype != HARP_F32 && in_dtype != HARP_BF16) || (out_dtype != HARP_F32 && out_dtype != HARP_BF16))
        return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (dir != HARP_FORWARD && dir != HARP_INVERSE) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown direction");
    if (rows < 0) return harp_fail(HARP_ERR_INVALID_ARG, "rows < 0");
    const int64_t d = p->desc.d;
    if (ld_x < d || ld_y < d) return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than d");
    if (rows == 0) return HARP_OK;
    if (!x || !y) return harp_fail(HARP_ERR_INVALID_ARG, "x or y is NULL");
    harp_status st = harp_require_materialized(p, stream);
    if (st != HARP_OK) return st;
    st = check_device(p);
    if (st != HARP_OK) return st;
    const size_t es_in = esize(in_dtype), es_out = esize(out_dtype);
    if (x == y) {
        if (ld_x != ld_y || in_dtype != out_dtype)
            return harp_fail(HARP_ERR_INVALID_ARG, "in-place apply needs ld_x == ld_y and one element type");
    } else if (ranges_overlap(x, ((rows - 1) * ld_x + d) * es_in, y, ((rows - 1) * ld_y + d) * es_out)) {
        return harp_fail(HARP_ERR_INVALID_ARG, "x and y overlap without being equal");
    }
    return run_rows(p, x, y, rows, ld_x, ld_y, in_dtype, out_dtype, dir, stream);
}

}  // namespace

extern "C" harp_status harp_apply(harp_plan_t p, const void* x, void* y, int64_t rows,
                                  int64_t ld_x, int64_t ld_y, harp_dtype dtype, harp_dir dir,
                                  void* stream) {
    return apply_checked(p, x, y, rows, ld_x, ld_y, dtype, dtype, dir, stream);
}

extern "C" harp_status harp_apply_ex(harp_plan_t p, const void* x, void* y, int64_t rows, int64_t ld_x,
                                     int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir,
                                     void* stream) {
    return apply_checked(p, x, y, rows, ld_x, ld_y, in_dtype, out_dtype, dir, stream);
}

extern "C" harp_status harp_apply_quant(harp_plan_t p, const void* x, int64_t rows, int64_t ld_x, harp_dtype in_dtype,
                                        int8_t* q, int64_t ld_q, float* scales, int64_t ld_s, int32_t qblock,
                                        harp_dir dir, void* stream) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (in_dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "the fused quantizer takes bf16 rows");
    if (dir != HARP_FORWARD && dir != HARP_INVERSE) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown direction");
    if (rows < 0) return harp_fail(HARP_ERR_INVALID_ARG, "rows < 0");
    const int64_t d = p->desc.d;
    if (qblock != 32 && qblock != 64 && qblock != 128 && qblock != 256)
        return harp_fail(HARP_ERR_INVALID_ARG, "qblock must be 32, 64, 128 or 256");
    if (d % qblock) return harp_fail(HARP_ERR_INVALID_ARG, "qblock must divide d");
    if (ld_x < d || ld_q < d || ld_s < d / qblock)
        return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than the row");
    if (rows == 0) return HARP_OK;
    if (!x || !q || !scales) return harp_fail(HARP_ERR_INVALID_ARG, "x, q or scales is NULL");
    harp_status st = harp_require_materialized(p, stream);
    if (st != HARP_OK) return st;
    st = check_device(p);
    if (st != HARP_OK) return st;
    const size_t xb = ((rows - 1) * ld_x + d) * 2, qb = (rows - 1) * ld_q + d,
                 sb = ((rows - 1) * ld_s + d / qblock) * sizeof(float);
    if (ranges_overlap(x, xb, q, qb) || ranges_overlap(x, xb, scales, sb) || ranges_overlap(q, qb, scales, sb))
        return harp_fail(HARP_ERR_INVALID_ARG, "x, q and scales overlap");
    const int choice = kernel_choice();
    if (choice == kAuto || choice == kFast) {
        st = launch_apply_fast_quant(p, x, rows, ld_x, q, ld_q, scales, ld_s, qblock, dir, stream);
        if (st != HARP_ERR_UNSUPPORTED || choice == kFast) return st;
        harp_clear_error();
    }
    QuantOut qo{scales, ld_s, qblock};
    st = launch_apply_tiled(p, x, q, rows, ld_x, ld_q, HARP_BF16, HARP_BF16, dir, stream, &qo);
    if (st == HARP_ERR_UNSUPPORTED)
        return harp_fail(HARP_ERR_UNSUPPORTED, "the fused quantizer needs radices <= 8, d % 8 == 0, 16-byte "
                                               "aligned x and q rows (ld_q a multiple of 16)");
    return st;
}

extern "C" harp_status harp_apply_columns(harp_plan_t p, float* x, int64_t ld_x, int64_t ncols, void* y,
                                          int64_t ld_y, harp_dtype out_dtype, harp_dir dir, void* stream) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (out_dtype != HARP_F32 && out_dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (dir != HARP_FORWARD && dir != HARP_INVERSE) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown direction");
    if (ncols < 0) return harp_fail(HARP_ERR_INVALID_ARG, "ncols < 0");
    if (ld_x < ncols || ld_y < ncols) return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than ncols");
    if (ncols == 0) return HARP_OK;
    if (!x || !y) return harp_fail(HARP_ERR_INVALID_ARG, "x or y is NULL");
    harp_status st = harp_require_materialized(p, stream);
    if (st != HARP_OK) return st;
    st = check_device(p);
    if (st != HARP_OK) return st;
    const int64_t d = p->desc.d;
    const size_t xb = ((d - 1) * ld_x + ncols) * sizeof(float), yb = ((d - 1) * ld_y + ncols) * esize(out_dtype);
    if ((void*)x == y) {
        if (ld_x != ld_y || out_dtype != HARP_F32)
            return harp_fail(HARP_ERR_INVALID_ARG, "in place needs ld_x == ld_y and fp32 output");
    } else if (ranges_overlap(x, xb, y, yb)) {
        return harp_fail(HARP_ERR_INVALID_ARG, "x and y overlap without being equal");
    }
    st = launch_cols(p, x, ld_x, ncols, y, ld_y, out_dtype, dir, stream);
    if (st == HARP_ERR_UNSUPPORTED) return harp_fail(st, "shape or alignment not covered by the column kernel");
    return st;
}

extern "C" size_t harp_two_sided_workspace_bytes(int64_t n_out, int64_t n_in) {
    if (n_out <= 0 || n_in <= 0) return 0;
    const size_t one = ((size_t)n_out * (size_t)n_in * sizeof(float) + 255) & ~(size_t)255;
    return 2 * one;
}

extern "C" harp_status harp_apply_two_sided(harp_plan_t pu, harp_plan_t pv, const void* W,
                                            void* W_out, int64_t n_out, int64_t n_in, int64_t ld,
                                            harp_dtype dtype, void* workspace, size_t ws_bytes,
                                            void* stream) {
    harp_clear_error();
    if (!pu || !pv) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (n_out <= 0 || n_in <= 0) return harp_fail(HARP_ERR_INVALID_ARG, "empty weight");
    if (pu->desc.d != n_out) return harp_fail(HARP_ERR_INVALID_ARG, "planU dimension differs from n_out");
    if (pv->desc.d != n_in) return harp_fail(HARP_ERR_INVALID_ARG, "planV dimension differs from n_in");
    if (ld < n_in) return harp_fail(HARP_ERR_INVALID_ARG, "ld smaller than n_in");
    if (!W || !W_out || !workspace) return harp_fail(HARP_ERR_INVALID_ARG, "NULL pointer");
    if (((uintptr_t)workspace & 255) != 0) return harp_fail(HARP_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    if (ws_bytes < harp_two_sided_workspace_bytes(n_out, n_in))
        return harp_fail(HARP_ERR_INVALID_ARG, "workspace too small");
    harp_status st;
    if ((st = harp_require_materialized(pu, stream)) != HARP_OK || (st = harp_require_materialized(pv, stream)) != HARP_OK)
        return st;
    if ((st = check_device(pu)) != HARP_OK || (st = check_device(pv)) != HARP_OK) return st;
    const size_t es = esize(dtype);
    const size_t wbytes = ((n_out - 1) * ld + n_in) * es;
    if (W != W_out && ranges_overlap(W, wbytes, W_out, wbytes))
        return harp_fail(HARP_ERR_INVALID_ARG, "W and W_out overlap without being equal");
    if (ranges_overlap(W, wbytes, workspace, ws_bytes) || ranges_overlap(W_out, wbytes, workspace, ws_bytes))
        return harp_fail(HARP_ERR_INVALID_ARG, "workspace overlaps the weight");

    float* ws1 = (float*)workspace;
    float* ws2 = (float*)((char*)workspace + harp_two_sided_workspace_bytes(n_out, n_in) / 2);
    // rows of W: w_r <- T_V^T w_r (fp32 out)
    st = run_rows(pv, W, ws1, n_out, ld, n_in, dtype, HARP_F32, HARP_INVERSE, stream);
    if (st != HARP_OK) return st;
    // columns: col <- T_U^T col, in two passes over ws1, the second writing W_out
    if (kernel_choice() != kSimple) {
        st = launch_cols(pu, ws1, n_in, n_in, W_out, ld, dtype, HARP_INVERSE, stream);
        if (st != HARP_ERR_UNSUPPORTED) return st;
        harp_clear_error();
    }
    // otherwise: transpose, rows of W^T, transpose back
    if ((st = launch_transpose(ws1, ws2, n_out, n_in, n_in, n_out, HARP_F32, HARP_F32, stream)) != HARP_OK)
        return st;
    st = run_rows(pu, ws2, ws2, n_in, n_out, n_out, HARP_F32, HARP_F32, HARP_INVERSE, stream);
    if (st != HARP_OK) return st;
    return launch_transpose(ws2, W_out, n_in, n_out, n_out, ld, HARP_F32, dtype, stream);
}
