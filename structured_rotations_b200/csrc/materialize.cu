// Block construction on the device (HARP technical summary §2.2 Hadamard
// Preconditioning; §2.4 int8 storage): one thread per block computes
//   Q = Givens(theta)                     (b = 2)
//   Q = (I - A)^{-1} (I + A), A skew       (b > 2, Cayley map)
//   B = Q G_b, with stage 0's columns multiplied by the sign diagonal S,
// in double, and stores B as float32.  int8 parameters are dequantized here
// (q * scale_t), so theta stays in its storage form until this kernel.
#include <mutex>

#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

__global__ void materialize_kernel(PlanDesc pd, const float* __restrict__ theta_f32,
                                   const int8_t* __restrict__ theta_i8,
                                   const float* __restrict__ scales,
                                   const double* __restrict__ mixers,
                                   const int8_t* __restrict__ signs, float* __restrict__ blocks,
                                   int64_t total_blocks) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= total_blocks) return;
    int t = 0;
    int64_t c = gid;
    while (t < pd.m - 1 && c >= pd.st[t].nblocks) {
        c -= pd.st[t].nblocks;
        ++t;
    }
    const StageDesc sd = pd.st[t];
    const int b = sd.b;
    const int64_t poff = sd.theta_off + c * sd.p;
    const double scale = theta_i8 ? (double)scales[t] : 1.0;
    auto param = [&](int k) -> double {
        return theta_i8 ? (double)theta_i8[poff + k] * scale : (double)theta_f32[poff + k];
    };

    double q[HARP_MAX_RADIX][HARP_MAX_RADIX];
    if (b == 2) {
        const double th = param(0);
        const double cs = cos(th), sn = sin(th);
        q[0][0] = cs; q[0][1] = -sn;
        q[1][0] = sn; q[1][1] = cs;
    } else {
        // Augmented system [I - A | I + A]; Gaussian elimination without pivoting
        // (every leading principal minor of I - A is prod(1 + lambda^2) > 0).
        double lhs[HARP_MAX_RADIX][HARP_MAX_RADIX];
        for (int i = 0; i < b; ++i)
            for (int j = 0; j < b; ++j) {
                lhs[i][j] = (i == j) ? 1.0 : 0.0;
                q[i][j] = (i == j) ? 1.0 : 0.0;
            }
        int k = 0;
        for (int i = 0; i < b; ++i)
            for (int j = i + 1; j < b; ++j, ++k) {
                const double a = param(k);
                lhs[i][j] = -a;  lhs[j][i] = a;     // I - A
                q[i][j] = a;     q[j][i] = -a;      // I + A
            }
        for (int col = 0; col < b; ++col) {
            const double inv = 1.0 / lhs[col][col];
            for (int r = col + 1; r < b; ++r) {
                const double f = lhs[r][col] * inv;
                if (f == 0.0) continue;
                for (int j = col; j < b; ++j) lhs[r][j] -= f * lhs[col][j];
                for (int j = 0; j < b; ++j) q[r][j] -= f * q[col][j];
            }
        }
        for (int r = b - 1; r >= 0; --r) {
            for (int j = 0; j < b; ++j) {
                double acc = q[r][j];
                for (int kk = r + 1; kk < b; ++kk) acc -= lhs[r][kk] * q[kk][j];
                q[r][j] = acc / lhs[r][r];
            }
        }
    }

    const double* g = mixers + sd.mixer_off;
    float* out = blocks + sd.block_off + c * b * b;
    for (int k = 0; k < b; ++k) {
        for (int l = 0; l < b; ++l) {
            double acc = 0.0;
            for (int j = 0; j < b; ++j) acc += q[k][j] * g[j * b + l];
            // stage 0 has stride 1, so input l of block c is coordinate l + b*c
            if (t == 0 && signs[l + b * c] < 0) acc = -acc;
            out[k * b + l] = (float)acc;
        }
    }
}

// Blocks of one stage -> the lane-interleaved layout described in harp_internal.h.
__global__ void interleave_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t nb, int bb) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= nb * bb) return;
    const int64_t c = idx / bb;
    const int e = (int)(idx - c * bb);
    const int64_t group = c >> 5, lane = c & 31;
    int64_t to;
    if (bb % 4 == 0) to = ((group * (bb / 4) + e / 4) * 32 + lane) * 4 + (e & 3);
    else to = (group * bb + e) * 32 + lane;
    dst[to] = src[idx];
}

template <typename T>
harp_status dev_alloc_copy(T** dst, const T* src, size_t n, cudaStream_t stream) {
    if (*dst == nullptr) {
        if (cudaMalloc((void**)dst, sizeof(T) * (n ? n : 1)) != cudaSuccess) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_ALLOC, "cudaMalloc failed");
        }
    }
    if (n && cudaMemcpyAsync(*dst, src, sizeof(T) * n, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(cudaGetLastError()));
    return HARP_OK;
}

}  // namespace

harp_status harp_device_free(harp_plan_s* p) {
    if (p->device < 0) return HARP_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(p->device);
    cudaDeviceSynchronize();
    fast_state_free(p);
    cluster_state_free(p);
    host_io_free(p);
    cudaFree(p->d_blocks);
    cudaFree(p->d_blocks_lanes);
    cudaFree(p->d_theta);
    cudaFree(p->d_scales);
    cudaFree(p->d_mixers);
    cudaFree(p->d_signs);
    cudaFree(p->d_status);
    p->d_blocks = nullptr; p->d_blocks_lanes = nullptr; p->d_theta = nullptr; p->d_scales = nullptr;
    p->d_mixers = nullptr; p->d_signs = nullptr; p->d_status = nullptr;
    p->materialized = false;
    p->device = -1;
    cudaSetDevice(prev);
    return cudaGetLastError() == cudaSuccess ? HARP_OK : HARP_ERR_CUDA;
}

namespace {

// Uploads and builds everything on `stream_`; the caller holds the plan's materialize_mu
// and sets p->materialized afterwards.
harp_status materialize_locked(harp_plan_s* p, void* stream_) {
    cudaStream_t stream = (cudaStream_t)stream_;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (p->device >= 0 && p->device != dev)
        return harp_fail(HARP_ERR_WRONG_DEVICE, "plan materialized on device " + std::to_string(p->device));
    if (p->materialized) return HARP_OK;
    p->device = dev;

    harp_status st;
    if ((st = dev_alloc_copy(&p->d_signs, p->signs.data(), p->signs.size(), stream)) != HARP_OK) return st;
    if ((st = dev_alloc_copy(&p->d_mixers, p->mixers.data(), p->mixers.size(), stream)) != HARP_OK) return st;
    if ((st = dev_alloc_copy(&p->d_scales, p->scales.data(), p->scales.size(), stream)) != HARP_OK) return st;
    if (p->kind == HARP_THETA_F32) {
        float* th = (float*)p->d_theta;
        if ((st = dev_alloc_copy(&th, p->theta_f32.data(), p->theta_f32.size(), stream)) != HARP_OK) return st;
        p->d_theta = th;
    } else {
        int8_t* th = (int8_t*)p->d_theta;
        if ((st = dev_alloc_copy(&th, p->theta_i8.data(), p->theta_i8.size(), stream)) != HARP_OK) return st;
        p->d_theta = th;
    }
    if (!p->d_blocks && cudaMalloc((void**)&p->d_blocks, sizeof(float) * p->block_floats) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the blocks failed");
    }
    if (!p->d_blocks_lanes) {
        if (cudaMalloc((void**)&p->d_blocks_lanes, sizeof(float) * p->lane_floats) != cudaSuccess) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the interleaved blocks failed");
        }
        cudaMemsetAsync(p->d_blocks_lanes, 0, sizeof(float) * p->lane_floats, stream);
    }
    if (!p->d_status) {
        if (cudaMalloc((void**)&p->d_status, 64) != cudaSuccess) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the status word failed");
        }
        cudaMemsetAsync(p->d_status, 0, 64, stream);
    }

    int64_t total = 0;
    for (int t = 0; t < p->desc.m; ++t) total += p->desc.st[t].nblocks;
    const int threads = 128;
    const int64_t grid = (total + threads - 1) / threads;
    materialize_kernel<<<(unsigned)grid, threads, 0, stream>>>(
        p->desc, p->kind == HARP_THETA_F32 ? (const float*)p->d_theta : nullptr,
        p->kind == HARP_THETA_I8 ? (const int8_t*)p->d_theta : nullptr, p->d_scales, p->d_mixers,
        p->d_signs, p->d_blocks, total);
    for (int t = 0; t < p->desc.m; ++t) {
        const StageDesc& sd = p->desc.st[t];
        const int64_t n = sd.nblocks * sd.b * sd.b;
        interleave_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
            p->d_blocks + sd.block_off, p->d_blocks_lanes + p->lane_off[t], sd.nblocks, sd.b * sd.b);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    fast_prepare(p, stream);      // the specialized kernel's table, so that launches only read plan state
    cluster_prepare(p, stream);   // the cluster kernel's split and table
    e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    return HARP_OK;
}

}  // namespace

extern "C" harp_status harp_materialize_blocks(harp_plan_t p, void* stream) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    std::lock_guard<std::mutex> lock(p->materialize_mu);
    const harp_status st = materialize_locked(p, stream);
    if (st == HARP_OK) p->materialized = true;
    return st;
}

harp_status harp_require_materialized(harp_plan_s* p, void* stream) {
    if (p->materialized) return HARP_OK;
    if (p->kind != HARP_THETA_I8)
        return harp_fail(HARP_ERR_NOT_MATERIALIZED, "call harp_materialize_blocks first");
    std::lock_guard<std::mutex> lock(p->materialize_mu);
    if (p->materialized) return HARP_OK;   // another call got there first (and synchronized)
    harp_status st = materialize_locked(p, stream);
    if (st != HARP_OK) return st;
    const cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    p->materialized = true;
    return HARP_OK;
}



extern "C" harp_status harp_plan_device_status(harp_plan_t p) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (!p->materialized || !p->d_status) return harp_fail(HARP_ERR_NOT_MATERIALIZED, "plan not materialized");
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(p->device);
    int flag = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&flag, p->d_status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && flag) e = cudaMemset(p->d_status, 0, sizeof(int));
    cudaSetDevice(prev);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    if (flag) return harp_fail(HARP_ERR_TIMEOUT, "a bounded device wait gave up");
    return HARP_OK;
}
