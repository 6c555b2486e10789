// Calibration backward of the HARP transform (HARP technical summary §2.3 Optimization
// Objective: the parameters are fitted per layer from calibration data, which needs the
// gradient of the fit's loss through the transform).  For rows x_r and upstream gradients
// g_r = dL/dy_r of y_r = T x_r, harp_grad_theta returns dL/dtheta.
//
// Two kernels:
//  1. harp_grad_blocks_kernel: dL/dB_{t,c} = sum_r h_{t+1,r}[group] z_{t,r}[group]^T, with
//     z_t the input of stage t and h_{t+1} the gradient at its output.  A persistent CTA
//     takes tiles of R rows; per tile it holds x and g in shared memory as fp32, runs the
//     stages forward on x (z_m = y), then walks them backwards: in one pass over each
//     group it recovers the stage's input through the transposed block (z_t = B^T z_{t+1},
//     exact up to rounding because B is orthogonal, so no intermediate is stored), adds
//     the outer products h (x) z over the tile's rows, and moves the gradient down
//     (h_t = B^T h_{t+1}).  The tile's sums go to a float accumulator with one atomic
//     add per element (vector atomics where the block is a multiple of 4 floats).
//  2. harp_grad_theta_kernel: one thread per block maps dL/dB to dL/dtheta in double:
//     dL/dQ = dL/dB G^T; Givens: the derivative of the rotation; Cayley: with M = (I-A)^-1
//     and Q = M (I + A), dL/dA = M^T dL/dQ (Q + I)^T and dL/dtheta_k = dL/dA[i][j] -
//     dL/dA[j][i] for the k-th pair i < j.
// The device blocks of stage 0 carry the signs (B_0 diag(S)), so kernel 1 accumulates the
// gradient of those and kernel 2 multiplies column l by the sign of its coordinate.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxTileRows = 16;

struct GradParams {
    PlanDesc pd;
    const float* lanes;                   // lane-interleaved blocks (layout in harp_internal.h)
    int64_t lane_off[HARP_MAX_STAGES];
    const void* x;
    const void* g;
    int64_t rows, ld_x, ld_g;
    float* acc;                           // dL/dB accumulators, stage t at acc + acc_off[t], [c][k][l]
    int64_t acc_off[HARP_MAX_STAGES];
    int R;                                // rows per tile
    int rs;                               // row stride of the shared-memory tiles (floats)
    int64_t ntiles;
    int vec;                              // rows of x and g load as 16-byte vectors
};

// Coordinate i of a row sits at swz(i) in shared memory: bits 0-2 of i XOR bits 3-5, bits 3-4
// XOR bits 6-7.  It permutes each aligned block of 32 coordinates, and the 32 lanes of a
// warp that take 32 consecutive groups of a stage then hit 32 distinct banks for the radix
// 8, 5 and 2 stages of the workload schedules (groups of 8 contiguous coordinates, of 8
// at stride 8, and of any size at stride 64 or more).  An aligned run of 8 coordinates
// stays one aligned run of 8.
__device__ __forceinline__ int swz(int i) { return i ^ ((i >> 3) & 7) ^ (((i >> 6) & 3) << 3); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// The 16 bytes of a vector load as floats (8 bf16 or 4 fp32 values).
__device__ __forceinline__ void unpack(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x), f[1] = __uint_as_float(v.y), f[2] = __uint_as_float(v.z), f[3] = __uint_as_float(v.w);
}

// x and g rows [row0, row0 + nr) into the fp32 tiles.  Each thread keeps several loads in
// flight before it converts and stores them (a load followed directly by its store would
// wait out the memory latency once per element).
template <typename T>
__device__ void load_tile(const GradParams& p, float* A, float* H, int64_t row0, int nr) {
    const int d = (int)p.pd.d, rs = p.rs;
    const T* x = (const T*)p.x;
    const T* g = (const T*)p.g;
    if (p.vec) {
        constexpr int V = 16 / sizeof(T);   // elements per 16-byte load
        constexpr int U = 4;                // vector loads of x (and of g) in flight per thread
        const int cpr = d / V, total = nr * cpr;
        for (int q0 = threadIdx.x; q0 < total; q0 += kThreads * U) {
            uint4 vx[U], vg[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kThreads;
                if (q < total) {
                    const int r = q / cpr, j = q - r * cpr;
                    vx[u] = __ldg(reinterpret_cast<const uint4*>(x + (row0 + r) * p.ld_x) + j);
                    vg[u] = __ldg(reinterpret_cast<const uint4*>(g + (row0 + r) * p.ld_g) + j);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kThreads;
                if (q < total) {
                    const int r = q / cpr, j = q - r * cpr;
                    float fx[V], fg[V];
                    unpack(vx[u], fx);
                    unpack(vg[u], fg);
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        A[r * rs + swz(j * V + e)] = fx[e];
                        H[r * rs + swz(j * V + e)] = fg[e];
                    }
                }
            }
        }
    } else {
        constexpr int U = 8;
        const int total = nr * d;
        for (int q0 = threadIdx.x; q0 < total; q0 += kThreads * U) {
            float fx[U], fg[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kThreads;
                if (q < total) {
                    const int r = q / d, i = q - r * d;
                    fx[u] = to_f32(__ldg(x + (row0 + r) * p.ld_x + i));
                    fg[u] = to_f32(__ldg(g + (row0 + r) * p.ld_g + i));
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kThreads;
                if (q < total) {
                    const int r = q / d, i = q - r * d;
                    A[r * rs + swz(i)] = fx[u];
                    H[r * rs + swz(i)] = fg[u];
                }
            }
        }
    }
}

// Block c of a stage from the lane-interleaved copy: B[k][l] -> w[k * B + l].
template <int B>
__device__ __forceinline__ void load_block(const float* lanes, int64_t c, float (&w)[B * B]) {
    constexpr int BB = B * B;
    const int64_t grp = c >> 5, lane = c & 31;
    if constexpr (BB % 4 == 0) {
        const float4* p = reinterpret_cast<const float4*>(lanes) + grp * (BB / 4) * 32 + lane;
#pragma unroll
        for (int j = 0; j < BB / 4; ++j) {
            const float4 v = __ldg(p + j * 32);
            w[4 * j] = v.x, w[4 * j + 1] = v.y, w[4 * j + 2] = v.z, w[4 * j + 3] = v.w;
        }
    } else {
        const float* p = lanes + grp * BB * 32 + lane;
#pragma unroll
        for (int e = 0; e < BB; ++e) w[e] = __ldg(p + e * 32);
    }
}

// Forward stage t on the activation tile: z <- M_t z.
template <int B>
__device__ void stage_forward(float* A, int nr, int rs, int64_t nb, int s, const float* lanes) {
    for (int64_t c = threadIdx.x; c < nb; c += kThreads) {
        float w[B * B];
        load_block<B>(lanes, c, w);
        const int lo = (int)(c % s), hi = (int)(c / s);
        int off[B];
#pragma unroll
        for (int k = 0; k < B; ++k) off[k] = swz(lo + s * (k + B * hi));
        for (int r = 0; r < nr; ++r) {
            float* a = A + r * rs;
            float xv[B];
#pragma unroll
            for (int l = 0; l < B; ++l) xv[l] = a[off[l]];
#pragma unroll
            for (int k = 0; k < B; ++k) {
                float acc = 0.f;
#pragma unroll
                for (int l = 0; l < B; ++l) acc = fmaf(w[k * B + l], xv[l], acc);
                a[off[k]] = acc;
            }
        }
    }
}

// Backward stage t: with z = z_{t+1} in A and h = h_{t+1} in H, per group and row
//   z_t = B^T z,  dL/dB += h z_t^T,  h_t = B^T h,
// then the tile's sums of this group go to the accumulator.
template <int B>
__device__ void stage_backward(float* A, float* H, int nr, int rs, int64_t nb, int s, const float* lanes,
                               float* acc_t) {
    constexpr int BB = B * B;
    for (int64_t c = threadIdx.x; c < nb; c += kThreads) {
        float w[BB];
        load_block<B>(lanes, c, w);
        const int lo = (int)(c % s), hi = (int)(c / s);
        int off[B];
#pragma unroll
        for (int k = 0; k < B; ++k) off[k] = swz(lo + s * (k + B * hi));
        float sum[BB];
#pragma unroll
        for (int e = 0; e < BB; ++e) sum[e] = 0.f;
        for (int r = 0; r < nr; ++r) {
            float* a = A + r * rs;
            float* h = H + r * rs;
            float zo[B], ho[B];
#pragma unroll
            for (int k = 0; k < B; ++k) zo[k] = a[off[k]], ho[k] = h[off[k]];
#pragma unroll
            for (int l = 0; l < B; ++l) {
                float zi = 0.f, hin = 0.f;
#pragma unroll
                for (int k = 0; k < B; ++k) {
                    zi = fmaf(w[k * B + l], zo[k], zi);
                    hin = fmaf(w[k * B + l], ho[k], hin);
                }
#pragma unroll
                for (int k = 0; k < B; ++k) sum[k * B + l] = fmaf(ho[k], zi, sum[k * B + l]);
                a[off[l]] = zi;
                h[off[l]] = hin;
            }
        }
        float* dst = acc_t + c * BB;
        if constexpr (BB % 4 == 0) {
#pragma unroll
            for (int e = 0; e < BB; e += 4)
                atomicAdd(reinterpret_cast<float4*>(dst + e), make_float4(sum[e], sum[e + 1], sum[e + 2], sum[e + 3]));
        } else {
#pragma unroll
            for (int e = 0; e < BB; ++e) atomicAdd(dst + e, sum[e]);
        }
    }
}

template <bool FWD>
__device__ void run_stage(const GradParams& p, int t, float* A, float* H, int nr) {
    const StageDesc& sd = p.pd.st[t];
    const float* lanes = p.lanes + p.lane_off[t];
    const int s = (int)sd.s;
    const int64_t nb = sd.nblocks;
    float* acc_t = p.acc + p.acc_off[t];
#define HARP_GRAD_CASE(BV)                                                                 \
    case BV:                                                                               \
        if (FWD) stage_forward<BV>(A, nr, p.rs, nb, s, lanes);                             \
        else stage_backward<BV>(A, H, nr, p.rs, nb, s, lanes, acc_t);                      \
        break;
    switch (sd.b) {
        HARP_GRAD_CASE(2)
        HARP_GRAD_CASE(3)
        HARP_GRAD_CASE(4)
        HARP_GRAD_CASE(5)
        HARP_GRAD_CASE(6)
        HARP_GRAD_CASE(7)
        HARP_GRAD_CASE(8)
        default: break;
    }
#undef HARP_GRAD_CASE
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) harp_grad_blocks_kernel(const __grid_constant__ GradParams p) {
    extern __shared__ __align__(16) float smem[];
    float* A = smem;                   // activations [row][swz(i)]
    float* H = smem + p.R * p.rs;      // gradients   [row][swz(i)]
    const int m = p.pd.m;
    for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const int64_t row0 = tile * p.R;
        const int nr = (int)min((int64_t)p.R, p.rows - row0);
        load_tile<T>(p, A, H, row0, nr);
        __syncthreads();
        for (int t = 0; t < m; ++t) run_stage<true>(p, t, A, H, nr);
        for (int t = m - 1; t >= 0; --t) run_stage<false>(p, t, A, H, nr);
    }
}

struct StageOffsets {
    int64_t off[HARP_MAX_STAGES];
};

// dL/dB -> dL/dtheta, one thread per block, in double.
__global__ void harp_grad_theta_kernel(PlanDesc pd, const float* __restrict__ theta_f32,
                                       const int8_t* __restrict__ theta_i8, const float* __restrict__ scales,
                                       const double* __restrict__ mixers, const int8_t* __restrict__ signs,
                                       const float* __restrict__ acc, StageOffsets acc_off,
                                       float* __restrict__ dtheta, int64_t total_blocks) {
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
    const float* pb = acc + acc_off.off[t] + c * b * b;
    const double* gm = mixers + sd.mixer_off;
    // R = dL/dB G^T, with stage 0's sign on column l (the device blocks are B_0 diag(S))
    double R[8][8];
    for (int k = 0; k < b; ++k)
        for (int j = 0; j < b; ++j) {
            double v = 0.0;
            for (int l = 0; l < b; ++l) {
                double pkl = (double)pb[k * b + l];
                if (t == 0 && signs[l + b * c] < 0) pkl = -pkl;
                v += pkl * gm[j * b + l];
            }
            R[k][j] = v;
        }
    float* out = dtheta + poff;
    if (b == 2) {
        const double th = param(0), cs = cos(th), sn = sin(th);
        out[0] = (float)(-R[0][0] * sn - R[0][1] * cs + R[1][0] * cs - R[1][1] * sn);
        return;
    }
    // M = (I - A)^{-1} by Gauss-Jordan without pivoting (every leading principal minor of
    // I - A, A skew, is a product of (1 + lambda^2) > 0), then Q = M (I + A).
    double lhs[8][8], M[8][8], Q[8][8], E[8][8];
    int k = 0;
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) lhs[i][j] = (i == j) ? 1.0 : 0.0, M[i][j] = (i == j) ? 1.0 : 0.0;
    for (int i = 0; i < b; ++i)
        for (int j = i + 1; j < b; ++j, ++k) {
            const double a = param(k);
            lhs[i][j] = -a;
            lhs[j][i] = a;
        }
    for (int col = 0; col < b; ++col) {
        const double inv = 1.0 / lhs[col][col];
        for (int j = 0; j < b; ++j) lhs[col][j] *= inv, M[col][j] *= inv;
        for (int r = 0; r < b; ++r) {
            if (r == col) continue;
            const double f = lhs[r][col];
            if (f == 0.0) continue;
            for (int j = 0; j < b; ++j) lhs[r][j] -= f * lhs[col][j], M[r][j] -= f * M[col][j];
        }
    }
    // I + A = 2 I - (I - A); Q = M (I + A) = 2 M - I
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) Q[i][j] = 2.0 * M[i][j] - (i == j ? 1.0 : 0.0);
    // E = M^T R (Q + I)^T = M^T R (2 M)^T
    double T1[8][8];
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double v = 0.0;
            for (int l = 0; l < b; ++l) v += M[l][i] * R[l][j];
            T1[i][j] = v;
        }
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double v = 0.0;
            for (int l = 0; l < b; ++l) v += T1[i][l] * (Q[j][l] + (j == l ? 1.0 : 0.0));
            E[i][j] = v;
        }
    k = 0;
    for (int i = 0; i < b; ++i)
        for (int j = i + 1; j < b; ++j, ++k) out[k] = (float)(E[i][j] - E[j][i]);
}

int sms_of_current_device() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 1;
    }
    return n;
}

// Accumulator layout: per stage nblocks * b * b floats, each stage starting on a 16-byte
// boundary (vector atomics).
struct AccLayout {
    StageOffsets off = {};
    int64_t floats = 0;          // accumulator floats
    size_t bytes = 0;            // workspace bytes
};

AccLayout acc_layout(const PlanDesc& pd) {
    AccLayout L;
    int64_t off = 0;
    for (int t = 0; t < pd.m; ++t) {
        L.off.off[t] = off;
        off += (pd.st[t].nblocks * pd.st[t].b * pd.st[t].b + 3) / 4 * 4;
    }
    L.floats = off;
    L.bytes = (size_t)off * 4;
    return L;
}

}  // namespace

extern "C" size_t harp_grad_workspace_bytes(harp_plan_t p) {
    if (!p) return 0;
    return acc_layout(p->desc).bytes;
}

extern "C" harp_status harp_grad_theta(harp_plan_t p, const void* x, const void* g, int64_t rows, int64_t ld_x,
                                       int64_t ld_g, harp_dtype dtype, float* dtheta, void* workspace,
                                       size_t ws_bytes, void* stream) {
    harp_clear_error();
    if (!p) return harp_fail(HARP_ERR_INVALID_ARG, "plan is NULL");
    if (dtype != HARP_F32 && dtype != HARP_BF16) return harp_fail(HARP_ERR_UNSUPPORTED, "unknown dtype");
    if (rows < 0) return harp_fail(HARP_ERR_INVALID_ARG, "rows < 0");
    const PlanDesc& pd = p->desc;
    const int64_t d = pd.d;
    if (ld_x < d || ld_g < d) return harp_fail(HARP_ERR_INVALID_ARG, "leading dimension smaller than d");
    if (!dtheta) return harp_fail(HARP_ERR_INVALID_ARG, "dtheta is NULL");
    if (p->composite) return harp_fail(HARP_ERR_UNSUPPORTED, "the gradient is taken for one plan, not a composite");
    {
        const harp_status mst = harp_require_materialized(p, stream);
        if (mst != HARP_OK) return mst;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no CUDA device");
    }
    if (dev != p->device) return harp_fail(HARP_ERR_WRONG_DEVICE, "plan materialized on another device");
    for (int t = 0; t < pd.m; ++t)
        if (pd.st[t].b > 8) return harp_fail(HARP_ERR_UNSUPPORTED, "the gradient kernel takes radices up to 8");
    const AccLayout L = acc_layout(pd);
    if (!workspace || ws_bytes < L.bytes)
        return harp_fail(HARP_ERR_INVALID_ARG, "workspace smaller than harp_grad_workspace_bytes()");
    if (((uintptr_t)workspace & 15) != 0) return harp_fail(HARP_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    if (rows > 0 && (!x || !g)) return harp_fail(HARP_ERR_INVALID_ARG, "x or g is NULL");
    {
        // the accumulators are zeroed and then added to while x and g are read, and dtheta is
        // written last: none of them may share memory with another
        const size_t es = dtype == HARP_F32 ? 4 : 2;
        const size_t xb = rows > 0 ? ((size_t)(rows - 1) * ld_x + d) * es : 0;
        const size_t gb = rows > 0 ? ((size_t)(rows - 1) * ld_g + d) * es : 0;
        const size_t tb = (size_t)p->theta_total * sizeof(float);
        if (rows > 0 && (ranges_overlap(workspace, ws_bytes, x, xb) || ranges_overlap(workspace, ws_bytes, g, gb)))
            return harp_fail(HARP_ERR_INVALID_ARG, "workspace overlaps x or g");
        if (ranges_overlap(dtheta, tb, workspace, ws_bytes) ||
            (rows > 0 && (ranges_overlap(dtheta, tb, x, xb) || ranges_overlap(dtheta, tb, g, gb))))
            return harp_fail(HARP_ERR_INVALID_ARG, "dtheta overlaps the workspace, x or g");
    }
    // rows per tile: two fp32 tiles of rows rounded up to 32 coordinates (the swizzle
    // permutes aligned blocks of 32) within the 227 KiB of shared memory a CTA may use
    const int rs = (int)((d + 31) / 32 * 32);
    const int64_t per_row = 2 * (int64_t)rs * 4;
    const int64_t budget = 227 * 1024;
    const int R = (int)std::min<int64_t>(kMaxTileRows, budget / per_row);
    if (R < 1) return harp_fail(HARP_ERR_UNSUPPORTED, "a row is too long for the gradient kernel's tile");

    cudaStream_t s = (cudaStream_t)stream;
    float* acc = (float*)workspace;
    cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)L.floats * 4, s);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    if (rows > 0) {
        GradParams gp;
        gp.pd = pd;
        gp.lanes = p->d_blocks_lanes;
        for (int t = 0; t < HARP_MAX_STAGES; ++t) gp.lane_off[t] = p->lane_off[t], gp.acc_off[t] = L.off.off[t];
        gp.x = x;
        gp.g = g;
        gp.rows = rows;
        gp.ld_x = ld_x;
        gp.ld_g = ld_g;
        gp.acc = acc;
        gp.R = R;
        gp.rs = rs;
        gp.ntiles = (rows + R - 1) / R;
        const size_t es = dtype == HARP_F32 ? 4 : 2;
        gp.vec = ((uintptr_t)x % 16 == 0) && ((uintptr_t)g % 16 == 0) && (ld_x * es) % 16 == 0 &&
                 (ld_g * es) % 16 == 0 && (d * es) % 16 == 0;
        const size_t smem = (size_t)R * per_row;
        const int grid = (int)std::min<int64_t>(gp.ntiles, sms_of_current_device());
        if (dtype == HARP_BF16) {
            e = (cudaError_t)harp_set_smem_limit((const void*)harp_grad_blocks_kernel<__nv_bfloat16>, (int)smem);
            if (e == cudaSuccess) harp_grad_blocks_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(gp);
        } else {
            e = (cudaError_t)harp_set_smem_limit((const void*)harp_grad_blocks_kernel<float>, (int)smem);
            if (e == cudaSuccess) harp_grad_blocks_kernel<float><<<grid, kThreads, smem, s>>>(gp);
        }
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    int64_t total = 0;
    for (int t = 0; t < pd.m; ++t) total += pd.st[t].nblocks;
    const bool i8 = p->kind == HARP_THETA_I8;
    harp_grad_theta_kernel<<<(unsigned)((total + 127) / 128), 128, 0, s>>>(
        pd, i8 ? nullptr : (const float*)p->d_theta, i8 ? (const int8_t*)p->d_theta : nullptr, p->d_scales,
        p->d_mixers, p->d_signs, acc, L.off, dtheta, total);
    e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_grad_blocks_kernel");
    return HARP_OK;
}
