// General fast row kernel for the HARP transform (HARP technical summary §2.1 Core
// Architecture): any schedule whose radices are 2..8, d a multiple of 8, forward or
// inverse, fp32 or bf16 rows with 16-byte aligned rows.  Device code; the host
// launcher is apply_tiled.cu.
//
// One persistent CTA per SM owns a tile of R rows and keeps them in shared memory as
// fp32 across all m stages, so HBM is read once and written once.  While the stages
// of tile k run, the bulk-copy engine (cp.async.bulk, completed on an mbarrier)
// brings the raw rows of the CTA's next tile into a staging area, so loads overlap
// the arithmetic.
//
// Stage t: each thread takes whole groups {lo + s_t (k + b_t hi)} (block c = lo +
// s_t hi), holds the block B_{t,c} (b_t x b_t fp32, plain FMA arithmetic) in
// registers and applies it to every row of the tile, so a block is fetched from L2
// once per tile rather than once per row; the next block's coefficients are loaded
// while the current one is applied.  The inverse runs the stages backwards with
// B^T (the signs S are folded into stage 0's blocks, so B_0^T also applies S last).
//
// Shared-memory layout of a row: element i lives at word i ^ ((i >> 3) & 0x18)
// (bits 6-7 of i XORed into bits 3-4; identity if d is not a multiple of 32).
//  - stride 1 (stage 0 of a radix-8 schedule): a thread reads 8 consecutive words,
//    the XOR keeps 8-aligned runs contiguous, so two 16-byte accesses per row.
//  - stride 8: lanes c = lo + 8 hi read lo + 8k + 64 hi; the four lanes sharing lo
//    have four different hi & 3, so the XOR puts them in four different banks.
//  - stride >= 32: 32 consecutive lo per warp, one bank each.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace harp_tiled {

constexpr int kThreads = 256;
constexpr int kMaxTileRows = 32;
constexpr int kSmemOptIn = 227 * 1024;
constexpr long long kWaitLimit = 1ll << 26;   // mbarrier polls before giving up

struct TiledParams {
    PlanDesc pd;
    const float* blocks;
    const void* x;
    void* y;
    int64_t rows, ld_x, ld_y;   // in elements
    int64_t ntiles;
    int R;                      // rows per tile
    int staged;                 // 1: rows of the next tile arrive by bulk copy
    int swz;                    // 0x18 when d % 32 == 0, else 0
    int* status;
};

// ----------------------------------------------------------------- PTX ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait for the phase with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    for (long long i = 0; i < kWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
            "selp.u32 %0, 1, 0, p; }"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Global -> this CTA's shared memory, completed on the mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------ helpers ---

__device__ __forceinline__ int swz(int i, int mask) { return i ^ ((i >> 3) & mask); }

// 8 consecutive elements <-> 8 floats
__device__ __forceinline__ void load8(const float* src, float (&v)[8]) {
    const float4 a = *(const float4*)src, b = *(const float4*)(src + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&v)[8]) {
    const uint4 u = *(const uint4*)src;
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        v[2 * q] = __uint_as_float(w[q] << 16);
        v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
    }
}
__device__ __forceinline__ void store8(float* dst, const float (&v)[8]) {
    *(float4*)dst = make_float4(v[0], v[1], v[2], v[3]);
    *(float4*)(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
        w[q] = *(const uint32_t*)&h;
    }
    *(uint4*)dst = make_uint4(w[0], w[1], w[2], w[3]);
}

// Block B_{t,c}: b*b floats, row-major [output k][input l].
template <int B>
__device__ __forceinline__ void load_block(float (&w)[B * B], const float* __restrict__ src, bool vec) {
    if constexpr ((B * B) % 4 == 0) {
        if (vec) {
#pragma unroll
            for (int q = 0; q < B * B / 4; ++q) {
                const float4 v = __ldg((const float4*)src + q);
                w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
            }
            return;
        }
    }
#pragma unroll
    for (int q = 0; q < B * B; ++q) w[q] = __ldg(src + q);
}

// One group of one row: y = B x (forward) or y = B^T x (inverse), in place.
template <int B, bool INV>
__device__ __forceinline__ void group_row(float* __restrict__ row, const int (&pos)[B], bool contig,
                                          const float (&w)[B * B]) {
    float xv[B];
    if constexpr (B % 4 == 0) {
        if (contig) {
#pragma unroll
            for (int q = 0; q < B / 4; ++q) {
                const float4 v = *(const float4*)(row + pos[4 * q]);
                xv[4 * q] = v.x; xv[4 * q + 1] = v.y; xv[4 * q + 2] = v.z; xv[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int l = 0; l < B; ++l) xv[l] = row[pos[l]];
        }
    } else {
#pragma unroll
        for (int l = 0; l < B; ++l) xv[l] = row[pos[l]];
    }
    float yv[B];
#pragma unroll
    for (int k = 0; k < B; ++k) {
        float acc = 0.0f;
#pragma unroll
        for (int l = 0; l < B; ++l) acc = fmaf(INV ? w[l * B + k] : w[k * B + l], xv[l], acc);
        yv[k] = acc;
    }
    if constexpr (B % 4 == 0) {
        if (contig) {
#pragma unroll
            for (int q = 0; q < B / 4; ++q)
                *(float4*)(row + pos[4 * q]) = make_float4(yv[4 * q], yv[4 * q + 1], yv[4 * q + 2], yv[4 * q + 3]);
            return;
        }
    }
#pragma unroll
    for (int k = 0; k < B; ++k) row[pos[k]] = yv[k];
}

// Item = (block c, row group g): the rows g, g + G, ... of the tile.
template <int B, bool INV>
__device__ __forceinline__ void apply_item(float* data, int d, int nr, int G, int nb, int s, int swzmask,
                                           int item, const float (&w)[B * B]) {
    const int c = item % nb;
    const int g = item / nb;
    const int lo = c % s, hi = c / s;
    const int base = lo + s * B * hi;
    int pos[B];
#pragma unroll
    for (int k = 0; k < B; ++k) pos[k] = swz(base + s * k, swzmask);
    const bool contig = (s == 1);
    for (int r = g; r < nr; r += G) group_row<B, INV>(data + r * d, pos, contig, w);
}

// All items of one stage; the coefficients of the thread's next item are loaded while
// the current one is applied.
template <int B, bool INV>
__device__ __forceinline__ void run_stage(const StageDesc& sd, const float* __restrict__ blocks, float* data,
                                          int d, int nr, int swzmask) {
    const int nb = d / B;
    const int s = (int)sd.s;
    // Row groups: enough items to keep every thread busy, evenly spread.
    int G = 1;
    while (G < nr && G < 8) {
        const int items = nb * G;
        const int per = (items + kThreads - 1) / kThreads;
        if (per * kThreads <= items + items / 8) break;   // >= ~89% of the threads' slots used
        ++G;
    }
    const int items = nb * G;
    const float* sb = blocks + sd.block_off;
    const bool vec = (sd.block_off & 3) == 0;
    int j = threadIdx.x;
    if (j >= items) return;
    float wa[B * B], wb[B * B];
    load_block<B>(wa, sb + (j % nb) * (B * B), vec);
    while (true) {
        int jn = j + kThreads;
        if (jn < items) load_block<B>(wb, sb + (jn % nb) * (B * B), vec);
        apply_item<B, INV>(data, d, nr, G, nb, s, swzmask, j, wa);
        if (jn >= items) break;
        j = jn;
        jn = j + kThreads;
        if (jn < items) load_block<B>(wa, sb + (jn % nb) * (B * B), vec);
        apply_item<B, INV>(data, d, nr, G, nb, s, swzmask, j, wb);
        if (jn >= items) break;
        j = jn;
    }
}

template <typename TIn>
__device__ __forceinline__ void issue_tile(const TiledParams& p, int64_t tile, unsigned char* stage_buf,
                                           uint64_t* bar) {
    const int d = (int)p.pd.d;
    const int64_t row0 = tile * p.R;
    const int nr = (int)min((int64_t)p.R, p.rows - row0);
    const uint32_t row_bytes = (uint32_t)d * sizeof(TIn);
    mbar_arrive_expect_tx(bar, row_bytes * nr);
    const TIn* x = (const TIn*)p.x;
    for (int r = 0; r < nr; ++r) bulk_load(stage_buf + (size_t)r * row_bytes, x + (row0 + r) * p.ld_x, row_bytes, bar);
}

template <typename TIn, typename TOut, bool INV, int MASK>
__global__ void __launch_bounds__(kThreads, 1) harp_tiled_kernel(const __grid_constant__ TiledParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int d = (int)p.pd.d;
    const int R = p.R;
    const int tid = threadIdx.x;
    const int d8 = d / 8;
    float* data = (float*)smem;
    unsigned char* stage_buf = smem + (size_t)R * d * sizeof(float);
    uint64_t* bar = (uint64_t*)(stage_buf + (p.staged ? (size_t)R * d * sizeof(TIn) : 0));

    int64_t tile = blockIdx.x;
    if (tile >= p.ntiles) return;
    if (p.staged) {
        if (tid == 0) mbar_init(bar, 1);
        __syncthreads();
        if (tid == 0) issue_tile<TIn>(p, tile, stage_buf, bar);
    }
    uint32_t parity = 0;
    for (; tile < p.ntiles; tile += gridDim.x) {
        const int64_t row0 = tile * R;
        const int nr = (int)min((int64_t)R, p.rows - row0);
        // rows -> fp32 tile
        if (p.staged) {
            const bool ok = mbar_wait(bar, parity);
            parity ^= 1;
            if (__syncthreads_or(!ok)) {
                if (tid == 0) atomicExch(p.status, 1);
                return;
            }
            const TIn* src = (const TIn*)stage_buf;
            for (int r = 0; r < nr; ++r)
                for (int j = tid; j < d8; j += kThreads) {
                    float v[8];
                    load8(src + (size_t)r * d + 8 * j, v);
                    store8(data + r * d + swz(8 * j, p.swz), v);
                }
        } else {
            const TIn* x = (const TIn*)p.x;
            for (int r = 0; r < nr; ++r)
                for (int j = tid; j < d8; j += kThreads) {
                    float v[8];
                    load8(x + (row0 + r) * p.ld_x + 8 * j, v);
                    store8(data + r * d + swz(8 * j, p.swz), v);
                }
        }
        __syncthreads();
        if (p.staged && tid == 0 && tile + gridDim.x < p.ntiles) {
            fence_proxy_async_smem();   // the staging reads above happen before the copies' writes
            issue_tile<TIn>(p, tile + gridDim.x, stage_buf, bar);
        }
        for (int step = 0; step < p.pd.m; ++step) {
            const int t = INV ? p.pd.m - 1 - step : step;
            const StageDesc& sd = p.pd.st[t];
            switch (sd.b) {
#define HARP_TILED_CASE(R)                                                         \
    case R:                                                                        \
        if constexpr ((MASK >> R) & 1) run_stage<R, INV>(sd, p.blocks, data, d, nr, p.swz); \
        break;
                HARP_TILED_CASE(2) HARP_TILED_CASE(3) HARP_TILED_CASE(4) HARP_TILED_CASE(5)
                HARP_TILED_CASE(6) HARP_TILED_CASE(7) HARP_TILED_CASE(8)
#undef HARP_TILED_CASE
                default: break;
            }
            __syncthreads();
        }
        TOut* y = (TOut*)p.y;
        for (int r = 0; r < nr; ++r)
            for (int j = tid; j < d8; j += kThreads) {
                float v[8];
                load8(data + r * d + swz(8 * j, p.swz), v);
                store8(y + (row0 + r) * p.ld_y + 8 * j, v);
            }
        __syncthreads();
    }
}

// Radix sets with their own kernel: a kernel that instantiates every radix needs more
// registers than any single one, so the common schedules get kernels with only the
// radices they use.  The last entry (all of 2..8) covers every other schedule.
constexpr int kMasks[] = {1 << 8, (1 << 2) | (1 << 8), (1 << 2) | (1 << 5) | (1 << 8), (1 << 7) | (1 << 8),
                          (1 << 2) | (1 << 7) | (1 << 8), 0x1fc};
constexpr int kNumMasks = sizeof(kMasks) / sizeof(kMasks[0]);

template <typename TIn, typename TOut, bool INV, int I>
cudaError_t launch_mask(int which, const TiledParams& tp, size_t smem, int grid, cudaStream_t stream) {
    if constexpr (I < kNumMasks) {
        if (which != I) return launch_mask<TIn, TOut, INV, I + 1>(which, tp, smem, grid, stream);
        auto kern = harp_tiled_kernel<TIn, TOut, INV, kMasks[I]>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)grid, kThreads, smem, stream>>>(tp);
        return cudaGetLastError();
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename TIn, typename TOut>
cudaError_t launch(int which, bool inverse, const TiledParams& tp, size_t smem, int grid, cudaStream_t stream) {
    return inverse ? launch_mask<TIn, TOut, true, 0>(which, tp, smem, grid, stream)
                   : launch_mask<TIn, TOut, false, 0>(which, tp, smem, grid, stream);
}

}  // namespace harp_tiled

// One translation unit per I/O type pair (compiled in parallel).
cudaError_t harp_tiled_launch_bf16(int which, bool inverse, const harp_tiled::TiledParams& tp, size_t smem,
                                   int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_f32(int which, bool inverse, const harp_tiled::TiledParams& tp, size_t smem,
                                  int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_bf16_f32(int which, bool inverse, const harp_tiled::TiledParams& tp, size_t smem,
                                       int grid, cudaStream_t stream);
