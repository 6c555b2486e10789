// General fast row kernel for the HARP transform (HARP technical summary §2.1 Core
// Architecture): any schedule whose radices are 2..8, d a multiple of 8, forward or
// inverse, fp32 or bf16 rows with 16-byte aligned rows.  Device code; the host
// launcher is apply_tiled.cu.
//
// One persistent CTA per SM owns a tile of R rows and keeps them in shared memory as
// fp32 across all m stages, so HBM is read once and written once.  While the stages
// of tile k run, the bulk-copy engine (cp.async.bulk, completed on an mbarrier)
// brings the raw rows of the CTA's next tile into a staging area, so loads overlap
// the arithmetic (when the staging area fits next to the tile).
//
// Stage t: each thread takes whole groups {lo + s_t (k + b_t hi)} (block c = lo +
// s_t hi), holds the block B_{t,c} (b_t x b_t fp32, plain FMA arithmetic) in
// registers and applies it to every row of the tile, so a block is fetched from L2
// once per tile rather than once per row; the next block's coefficients are loaded
// while the current one is applied.  The inverse runs the stages backwards with
// B^T (the signs S are folded into stage 0's blocks, so B_0^T also applies S last).
//
// Shared-memory layout: the tile is a stack of sub-tiles of V = 4 rows; inside one,
// coordinate i holds the 4 rows' values as one 16-byte quad at quad index
// slot(i) = i ^ ((i >> 3) & 7).  A thread therefore moves 4 rows with one 16-byte access
// and keeps 4 independent accumulators per output.  The XOR spreads the quads a warp
// touches over the 8 bank groups a quarter-warp's 16-byte accesses need:
//  - stride 1 (lanes c read 8c + k): quad index mod 8 = k ^ (c & 7), 8 distinct;
//  - stride 8 (lanes c = lo + 8 hi read lo + 8k + 64 hi): mod 8 = lo ^ k, 8 distinct;
//  - stride >= 64 (consecutive lo): 8 consecutive quads permuted, 8 distinct.
// When even one 4-row sub-tile of fp32 does not fit (d > 14524), sub-tiles are single
// rows (V = 1) with word index i ^ ((i >> 3) & 0x18).
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
    const float* lanes;                      // lane-interleaved blocks
    int64_t lane_off[HARP_MAX_STAGES];       // per stage, in floats
    const void* x;
    void* y;
    int64_t rows, ld_x, ld_y;   // in elements
    int64_t ntiles;
    int R;                      // rows per tile (a multiple of the sub-tile height V)
    int staged_rows;            // the first rows of the next tile that arrive by bulk copy
    int mask;                   // V = 1 swizzle: 0x18 when d % 32 == 0, else 0
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

// Vector of the V rows of one sub-tile at one coordinate.
template <int V> struct VecOf;
template <> struct VecOf<4> { using T = float4; };
template <> struct VecOf<1> { using T = float; };

// Position of coordinate i inside a sub-tile, in units of VecOf<V> (layout notes above).
template <int V>
__device__ __forceinline__ int slot(int i, int mask) {
    if constexpr (V == 4) return i ^ ((i >> 3) & 7);
    else return i ^ ((i >> 3) & mask);
}

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

// Block B_{t,c} (b*b floats, row-major [output k][input l]) from the stage's
// lane-interleaved copy: lanes holding 32 consecutive c read contiguous memory.  The
// buffer holds the largest block (8 x 8); a radix-b stage uses its first b*b entries.
template <int B>
__device__ __forceinline__ void load_block(float (&w)[64], const float* __restrict__ stage, int c) {
    const int group = c >> 5, lane = c & 31;
    if constexpr ((B * B) % 4 == 0) {
        const float4* src = (const float4*)stage + (size_t)group * (B * B / 4) * 32 + lane;
#pragma unroll
        for (int q = 0; q < B * B / 4; ++q) {
            const float4 v = __ldg(src + q * 32);
            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
        }
    } else {
        const float* src = stage + (size_t)group * (B * B) * 32 + lane;
#pragma unroll
        for (int e = 0; e < B * B; ++e) w[e] = __ldg(src + e * 32);
    }
}

// The same for a radix known only at run time (the first block of the next stage).
__device__ __forceinline__ void load_block_any(float (&w)[64], const float* __restrict__ stage, int c, int bb) {
    const int group = c >> 5, lane = c & 31;
    if ((bb & 3) == 0) {
        const float4* src = (const float4*)stage + (size_t)group * (bb / 4) * 32 + lane;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (4 * q < bb) {
                const float4 v = __ldg(src + q * 32);
                w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
            }
        }
    } else {
        const float* src = stage + (size_t)group * bb * 32 + lane;
#pragma unroll
        for (int e = 0; e < 64; ++e)
            if (e < bb) w[e] = __ldg(src + e * 32);
    }
}

__device__ __forceinline__ void fma_v(float4& acc, float w, const float4& x) {
    acc.x = fmaf(w, x.x, acc.x);
    acc.y = fmaf(w, x.y, acc.y);
    acc.z = fmaf(w, x.z, acc.z);
    acc.w = fmaf(w, x.w, acc.w);
}
__device__ __forceinline__ void fma_v(float& acc, float w, const float& x) { acc = fmaf(w, x, acc); }
__device__ __forceinline__ void zero_v(float4& v) { v = make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ void zero_v(float& v) { v = 0.f; }

// One group in one sub-tile (V rows at once): y = B x (forward) or B^T x (inverse), in
// place.  Each output is summed as fma(B[k][l], x_l, acc) over l = 0..b-1 from zero.
template <int B, bool INV, typename VT>
__device__ __forceinline__ void group_vec(VT* __restrict__ st, const int (&pos)[B], const float (&w)[64]) {
    VT xv[B];
#pragma unroll
    for (int l = 0; l < B; ++l) xv[l] = st[pos[l]];
    // l outer, k inner: consecutive FMAs update different outputs, so dependent FMAs are
    // 4 B instructions apart; every output still sums over l = 0..b-1 in order.
    VT yv[B];
#pragma unroll
    for (int k = 0; k < B; ++k) zero_v(yv[k]);
#pragma unroll
    for (int l = 0; l < B; ++l)
#pragma unroll
        for (int k = 0; k < B; ++k) fma_v(yv[k], INV ? w[l * B + k] : w[k * B + l], xv[l]);
#pragma unroll
    for (int k = 0; k < B; ++k) st[pos[k]] = yv[k];
}

// Item = (block c, sub-tile group g): the sub-tiles g, g + G, ... of the tile; block c
// has lo = c % s, hi = c / s.  The caller steps (c, g, lo, hi) from item to item.
struct ItemPos {
    int c, g, lo, hi;
};

template <int B, bool INV, int V>
__device__ __forceinline__ void apply_item(typename VecOf<V>::T* tile, int d, int qv, int G, int s, int mask,
                                           const ItemPos& it, const float (&w)[64]) {
    const int base = it.lo + s * B * it.hi;
    int pos[B];
#pragma unroll
    for (int k = 0; k < B; ++k) pos[k] = slot<V>(base + s * k, mask);
    for (int q = it.g; q < qv; q += G) group_vec<B, INV>(tile + q * d, pos, w);
}

// Sub-tile groups of a stage: split the tile's sub-tiles over more items only while
// too few items would leave a fifth or more of the threads' slots empty.
__device__ __forceinline__ int stage_groups(int nb, int qv) {
    int G = 1;
    while (G < qv) {
        const int items = nb * G;
        const int per = (items + kThreads - 1) / kThreads;
        if (per * kThreads * 4 <= items * 5) break;
        ++G;
    }
    return G;
}

// What a thread prefetches after its last item of a stage: the first block it will
// apply in the next stage (of this tile, or stage 0 of its next tile).
struct NextFirst {
    const float* stage;   // lane-interleaved blocks of that stage (nullptr: nothing)
    int nb, bb;
};

// All items of one stage.  Coefficients are double-buffered in wa / wb: on entry the
// buffer named by cur_a holds (or is loading) the thread's first block of this stage;
// while an item is applied the other buffer loads the next one, which after the last
// item is the first block of the next stage, so on exit cur_a names that buffer.
template <int B, bool INV, int V>
__device__ __forceinline__ void run_stage(const float* __restrict__ sb, int s, typename VecOf<V>::T* tile,
                                          int d, int qv, int mask, float (&wa)[64], float (&wb)[64],
                                          bool& cur_a, const NextFirst& nx) {
    const int nb = d / B;
    const int G = stage_groups(nb, qv);
    const int items = nb * G;
    const int tid = threadIdx.x;
    int j = tid;
    if (j >= items) {   // idle in this stage: start loading the next stage's block now
        if (nx.stage) {
            if (cur_a) load_block_any(wa, nx.stage, tid % nx.nb, nx.bb);
            else load_block_any(wb, nx.stage, tid % nx.nb, nx.bb);
        }
        return;
    }
    // Items j = tid, tid + T, ...: c = j % nb, g = j / nb, and for the block lo = c % s,
    // hi = c / s, stepped by T without dividing (T % s, T / s once per stage).
    ItemPos it;
    it.c = tid % nb;
    it.g = tid / nb;
    it.lo = it.c % s;
    it.hi = it.c / s;
    const int dlo = kThreads % s, dhi = kThreads / s;
    while (true) {
        const int jn = j + kThreads;
        ItemPos nt = it;
        nt.c += kThreads;
        nt.lo += dlo;
        nt.hi += dhi;
        if (nt.lo >= s) {
            nt.lo -= s;
            ++nt.hi;
        }
        if (nt.c >= nb) {   // wrapped into the next sub-tile group (small nb only)
            nt.c -= nb;
            ++nt.g;
            while (nt.c >= nb) {
                nt.c -= nb;
                ++nt.g;
            }
            nt.lo = nt.c % s;
            nt.hi = nt.c / s;
        }
        if (cur_a) {
            if (jn < items) load_block<B>(wb, sb, nt.c);
            else if (nx.stage) load_block_any(wb, nx.stage, tid % nx.nb, nx.bb);
            apply_item<B, INV, V>(tile, d, qv, G, s, mask, it, wa);
        } else {
            if (jn < items) load_block<B>(wa, sb, nt.c);
            else if (nx.stage) load_block_any(wa, nx.stage, tid % nx.nb, nx.bb);
            apply_item<B, INV, V>(tile, d, qv, G, s, mask, it, wb);
        }
        cur_a = !cur_a;
        if (jn >= items) break;
        j = jn;
        it = nt;
    }
}

template <typename TIn>
__device__ __forceinline__ void issue_tile(const TiledParams& p, int64_t tile, unsigned char* stage_buf,
                                           uint64_t* bar) {
    const int d = (int)p.pd.d;
    const int64_t row0 = tile * p.R;
    const int nr = (int)min((int64_t)p.staged_rows, p.rows - row0);
    const uint32_t row_bytes = (uint32_t)d * sizeof(TIn);
    mbar_arrive_expect_tx(bar, row_bytes * nr);
    const TIn* x = (const TIn*)p.x;
    for (int r = 0; r < nr; ++r) bulk_load(stage_buf + (size_t)r * row_bytes, x + (row0 + r) * p.ld_x, row_bytes, bar);
}

// Rows -> sub-tiles.  V = 4: a thread takes 8 consecutive coordinates of the 4 rows of a
// sub-tile and writes them as 8 quads.  V = 1: 8 consecutive coordinates of one row, two
// 16-byte stores (the XOR keeps 8-aligned runs contiguous).  Rows past the end of the
// batch are zero.
template <int V, typename TIn>
__device__ __forceinline__ void fill_tile(typename VecOf<V>::T* tile, int d, int nr, int n_staged, const TIn* staged,
                                          const TIn* src, int64_t ld, int mask) {
    const int d8 = d / 8;
    // row r of the tile: the staging area for r < n_staged, else global memory
    auto row_ptr = [&](int r) -> const TIn* { return r < n_staged ? staged + (size_t)r * d : src + r * ld; };
    for (int q = 0; V * q < nr; ++q)
        for (int j = threadIdx.x; j < d8; j += kThreads) {
            if constexpr (V == 4) {
                float v[4][8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (4 * q + e < nr) {
                        load8(row_ptr(4 * q + e) + 8 * j, v[e]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) v[e][k] = 0.0f;
                    }
                }
                float4* st = tile + q * d;
#pragma unroll
                for (int k = 0; k < 8; ++k) st[slot<4>(8 * j + k, mask)] = make_float4(v[0][k], v[1][k], v[2][k], v[3][k]);
            } else {
                float v[8];
                load8(row_ptr(q) + 8 * j, v);
                store8(tile + q * d + slot<1>(8 * j, mask), v);
            }
        }
}

template <int V, typename TOut>
__device__ __forceinline__ void drain_tile(const typename VecOf<V>::T* tile, int d, int nr, TOut* dst, int64_t ld,
                                           int mask) {
    const int d8 = d / 8;
    for (int q = 0; V * q < nr; ++q)
        for (int j = threadIdx.x; j < d8; j += kThreads) {
            if constexpr (V == 4) {
                const float4* st = tile + q * d;
                float4 v4[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v4[k] = st[slot<4>(8 * j + k, mask)];
                float v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = v4[k].x;
                store8(dst + (4 * q) * ld + 8 * j, v);
                if (4 * q + 1 < nr) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].y;
                    store8(dst + (4 * q + 1) * ld + 8 * j, v);
                }
                if (4 * q + 2 < nr) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].z;
                    store8(dst + (4 * q + 2) * ld + 8 * j, v);
                }
                if (4 * q + 3 < nr) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].w;
                    store8(dst + (4 * q + 3) * ld + 8 * j, v);
                }
            } else {
                float v[8];
                load8(tile + q * d + slot<1>(8 * j, mask), v);
                store8(dst + q * ld + 8 * j, v);
            }
        }
}

template <typename TIn, typename TOut, bool INV, int MASK, int V>
__global__ void __launch_bounds__(kThreads, 1) harp_tiled_kernel(const __grid_constant__ TiledParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    using VT = typename VecOf<V>::T;
    const int d = (int)p.pd.d;
    const int m = p.pd.m;
    const int R = p.R;
    const int tid = threadIdx.x;
    VT* tile = (VT*)smem;
    unsigned char* stage_buf = smem + (size_t)R * d * sizeof(float);
    uint64_t* bar = (uint64_t*)(stage_buf + (size_t)p.staged_rows * d * sizeof(TIn));

    int64_t t_idx = blockIdx.x;
    if (t_idx >= p.ntiles) return;
    if (p.staged_rows) {
        if (tid == 0) mbar_init(bar, 1);
        __syncthreads();
        if (tid == 0) issue_tile<TIn>(p, t_idx, stage_buf, bar);
    }
    // The stage order: forward 0..m-1, inverse m-1..0.
    auto stage_of = [&](int step) { return INV ? m - 1 - step : step; };
    auto first_of = [&](int step, int qv_) {
        const int t = stage_of(step);
        const int b = p.pd.st[t].b, nb = d / b;
        NextFirst f;
        f.stage = tid < nb * stage_groups(nb, qv_) ? p.lanes + p.lane_off[t] : nullptr;
        f.nb = nb;
        f.bb = b * b;
        return f;
    };
    float wa[64], wb[64];
    bool cur_a = true;
    {
        const int nr0 = (int)min((int64_t)R, p.rows - t_idx * R);
        const NextFirst f = first_of(0, (nr0 + V - 1) / V);
        if (f.stage) load_block_any(wa, f.stage, tid % f.nb, f.bb);
    }
    uint32_t parity = 0;
    for (; t_idx < p.ntiles; t_idx += gridDim.x) {
        const int64_t row0 = t_idx * R;
        const int nr = (int)min((int64_t)R, p.rows - row0);
        const int qv = (nr + V - 1) / V;
        const int n_staged = min(nr, p.staged_rows);
        if (n_staged) {
            const bool ok = mbar_wait(bar, parity);
            parity ^= 1;
            if (__syncthreads_or(!ok)) {
                if (tid == 0) atomicExch(p.status, 1);
                return;
            }
        }
        fill_tile<V, TIn>(tile, d, nr, n_staged, (const TIn*)stage_buf, (const TIn*)p.x + row0 * p.ld_x, p.ld_x,
                          p.mask);
        __syncthreads();
        const int64_t t_next = t_idx + gridDim.x;
        if (p.staged_rows && tid == 0 && t_next < p.ntiles) {
            fence_proxy_async_smem();   // the staging reads above happen before the copies' writes
            issue_tile<TIn>(p, t_next, stage_buf, bar);
        }
        const int nr_next = t_next < p.ntiles ? (int)min((int64_t)R, p.rows - t_next * R) : 0;
        for (int step = 0; step < m; ++step) {
            const int t = stage_of(step);
            const StageDesc& sd = p.pd.st[t];
            NextFirst nx;
            if (step + 1 < m) nx = first_of(step + 1, qv);
            else if (nr_next) nx = first_of(0, (nr_next + V - 1) / V);
            else nx.stage = nullptr, nx.nb = 1, nx.bb = 0;
            const float* sb = p.lanes + p.lane_off[t];
            const int s = (int)sd.s;
            switch (sd.b) {
#define HARP_TILED_CASE(R)                                                                       \
    case R:                                                                                      \
        if constexpr ((MASK >> R) & 1) run_stage<R, INV, V>(sb, s, tile, d, qv, p.mask, wa, wb, cur_a, nx); \
        break;
                HARP_TILED_CASE(2) HARP_TILED_CASE(3) HARP_TILED_CASE(4) HARP_TILED_CASE(5)
                HARP_TILED_CASE(6) HARP_TILED_CASE(7) HARP_TILED_CASE(8)
#undef HARP_TILED_CASE
                default: break;
            }
            __syncthreads();
        }
        drain_tile<V, TOut>(tile, d, nr, (TOut*)p.y + row0 * p.ld_y, p.ld_y, p.mask);
        __syncthreads();
    }
}

// Radix sets with their own kernel: a kernel that instantiates every radix needs more
// registers than any single one, so the common schedules get kernels with only the
// radices they use.  The last entry (all of 2..8) covers every other schedule.
constexpr int kMasks[] = {1 << 8, (1 << 2) | (1 << 8), (1 << 2) | (1 << 5) | (1 << 8), (1 << 7) | (1 << 8),
                          (1 << 2) | (1 << 7) | (1 << 8), 0x1fc};
constexpr int kNumMasks = sizeof(kMasks) / sizeof(kMasks[0]);

// Sub-tiles of one row (V = 1) are needed only when four fp32 rows do not fit in shared
// memory (d > 14524); they are built for the radix sets without 5.
constexpr bool has_row_major_kernel(int mask) { return ((mask >> 5) & 1) == 0; }

template <typename TIn, typename TOut, bool INV, int V, int I>
cudaError_t launch_mask(int which, const TiledParams& tp, size_t smem, int grid, cudaStream_t stream) {
    if constexpr (I < kNumMasks) {
        if (which != I) return launch_mask<TIn, TOut, INV, V, I + 1>(which, tp, smem, grid, stream);
        if constexpr (V == 1 && !has_row_major_kernel(kMasks[I])) {
            return cudaErrorInvalidValue;
        } else {
            auto kern = harp_tiled_kernel<TIn, TOut, INV, kMasks[I], V>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<(unsigned)grid, kThreads, smem, stream>>>(tp);
            return cudaGetLastError();
        }
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename TIn, typename TOut>
cudaError_t launch(int which, int V, bool inverse, const TiledParams& tp, size_t smem, int grid,
                   cudaStream_t stream) {
    if (V == 4)
        return inverse ? launch_mask<TIn, TOut, true, 4, 0>(which, tp, smem, grid, stream)
                       : launch_mask<TIn, TOut, false, 4, 0>(which, tp, smem, grid, stream);
    return inverse ? launch_mask<TIn, TOut, true, 1, 0>(which, tp, smem, grid, stream)
                   : launch_mask<TIn, TOut, false, 1, 0>(which, tp, smem, grid, stream);
}

}  // namespace harp_tiled

// One translation unit per I/O type pair (compiled in parallel).
cudaError_t harp_tiled_launch_bf16(int which, int V, bool inverse, const harp_tiled::TiledParams& tp,
                                   size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_f32(int which, int V, bool inverse, const harp_tiled::TiledParams& tp,
                                  size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_bf16_f32(int which, int V, bool inverse, const harp_tiled::TiledParams& tp,
                                       size_t smem, int grid, cudaStream_t stream);
