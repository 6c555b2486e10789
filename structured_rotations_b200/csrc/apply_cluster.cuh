// Cluster row kernel for the HARP transform (HARP technical summary §2.1 Core Architecture:
// stages of b_t x b_t blocks on stride-separated groups; §2.2 the blocks): the d coordinates of
// every row are split over the CL CTAs of a thread-block cluster, so each CTA holds only 1/CL of
// the plan's blocks, staged once in its shared memory by one bulk copy, and reads them there.
// Device code; the host side is apply_cluster.cu.
//
// Split at stage t*: S = s_{t*} = prod_{t<t*} b_t, N = d / S, P = S / CL.
//  * Phase A, stages t < t*, mix only the low digits, i.e. the S coordinates of a "chunk"
//    j (coordinates [S j, S j + S)).  CTA r owns the N / CL chunks of the contiguous slab
//    [r dl, r dl + dl), dl = d / CL, held in local order l = i - r dl; stage t acts there with
//    stride s_t, and local block c_l is global block c_l + r dl / b_t.
//  * Phase B, stages t >= t*, mix only the high digits, i.e. the N coordinates a + S j of a
//    "pencil" a < S.  CTA r owns the P pencils a = r P + p, held in local order l = j P + p;
//    stage t acts there with stride s_t / CL, and local block c_l = p + P c' is global block
//    r P + p + S c' (c' the block's index within the pencil).
// Forward runs phase A, then phase B; the inverse runs phase B backwards, then phase A
// backwards, with transposed blocks.  Between the phases every CTA writes each coordinate of
// its buffer into the other phase's buffer of the CTA that owns it (remote shared-memory
// stores across the cluster), and a cluster barrier makes them visible.  Global memory sees
// rows only: slabs are contiguous, and a CTA's pencils are runs of P consecutive coordinates
// (P a multiple of 8, so every run is whole 16-byte pieces).
//
// Per CTA, shared memory holds the CTA's blocks (its segment of the plan's cluster table: per
// stage, its local blocks lane-interleaved in groups of 32, the layout of the tiled kernel's
// block copy, so a warp's block loads are conflict-free) and the two phases' buffers of R rows
// as 4-row quads with the tiled kernel's swizzle.  The stage arithmetic is the tiled kernel's
// (one block in registers per item, applied to whole 4-row quads, plain fp32 FMAs, each output
// summed over its inputs in order), so both kernels give the same bits.
#pragma once

#include "apply_tiled.cuh"

namespace harp_cluster {

using harp_tiled::FastDiv;

constexpr int kMaxCluster = 16;
constexpr int kThreads = 256;

struct ClusterParams {
    PlanDesc pd;
    const float* table;                   // cluster table: rank r's segment at table + r * seg_floats
    int64_t seg_floats;                   // floats per rank (a multiple of 4)
    int64_t stage_off[HARP_MAX_STAGES];   // floats, a stage's blocks within a segment
    int ls[HARP_MAX_STAGES];              // local stride of stage t
    FastDiv nb_div[HARP_MAX_STAGES];      // division by dl / b_t
    FastDiv s_div[HARP_MAX_STAGES];       // division by ls[t]
    int t_split;                          // t*
    int cl;                               // CTAs per cluster
    int dl;                               // coordinates per CTA
    int S;                                // chunk length s_{t*}
    int P;                                // pencils per CTA
    FastDiv S_div, P_div, dl_div;
    const void* x;
    void* y;
    int64_t rows, ld_x, ld_y;             // elements
    int R;                                // rows per tile (a multiple of 4)
    int early;                            // the table is known complete: stage it before the
                                          // wait for the previous kernel of the stream
    int* status;
};

// ----------------------------------------------------------------- PTX ---

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel of the stream start its prologue now /
// wait until the previous kernel of the stream has finished and its memory is visible.
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_previous_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16 bytes into another CTA's shared memory (cluster address), counted on that CTA's mbarrier
// (cluster address) as completed transaction bytes.
__device__ __forceinline__ void st_async4(uint32_t addr, const float4& v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     addr),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
                 : "memory");
}

// ------------------------------------------------------------ helpers ---

// Block c of a stage from its lane-interleaved segment in shared memory (see the tiled
// kernel's load_block; 32 consecutive blocks are read as contiguous 16-byte pieces).
template <int B>
__device__ __forceinline__ void load_block_smem(float (&w)[64], const float* stage, int c) {
    const int group = c >> 5, lane = c & 31;
    if constexpr ((B * B) % 4 == 0) {
        const float4* src = (const float4*)stage + group * (B * B / 4) * 32 + lane;
#pragma unroll
        for (int q = 0; q < B * B / 4; ++q) {
            const float4 v = src[q * 32];
            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
        }
    } else {
        const float* src = stage + group * (B * B) * 32 + lane;
#pragma unroll
        for (int e = 0; e < B * B; ++e) w[e] = src[e * 32];
    }
}

// One stage on a buffer of qv quads of dl local coordinates: items j = tid, tid + NT, ...;
// item j is local block c = j % nb applied to quads g = j / nb, g + G, ... (as the tiled kernel).
template <int B, bool INV, int NT>
__device__ __forceinline__ void run_stage(const float* __restrict__ sb, int s, const FastDiv& nbd, const FastDiv& sdv,
                                          float4* buf, int dl, int qv) {
    const int nb = dl / B;
    const int G = harp_tiled::stage_groups(nb, qv, NT);
    const int items = nb * G;
    float w[64];
    for (int j = threadIdx.x; j < items; j += NT) {
        harp_tiled::ItemPos it;
        it.g = nbd.div(j);
        it.c = j - nb * it.g;
        it.hi = sdv.div(it.c);
        it.lo = it.c - s * it.hi;
        load_block_smem<B>(w, sb, it.c);
        harp_tiled::apply_item<B, INV, 4>(buf, dl, qv, G, s, 0, it, w);
    }
}

template <int MASK, bool INV>
__device__ __forceinline__ void stage(const ClusterParams& p, const float* coef, int t, float4* buf, int qv) {
    const float* sb = coef + p.stage_off[t];
    const int s = p.ls[t];
    switch (p.pd.st[t].b) {
#define HARP_CLUSTER_CASE(RB)                                                                       \
    case RB:                                                                                        \
        if constexpr ((MASK >> RB) & 1) run_stage<RB, INV, kThreads>(sb, s, p.nb_div[t], p.s_div[t], buf, p.dl, qv); \
        break;
        HARP_CLUSTER_CASE(2) HARP_CLUSTER_CASE(3) HARP_CLUSTER_CASE(4) HARP_CLUSTER_CASE(5)
        HARP_CLUSTER_CASE(6) HARP_CLUSTER_CASE(7) HARP_CLUSTER_CASE(8)
#undef HARP_CLUSTER_CASE
        default: break;
    }
    __syncthreads();
}

// Column of the row where the 8-coordinate run starting at local l8 (a multiple of 8) lives:
// slab order (phase A) or pencil order (phase B) of CTA r.
__device__ __forceinline__ int run_col(const ClusterParams& p, bool slab, int r, int l8) {
    if (slab) return r * p.dl + l8;
    const int j = p.P_div.div(l8);
    return r * p.P + (l8 - j * p.P) + p.S * j;
}

// Rows [row0, row0 + nr) of x, this CTA's coordinates, into qv quads of `buf` (rows past nr of
// the last quad are zero).
template <typename TIn>
__device__ __forceinline__ void fill(const ClusterParams& p, float4* buf, bool slab, int r, int64_t row0, int nr,
                                     int qv) {
    const int d8 = p.dl / 8;
    const TIn* x = (const TIn*)p.x;
    for (int e8 = threadIdx.x; e8 < qv * d8; e8 += kThreads) {
        const int q = e8 / d8, jj = e8 - q * d8;
        const int col = run_col(p, slab, r, 8 * jj);
        float v[4][8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = 4 * q + e;
            if (row < nr) {
                harp_tiled::load8(x + (row0 + row) * p.ld_x + col, v[e]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[e][k] = 0.f;
            }
        }
        const int jx = jj & 7;
        float4* st = buf + q * p.dl + 8 * jj;
#pragma unroll
        for (int k = 0; k < 8; ++k) st[k ^ jx] = make_float4(v[0][k], v[1][k], v[2][k], v[3][k]);
    }
}

template <typename TOut>
__device__ __forceinline__ void drain(const ClusterParams& p, const float4* buf, bool slab, int r, int64_t row0, int nr,
                                      int qv) {
    const int d8 = p.dl / 8;
    TOut* y = (TOut*)p.y;
    for (int e8 = threadIdx.x; e8 < qv * d8; e8 += kThreads) {
        const int q = e8 / d8, jj = e8 - q * d8;
        const int col = run_col(p, slab, r, 8 * jj);
        const int jx = jj & 7;
        const float4* st = buf + q * p.dl + 8 * jj;
        float4 v4[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v4[k] = st[k ^ jx];
        float v[8];
        const int nrow = min(4, nr - 4 * q);
        TOut* yr = y + (row0 + 4 * q) * p.ld_y + col;
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = v4[k].x;
        harp_tiled::store8(yr, v);
        if (nrow > 1) {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = v4[k].y;
            harp_tiled::store8(yr + p.ld_y, v);
        }
        if (nrow > 2) {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = v4[k].z;
            harp_tiled::store8(yr + 2 * p.ld_y, v);
        }
        if (nrow > 3) {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = v4[k].w;
            harp_tiled::store8(yr + 3 * p.ld_y, v);
        }
    }
}

// Every coordinate of this CTA's `src` buffer (slab order if from_slab, else pencil order) to the
// other phase's buffer `dst` of the CTA that owns it, by 8-coordinate runs (a run has one owner
// and maps to one aligned run there, since P is a multiple of 8).  The stores are asynchronous
// and complete on the owner's exchange mbarrier `xbar`, which expects all of its buffer's bytes.
__device__ __forceinline__ void exchange(const ClusterParams& p, const float4* src, const float4* dst, bool from_slab,
                                         int r, int qv, const uint64_t* xbar) {
    const int d8 = p.dl / 8;
    const uint32_t dst_local = (uint32_t)__cvta_generic_to_shared(dst);
    const uint32_t bar_local = (uint32_t)__cvta_generic_to_shared(xbar);
    for (int e8 = threadIdx.x; e8 < qv * d8; e8 += kThreads) {
        const int q = e8 / d8, jj = e8 - q * d8;
        int owner, ld8;
        if (from_slab) {                    // slab -> pencils: i = r dl + l, j = i / S, a = i % S
            const int i0 = r * p.dl + 8 * jj;
            const int j = p.S_div.div(i0);
            const int a = i0 - j * p.S;
            owner = p.P_div.div(a);
            ld8 = j * p.P + (a - owner * p.P);
        } else {                            // pencils -> slab: l = j P + pp, i = r P + pp + S j
            const int l8 = 8 * jj;
            const int j = p.P_div.div(l8);
            const int i0 = r * p.P + (l8 - j * p.P) + p.S * j;
            owner = p.dl_div.div(i0);
            ld8 = i0 - owner * p.dl;
        }
        const int jx = jj & 7, jd = (ld8 >> 3) & 7;
        const float4* s = src + q * p.dl + 8 * jj;
        const uint32_t base = harp_tiled::map_to_rank(dst_local + (uint32_t)((q * p.dl + ld8) * 16), (uint32_t)owner);
        const uint32_t rbar = harp_tiled::map_to_rank(bar_local, (uint32_t)owner);
#pragma unroll
        for (int k = 0; k < 8; ++k) st_async4(base + (uint32_t)((k ^ jd) * 16), s[k ^ jx], rbar);
    }
}

// Persistent over tiles of R rows: cluster c takes tiles c, c + nclusters, ... (every CTA of a
// cluster the same tiles, so the cluster barriers below are met by all of them the same number
// of times).  Shared memory: [this rank's blocks | phase-A buffer | phase-B buffer | mbarriers].
// The blocks arrive by one bulk copy per stage, each on its own mbarrier, so the first stage
// starts as soon as its own blocks have landed; they then stay for every tile.
template <typename TIn, typename TOut, bool INV, int MASK>
__global__ void __launch_bounds__(kThreads, 1) harp_cluster_kernel(const __grid_constant__ ClusterParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t r = harp_tiled::cluster_rank();
    float* coef = (float*)smem;
    float4* bufA = (float4*)(smem + p.seg_floats * 4);
    float4* bufB = bufA + (size_t)(p.R / 4) * p.dl;
    uint64_t* bar = (uint64_t*)(bufB + (size_t)(p.R / 4) * p.dl);   // one per stage
    uint64_t* xbar = bar + HARP_MAX_STAGES;                             // the exchange's bytes into `second`
    const int tid = threadIdx.x;
    const int m = p.pd.m, ts = p.t_split;
    const int64_t nclusters = gridDim.x / p.cl;
    const int64_t ntiles = (p.rows + p.R - 1) / p.R;

    // this rank's blocks, one bulk copy per stage, in the order the stages run
    if (tid == 0) {
        for (int t = 0; t < m; ++t) harp_tiled::mbar_init(bar + t, 1);
        harp_tiled::mbar_init(xbar, 1);     // initialised before the cluster barrier that lets others write
    }
    __syncthreads();
    auto stage_blocks = [&] {
        for (int k = 0; k < m; ++k) {
            const int t = INV ? m - 1 - k : k;
            const int64_t end = t + 1 < m ? p.stage_off[t + 1] : p.seg_floats;
            const uint32_t bytes = (uint32_t)((end - p.stage_off[t]) * 4);
            harp_tiled::mbar_arrive_expect_tx(bar + t, bytes);
            harp_tiled::bulk_load(coef + p.stage_off[t], p.table + (int64_t)r * p.seg_floats + p.stage_off[t], bytes,
                                  bar + t);
        }
    };
    // The next kernel of the stream may start its own prologue now.  Rows are touched only
    // after the wait for the kernel before this one (which may write x or read y); the plan's
    // table, which nothing writes after it is built, is staged before that wait when the host
    // has seen its build complete (p.early), else after it.
    launch_dependents();
    if (tid == 0 && p.early) stage_blocks();
    cluster_arrive();   // this CTA runs: the others may write into its buffers (matched below)
    wait_previous_grid();
    if (tid == 0 && !p.early) stage_blocks();

    float4* first = INV ? bufB : bufA;      // the first phase's buffer
    float4* second = INV ? bufA : bufB;
    bool have_blocks = false;
    uint32_t xparity = 0;
    for (int64_t tile = blockIdx.x / p.cl; tile < ntiles; tile += nclusters) {
        const int64_t row0 = tile * p.R;
        const int nr = (int)min((int64_t)p.R, p.rows - row0);
        const int qv = (nr + 3) / 4;
        // every CTA of the cluster stores this tile's qv quads of dl coordinates into `second`
        if (tid == 0) harp_tiled::mbar_arrive_expect_tx(xbar, (uint32_t)(qv * p.dl * 16));
        fill<TIn>(p, first, !INV, (int)r, row0, nr, qv);
        __syncthreads();
        if (!INV) {
            for (int t = 0; t < ts; ++t) {
                if (!have_blocks && !harp_tiled::mbar_wait(bar + t, 0)) {
                    if (tid == 0) atomicExch(p.status, 1);
                    harp_tiled::mbar_wait(bar + t, 0);   // bounded again: no copy may land after exit
                }
                stage<MASK, false>(p, coef, t, first, qv);
            }
        } else {
            for (int t = m - 1; t >= ts; --t) {
                if (!have_blocks && !harp_tiled::mbar_wait(bar + t, 0)) {
                    if (tid == 0) atomicExch(p.status, 1);
                    harp_tiled::mbar_wait(bar + t, 0);
                }
                stage<MASK, true>(p, coef, t, first, qv);
            }
        }
        cluster_wait();     // every CTA runs, and has drained its `second` buffer of the last tile
        exchange(p, first, second, !INV, (int)r, qv, xbar);
        if (!harp_tiled::mbar_wait(xbar, xparity)) {   // every CTA's stores into `second` have landed
            if (tid == 0) atomicExch(p.status, 1);
            harp_tiled::mbar_wait(xbar, xparity);     // bounded again: no store may land after exit
        }
        xparity ^= 1;
        if (!INV) {
            for (int t = ts; t < m; ++t) {
                if (!have_blocks && !harp_tiled::mbar_wait(bar + t, 0)) {
                    if (tid == 0) atomicExch(p.status, 1);
                    harp_tiled::mbar_wait(bar + t, 0);
                }
                stage<MASK, false>(p, coef, t, second, qv);
            }
        } else {
            for (int t = ts - 1; t >= 0; --t) {
                if (!have_blocks && !harp_tiled::mbar_wait(bar + t, 0)) {
                    if (tid == 0) atomicExch(p.status, 1);
                    harp_tiled::mbar_wait(bar + t, 0);
                }
                stage<MASK, true>(p, coef, t, second, qv);
            }
        }
        have_blocks = true;
        drain<TOut>(p, second, INV, (int)r, row0, nr, qv);
        cluster_arrive();   // this CTA's `second` buffer may take the next tile's exchange
    }
    cluster_wait();         // matches the last arrive
    if (!have_blocks) {
        // no tile for this cluster: the block copies were issued all the same; wait for them
        for (int t = 0; t < m; ++t) harp_tiled::mbar_wait(bar + t, 0);
    }
}

template <typename TIn, typename TOut, bool INV, int I>
cudaError_t launch_mask(int which, int cl, const ClusterParams& cp, size_t smem, int grid, cudaStream_t stream) {
    if constexpr (I < harp_tiled::kNumMasks) {
        if (which != I) return launch_mask<TIn, TOut, INV, I + 1>(which, cl, cp, smem, grid, stream);
        auto kern = harp_cluster_kernel<TIn, TOut, INV, harp_tiled::kMasks[I]>;
        cudaError_t e = (cudaError_t)harp_set_smem_limit((const void*)kern, (int)smem);
        if (e != cudaSuccess) return e;
        if (cl > 8) {
            e = cudaFuncSetAttribute((const void*)kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        // may start before the previous kernel of the stream ends; it waits for it (above)
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, kern, cp);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename TIn, typename TOut>
cudaError_t launch(int which, int cl, bool inverse, const ClusterParams& cp, size_t smem, int grid,
                   cudaStream_t stream) {
    return inverse ? launch_mask<TIn, TOut, true, 0>(which, cl, cp, smem, grid, stream)
                   : launch_mask<TIn, TOut, false, 0>(which, cl, cp, smem, grid, stream);
}

}  // namespace harp_cluster

cudaError_t harp_cluster_launch_bf16(int which, int cl, bool inverse, const harp_cluster::ClusterParams& cp,
                                     size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_cluster_launch_f32(int which, int cl, bool inverse, const harp_cluster::ClusterParams& cp,
                                    size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_cluster_launch_bf16_f32(int which, int cl, bool inverse, const harp_cluster::ClusterParams& cp,
                                         size_t smem, int grid, cudaStream_t stream);
