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
// once per tile rather than once per row; 8 warps per SM hide the load latency.  The
// inverse runs the stages backwards with
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

#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace harp_tiled {

constexpr int kMaxTileRows = 32;
constexpr int kSmemOptIn = 227 * 1024;
constexpr long long kWaitLimit = 1ll << 26;   // mbarrier polls before giving up

// Division by a constant n >= 1 of x < 2^21 by multiply and shift: with l = ceil(log2 n)
// and m = ceil(2^(32+l) / n) - 2^32, x / n = (umulhi(x, m) + x) >> l (built on the host,
// see make_fast_div).
struct FastDiv {
    uint32_t m;
    int l;
    int n;
#ifdef __CUDACC__
    __device__ __forceinline__ int div(int x) const { return (int)((__umulhi((uint32_t)x, m) + (uint32_t)x) >> l); }
#endif
};

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
    FastDiv nb_div[HARP_MAX_STAGES];   // division by (coordinates per CTA) / b_t
    FastDiv s_div[HARP_MAX_STAGES];    // division by s_t
    const float* last_blocks;          // slab mode: plain 2 x 2 blocks of the last stage
    float* scales;                     // quantized output (int8 codes in y): per-block scales
    int64_t ld_s;                      // scales per row of the scales array (row stride)
    int qlanes;                        // quantizer block / 8: lanes that hold one block
    int fuse_first, fuse_last;         // stage applied while filling / draining the tile (kFuse*)
    long long wait_limit;              // polls of a staging wait before it gives up (kWaitLimit)
    uint32_t extra_tx;                 // test hook, normally 0: bytes each staging barrier is told to
                                       // expect beyond what is copied, so its first wait runs out
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

// Retires `bytes` of a barrier's expected transaction count without a copy.
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait for the phase with the given parity; false after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit = kWaitLimit) {
    const uint32_t addr = smem_u32(bar);
    for (long long i = 0; i < limit; ++i) {
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

// Global -> this CTA's own shared memory, completed on the mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Both CTAs of the cluster reach this point; shared-memory writes before it are
// visible to the partner after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_cluster4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_cluster4(uint32_t addr, const float4& v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
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
__host__ __device__ __forceinline__ int stage_groups(int nb, int qv, int nthreads) {
    int G = 1;
    while (G < qv) {
        const int items = nb * G;
        const int per = (items + nthreads - 1) / nthreads;
        if (per * nthreads * 4 <= items * 5) break;
        ++G;
    }
    return G;
}

// All items of one stage: items j = tid, tid + T, ...; item j is block c = j % nb of the
// sub-tiles g = j / nb, g + G, ...  The block's coefficients are loaded into registers at
// the start of the item (for radix 8 with 256 threads, one item ahead into a second register
// block; elsewhere the registers are not there), except the first item's, which the caller has
// already requested (prefetch_first) before the barrier that opens the stage, so its L2
// latency overlaps the barrier wait.
template <int B, bool INV, int V, int NT>
__device__ __forceinline__ void run_stage(const float* __restrict__ sb, int s, const FastDiv& nbd,
                                          const FastDiv& sdv, typename VecOf<V>::T* tile, int d, int qv,
                                          int mask, float (&w)[64]) {
    const int nb = d / B;
    const int G = stage_groups(nb, qv, NT);
    const int items = nb * G;
    const int tid = threadIdx.x;
    if (tid >= items) return;
    // (c, g, lo = c % s, hi = c / s) stepped by T from item to item
    ItemPos it;
    it.g = nbd.div(tid);
    it.c = tid - nb * it.g;
    it.hi = sdv.div(it.c);
    it.lo = it.c - s * it.hi;
    const int dhi = sdv.div(NT), dlo = NT - s * dhi;
    auto advance = [&](ItemPos& q) {
        q.c += NT;
        q.lo += dlo;
        q.hi += dhi;
        if (q.lo >= s) {
            q.lo -= s;
            ++q.hi;
        }
        if (q.c >= nb) {   // wrapped into the next sub-tile group (small nb only)
            do {
                q.c -= nb;
                ++q.g;
            } while (q.c >= nb);
            q.hi = sdv.div(q.c);
            q.lo = q.c - s * q.hi;
        }
    };
    if constexpr (B == 8 && NT == 256) {
        // Radix 8 with 256 threads (registers to spare): two register blocks take turns, so
        // the next item's block is in flight while this item's FMAs run, with no moves.
        float w1[64];
        for (int j = tid; j < items; j += 2 * NT) {
            ItemPos it1 = it;
            advance(it1);
            const bool has1 = j + NT < items;
            if (has1) load_block<B>(w1, sb, it1.c);
            apply_item<B, INV, V>(tile, d, qv, G, s, mask, it, w);
            ItemPos it2 = it1;
            advance(it2);
            if (j + 2 * NT < items) load_block<B>(w, sb, it2.c);
            if (has1) apply_item<B, INV, V>(tile, d, qv, G, s, mask, it1, w1);
            it = it2;
        }
        return;
    }
    for (int j = tid; j < items; j += NT) {
        if (j != tid) load_block<B>(w, sb, it.c);   // the first item's block is already requested
        apply_item<B, INV, V>(tile, d, qv, G, s, mask, it, w);
        advance(it);
    }
}

// Requests the block of this thread's first item of stage t (item j = tid) for a tile of qv
// sub-tiles, into w; run_stage then uses it without loading it again.
template <int MASK, int V, int NT>
__device__ __forceinline__ void prefetch_first(const TiledParams& p, int t, int qv, int dl, uint32_t rank,
                                               float (&w)[64]) {
    const StageDesc& sd = p.pd.st[t];
    const float* sb = p.lanes + p.lane_off[t] + (int64_t)rank * dl * sd.b;
    const int tid = threadIdx.x;
    switch (sd.b) {
#define HARP_PREFETCH_CASE(RB)                                                                      \
    case RB:                                                                                        \
        if constexpr ((MASK >> RB) & 1) {                                                           \
            const int nb = dl / RB;                                                                 \
            if (tid < nb * stage_groups(nb, qv, NT)) load_block<RB>(w, sb, tid - nb * p.nb_div[t].div(tid)); \
        }                                                                                           \
        break;
        HARP_PREFETCH_CASE(2) HARP_PREFETCH_CASE(3) HARP_PREFETCH_CASE(4) HARP_PREFETCH_CASE(5)
        HARP_PREFETCH_CASE(6) HARP_PREFETCH_CASE(7) HARP_PREFETCH_CASE(8)
#undef HARP_PREFETCH_CASE
        default: break;
    }
}

// The first staged_rows rows of a tile, columns [col0, col0 + dl), to the staging area.
template <typename TIn>
__device__ __forceinline__ void issue_tile(const TiledParams& p, int64_t tile, int dl, int col0,
                                           unsigned char* stage_buf, uint64_t* bar) {
    const int64_t row0 = tile * p.R;
    const int nr = (int)min((int64_t)p.staged_rows, p.rows - row0);
    const uint32_t row_bytes = (uint32_t)dl * sizeof(TIn);
    mbar_arrive_expect_tx(bar, row_bytes * nr + p.extra_tx);
    const TIn* x = (const TIn*)p.x + col0;
    for (int r = 0; r < nr; ++r) bulk_load(stage_buf + (size_t)r * row_bytes, x + (row0 + r) * p.ld_x, row_bytes, bar);
}

// Slab mode, the last stage (radix 2, stride dl = d / 2): position p of the two slabs
// forms a group; this CTA (cluster rank r) computes positions p in [r dl/2, (r+1) dl/2)
// for both slabs, reading and writing the partner's quads through distributed shared
// memory.  Block c = p; each output sums over its two inputs in order.
template <bool INV, int NT>
__device__ __forceinline__ void cross_stage(float4* tile, int dl, int qv, uint32_t rank,
                                            const float* __restrict__ blocks) {
    const int half = dl / 2;
    for (int q = 0; q < qv; ++q) {
        float4* st = tile + q * dl;
        for (int pp = threadIdx.x; pp < half; pp += NT) {
            const int pos = (int)rank * half + pp;
            float4* own = st + slot<4>(pos, 0);
            const uint32_t rem = map_to_rank((uint32_t)__cvta_generic_to_shared(own), rank ^ 1);
            const float4 a = *own, b = ld_cluster4(rem);
            const float4 x0 = rank == 0 ? a : b, x1 = rank == 0 ? b : a;   // slab 0, slab 1
            const float4 w = __ldg((const float4*)blocks + pos);          // B[0][0], B[0][1], B[1][0], B[1][1]
            const float w00 = w.x, w01 = INV ? w.z : w.y, w10 = INV ? w.y : w.z, w11 = w.w;
            float4 y0, y1;
            y0.x = fmaf(w01, x1.x, fmaf(w00, x0.x, 0.f));
            y0.y = fmaf(w01, x1.y, fmaf(w00, x0.y, 0.f));
            y0.z = fmaf(w01, x1.z, fmaf(w00, x0.z, 0.f));
            y0.w = fmaf(w01, x1.w, fmaf(w00, x0.w, 0.f));
            y1.x = fmaf(w11, x1.x, fmaf(w10, x0.x, 0.f));
            y1.y = fmaf(w11, x1.y, fmaf(w10, x0.y, 0.f));
            y1.z = fmaf(w11, x1.z, fmaf(w10, x0.z, 0.f));
            y1.w = fmaf(w11, x1.w, fmaf(w10, x0.w, 0.f));
            *own = rank == 0 ? y0 : y1;
            st_cluster4(rem, rank == 0 ? y1 : y0);
        }
    }
}

// Rows -> sub-tiles.  V = 4: a thread takes 8 consecutive coordinates of the 4 rows of a
// sub-tile and writes them as 8 quads.  V = 1: 8 consecutive coordinates of one row, two
// 16-byte stores (the XOR keeps 8-aligned runs contiguous).  Rows past the end of the
// batch are zero.
template <int V, int NT, typename TIn>
__device__ __forceinline__ void fill_tile(typename VecOf<V>::T* tile, int d, int nr, int n_staged, const TIn* staged,
                                          const TIn* src, int64_t ld, int mask) {
    const int d8 = d / 8;
    // row r of the tile: the staging area for r < n_staged, else global memory
    auto row_ptr = [&](int r) -> const TIn* { return r < n_staged ? staged + (size_t)r * d : src + r * ld; };
    for (int q = 0; V * q < nr; ++q) {
        if constexpr (V == 4) {
            const TIn* rp[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) rp[e] = row_ptr(min(4 * q + e, nr - 1));
            float4* st = tile + q * d;
            for (int j = threadIdx.x; j < d8; j += NT) {
                float v[4][8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    load8(rp[e] + 8 * j, v[e]);
                    if (4 * q + e >= nr) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) v[e][k] = 0.0f;
                    }
                }
                const int jx = j & 7;
#pragma unroll
                for (int k = 0; k < 8; ++k) st[8 * j + (k ^ jx)] = make_float4(v[0][k], v[1][k], v[2][k], v[3][k]);
            }
        } else {
            const TIn* rp = row_ptr(q);
            for (int j = threadIdx.x; j < d8; j += NT) {
                float v[8];
                load8(rp + 8 * j, v);
                store8(tile + q * d + slot<1>(8 * j, mask), v);
            }
        }
    }
}

template <int V, int NT, typename TOut>
__device__ __forceinline__ void drain_tile(const typename VecOf<V>::T* tile, int d, int nr, TOut* dst, int64_t ld,
                                           int mask) {
    const int d8 = d / 8;
    for (int q = 0; V * q < nr; ++q) {
        if constexpr (V == 4) {
            const float4* st = tile + q * d;
            TOut* rp = dst + (4 * q) * ld;
            const int rows = min(4, nr - 4 * q);
            for (int j = threadIdx.x; j < d8; j += NT) {
                const int jx = j & 7;
                float4 v4[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v4[k] = st[8 * j + (k ^ jx)];
                float v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = v4[k].x;
                store8(rp + 8 * j, v);
                if (rows > 1) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].y;
                    store8(rp + ld + 8 * j, v);
                }
                if (rows > 2) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].z;
                    store8(rp + 2 * ld + 8 * j, v);
                }
                if (rows > 3) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = v4[k].w;
                    store8(rp + 3 * ld + 8 * j, v);
                }
            }
        } else {
            TOut* rp = dst + q * ld;
            for (int j = threadIdx.x; j < d8; j += NT) {
                float v[8];
                load8(tile + q * d + slot<1>(8 * j, mask), v);
                store8(rp + 8 * j, v);
            }
        }
    }
}

// Stages applied while a tile is filled or drained (4-row sub-tiles), so they cost no pass of
// their own over the tile in shared memory:
//  kFuseS1R8  radix 8 at stride 1: the 8 consecutive coordinates a thread moves are one group
//             (block c = the run's index);
//  kFuseH2R2  radix 2 at stride d / 2: runs j and j + d / 16 hold the groups c = 8 j + e
//             (coordinates c and c + d / 2).
// The arithmetic is group_vec's: every output summed over its inputs in order from zero.
enum { kFuseNone = 0, kFuseS1R8 = 1, kFuseH2R2 = 2 };

// The 8 x 8 block c of a stage (lane-interleaved at sb; B, or B^T when TR) applied to 8 quads,
// in two halves of four outputs so that only half of the block is in registers at a time:
// outputs 4h .. 4h + 3 need rows 4h .. of B (pieces 8h .. 8h + 7 of the block) or columns
// 4h .. of B (the first or second 16 bytes of each row: pieces 2l + h).
template <bool TR>
__device__ __forceinline__ void block8_quads(const float* __restrict__ sb, int c, const float4 (&xv)[8],
                                             float4 (&yv)[8]) {
    const float4* src = (const float4*)sb + (size_t)(c >> 5) * 16 * 32 + (c & 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float w[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = __ldg(src + (TR ? 2 * i + h : 8 * h + i) * 32);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
        // forward: w[kk * 8 + l] = B[4h + kk][l]; inverse: w[l * 4 + kk] = B[l][4h + kk]
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) zero_v(yv[4 * h + kk]);
#pragma unroll
        for (int l = 0; l < 8; ++l)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) fma_v(yv[4 * h + kk], TR ? w[l * 4 + kk] : w[kk * 8 + l], xv[l]);
    }
}

// One 2 x 2 block (stored B00, B01, B10, B11) applied to the quads of coordinates c and c + d/2.
template <bool TR>
__device__ __forceinline__ void block2_quads(const float4& wb, const float4& x0, const float4& x1, float4& y0,
                                             float4& y1) {
    const float w00 = wb.x, w01 = TR ? wb.z : wb.y, w10 = TR ? wb.y : wb.z, w11 = wb.w;
    zero_v(y0);
    zero_v(y1);
    fma_v(y0, w00, x0);
    fma_v(y0, w01, x1);
    fma_v(y1, w10, x0);
    fma_v(y1, w11, x1);
}

// fill_tile (4-row sub-tiles) with the stage `kind` applied on the way (blocks of that stage,
// lane-interleaved, at sb; TR: transposed blocks, the inverse).
template <int NT, typename TIn, bool TR>
__device__ __forceinline__ void fill_tile_fused(float4* tile, int d, int nr, int n_staged, const TIn* staged,
                                                const TIn* src, int64_t ld, int kind, const float* __restrict__ sb) {
    auto row_ptr = [&](int r) -> const TIn* { return r < n_staged ? staged + (size_t)r * d : src + r * ld; };
    auto load_rows = [&](const TIn* const (&rp)[4], int q, int col, float (&v)[4][8]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            load8(rp[e] + col, v[e]);
            if (4 * q + e >= nr) {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[e][k] = 0.0f;
            }
        }
    };
    for (int q = 0; 4 * q < nr; ++q) {
        const TIn* rp[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) rp[e] = row_ptr(min(4 * q + e, nr - 1));
        float4* st = tile + q * d;
        if (kind == kFuseS1R8) {
            for (int j = threadIdx.x; j < d / 8; j += NT) {
                float v[4][8];
                load_rows(rp, q, 8 * j, v);
                float4 xv[8], yv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) xv[k] = make_float4(v[0][k], v[1][k], v[2][k], v[3][k]);
                block8_quads<TR>(sb, j, xv, yv);
                const int jx = j & 7;
#pragma unroll
                for (int k = 0; k < 8; ++k) st[8 * j + (k ^ jx)] = yv[k];
            }
        } else {
            const int h = d / 16;
            for (int j = threadIdx.x; j < h; j += NT) {
                float a[4][8], b[4][8];
                load_rows(rp, q, 8 * j, a);
                load_rows(rp, q, 8 * j + d / 2, b);
                const int ja = j & 7, jb = (j + h) & 7;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 wb = __ldg((const float4*)sb + 8 * j + e);
                    float4 y0, y1;
                    block2_quads<TR>(wb, make_float4(a[0][e], a[1][e], a[2][e], a[3][e]),
                                     make_float4(b[0][e], b[1][e], b[2][e], b[3][e]), y0, y1);
                    st[8 * j + (e ^ ja)] = y0;
                    st[8 * (j + h) + (e ^ jb)] = y1;
                }
            }
        }
    }
}

// 8 floats of row component e of 8 quads
__device__ __forceinline__ void quad_lane(const float4 (&v4)[8], int e, float (&v)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = e == 0 ? v4[k].x : e == 1 ? v4[k].y : e == 2 ? v4[k].z : v4[k].w;
}

// drain_tile (4-row sub-tiles) with the stage `kind` applied on the way.
template <int NT, typename TOut, bool TR>
__device__ __forceinline__ void drain_tile_fused(const float4* tile, int d, int nr, TOut* dst, int64_t ld, int kind,
                                                 const float* __restrict__ sb) {
    for (int q = 0; 4 * q < nr; ++q) {
        const float4* st = tile + q * d;
        TOut* rp = dst + (4 * q) * ld;
        const int rows = min(4, nr - 4 * q);
        auto put = [&](const float4 (&y)[8], int col) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (e < rows) {
                    quad_lane(y, e, v);
                    store8(rp + e * ld + col, v);
                }
            }
        };
        if (kind == kFuseS1R8) {
            for (int j = threadIdx.x; j < d / 8; j += NT) {
                const int jx = j & 7;
                float4 xv[8], yv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) xv[k] = st[8 * j + (k ^ jx)];
                block8_quads<TR>(sb, j, xv, yv);
                put(yv, 8 * j);
            }
        } else {
            const int h = d / 16;
            for (int j = threadIdx.x; j < h; j += NT) {
                const int ja = j & 7, jb = (j + h) & 7;
                float4 y0[8], y1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 wb = __ldg((const float4*)sb + 8 * j + e);
                    block2_quads<TR>(wb, st[8 * j + (e ^ ja)], st[8 * (j + h) + (e ^ jb)], y0[e], y1[e]);
                }
                put(y0, 8 * j);
                put(y1, 8 * j + d / 2);
            }
        }
    }
}

// Fused quantizer epilogue (the rotated rows feed a blockwise quantizer, HARP technical
// summary §2.4: a drop-in preprocessing step in front of the quantizer).  Each aligned
// block of 8 qlanes coordinates of a row, with maximum magnitude a, becomes one fp32 scale
// s = a / 127 and int8 codes q = clamp(rne(y * (127 / a)), -127, 127) (the quotient and the
// reciprocal rounded to nearest in fp32; s = 0 and q = 0 for an all-zero block).  The
// qlanes consecutive lanes that hold a block, 8 coordinates each, reduce its maximum with
// shuffles; the NR rows a thread holds reduce in the same shuffle rounds.
template <int NR>
__device__ __forceinline__ void quant_rows(const float (&v)[NR][8], int nrows, int8_t* dst, int64_t ld, float* sdst,
                                           int64_t ld_s, int qlanes, unsigned mask, bool lead) {
    float a[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        a[r] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) a[r] = fmaxf(a[r], fabsf(v[r][k]));
    }
    for (int o = 1; o < qlanes; o <<= 1) {
#pragma unroll
        for (int r = 0; r < NR; ++r) a[r] = fmaxf(a[r], __shfl_xor_sync(mask, a[r], o));
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (r >= nrows) break;
        const float inv = a[r] > 0.f ? __fdiv_rn(127.f, a[r]) : 0.f;
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int q = max(-127, min(127, __float2int_rn(v[r][k] * inv)));
            w[k >> 2] |= ((uint32_t)q & 0xffu) << (8 * (k & 3));
        }
        *(uint2*)(dst + r * ld) = make_uint2(w[0], w[1]);
        if (lead) sdst[r * ld_s] = __fdiv_rn(a[r], 127.f);
    }
}

template <int V, int NT>
__device__ __forceinline__ void drain_tile_quant(const typename VecOf<V>::T* tile, int d, int nr, int8_t* dst,
                                                 int64_t ld, int mask, float* sdst, int64_t ld_s, int qlanes) {
    const int d8 = d / 8;
    const int lane = threadIdx.x & 31;
    for (int q = 0; V * q < nr; ++q) {
        // warp-uniform loop: every lane of a warp takes the same trips, so the shuffles'
        // mask is exact; lanes past the row's end sit out (whole quantizer blocks)
        for (int j0 = (int)threadIdx.x - lane; j0 < d8; j0 += NT) {
            const int j = j0 + lane;
            const bool act = j < d8;
            const unsigned amask = __ballot_sync(0xffffffffu, act);
            if (!act) continue;
            const bool lead = (j & (qlanes - 1)) == 0;
            const int sj = j / qlanes;
            if constexpr (V == 4) {
                const float4* st = tile + q * d;
                const int jx = j & 7;
                float v[4][8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 t = st[8 * j + (k ^ jx)];
                    v[0][k] = t.x, v[1][k] = t.y, v[2][k] = t.z, v[3][k] = t.w;
                }
                quant_rows<4>(v, min(4, nr - 4 * q), dst + (4 * q) * ld + 8 * j, ld, sdst + (4 * q) * ld_s + sj,
                              ld_s, qlanes, amask, lead);
            } else {
                float v[1][8];
                load8(tile + q * d + slot<1>(8 * j, mask), v[0]);
                quant_rows<1>(v, 1, dst + q * ld + 8 * j, ld, sdst + q * ld_s + sj, ld_s, qlanes, amask, lead);
            }
        }
    }
}

// CL = 1: one CTA holds whole rows.  CL = 2 (slab mode, schedules whose last radix is 2):
// a cluster of two CTAs shares each tile, CTA r holding columns [r d/2, (r+1) d/2) of its
// rows; stages 0..m-2 stay inside a slab, the last one is cross_stage.
// FUSED: a stage runs inside the fill or the drain (p.fuse_first / p.fuse_last); a kernel of its
// own, so that the kernels without fused stages carry none of their code and registers.
template <typename TIn, typename TOut, bool INV, int MASK, int V, int NT, int CL, bool FUSED>
__global__ void __launch_bounds__(NT, 1) harp_tiled_kernel(const __grid_constant__ TiledParams p) {
    static_assert(!FUSED || (V == 4 && CL == 1 && NT == 256), "fused stages: whole rows, 4-row sub-tiles, 256 threads");
    extern __shared__ __align__(128) unsigned char smem[];
    using VT = typename VecOf<V>::T;
    const int d = (int)p.pd.d;
    const int m = p.pd.m;
    const int R = p.R;
    const int tid = threadIdx.x;
    const uint32_t rank = CL == 2 ? cluster_rank() : 0;
    const int dl = d / CL;                  // coordinates of a row held by this CTA
    const int col0 = (int)rank * dl;
    const int m_local = CL == 2 ? m - 1 : m;
    VT* tile = (VT*)smem;
    unsigned char* stage_buf = smem + (size_t)R * dl * sizeof(float);
    uint64_t* bar = (uint64_t*)(stage_buf + (size_t)p.staged_rows * dl * sizeof(TIn));

    int64_t t_idx = blockIdx.x / CL;
    const int64_t t_step = gridDim.x / CL;
    if (t_idx >= p.ntiles) return;          // both CTAs of a cluster have the same t_idx
    if (p.staged_rows) {
        if (tid == 0) mbar_init(bar, 1);
        __syncthreads();
        if (tid == 0) issue_tile<TIn>(p, t_idx, dl, col0, stage_buf, bar);
    }
    // local stages in order: forward 0..m_local-1, inverse m_local-1..0; each stage's first
    // block is requested before the barrier that precedes the stage
    float w[64];
    // stages fused into the fill / drain (4-row sub-tiles of whole rows only) are not run here
    constexpr bool fused = FUSED;
    const int step0 = fused && p.fuse_first ? 1 : 0;
    const int step1 = m_local - (fused && p.fuse_last ? 1 : 0);
    const int t_first = INV ? m_local - 1 - step0 : step0;
    auto sb_of = [&](int t) { return p.lanes + p.lane_off[t] + (int64_t)rank * dl * p.pd.st[t].b; };
    // Without fused stages the first block is requested early (before the loop, and before the
    // drain of the previous tile), so its latency hides behind the drain and the fill; with them
    // it is requested after the fill, whose fused stage needs the registers.
    constexpr bool early = !FUSED;
    if (early && step0 < step1)
        prefetch_first<MASK, V, NT>(p, t_first, (int)((min((int64_t)R, p.rows - t_idx * R) + V - 1) / V), dl, rank,
                                    w);
    auto local_stages = [&](int qv) {
        for (int step = step0; step < step1; ++step) {
            const int t = INV ? m_local - 1 - step : step;
            const StageDesc& sd = p.pd.st[t];
            // the slab's blocks of stage t start at block r dl / b_t
            const float* sb = p.lanes + p.lane_off[t] + (int64_t)rank * dl * sd.b;
            const int s = (int)sd.s;
            switch (sd.b) {
#define HARP_TILED_CASE(RB)                                                                         \
    case RB:                                                                                        \
        if constexpr ((MASK >> RB) & 1)                                                             \
            run_stage<RB, INV, V, NT>(sb, s, p.nb_div[t], p.s_div[t], tile, dl, qv, p.mask, w);    \
        break;
                HARP_TILED_CASE(2) HARP_TILED_CASE(3) HARP_TILED_CASE(4) HARP_TILED_CASE(5)
                HARP_TILED_CASE(6) HARP_TILED_CASE(7) HARP_TILED_CASE(8)
#undef HARP_TILED_CASE
                default: break;
            }
            if (step + 1 < step1) prefetch_first<MASK, V, NT>(p, INV ? t - 1 : t + 1, qv, dl, rank, w);
            __syncthreads();
        }
    };
    uint32_t parity = 0;
    bool failed = false;    // a bounded wait gave up: keep every barrier, skip the waits
    for (; t_idx < p.ntiles; t_idx += t_step) {
        const int64_t row0 = t_idx * R;
        const int nr = (int)min((int64_t)R, p.rows - row0);
        const int qv = (nr + V - 1) / V;
        const int n_staged = min(nr, p.staged_rows);
        if constexpr (FUSED) {
            // w's value from the last tile is dead (the first stage's block is requested after
            // the fill): saying so leaves its registers to the fused fill and drain
#pragma unroll
            for (int k = 0; k < 64; ++k) w[k] = 0.f;
        }
        if (n_staged && !failed) {
            bool ok = mbar_wait(bar, parity, p.wait_limit);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) atomicExch(p.status, 1);
                if (p.extra_tx) {
                    // the test hook's over-declared bytes: retire them, then wait (bounded)
                    // for the copies that were really issued, and go on with correct data
                    if (tid == 0) mbar_complete_tx(bar, p.extra_tx);
                    ok = mbar_wait(bar, parity, kWaitLimit);
                    failed = __syncthreads_or(!ok);
                } else {
                    failed = true;
                }
            }
            parity ^= 1;
        }
        if constexpr (FUSED) {
            if (p.fuse_first)
                fill_tile_fused<NT, TIn, INV>((float4*)tile, dl, nr, n_staged, (const TIn*)stage_buf,
                                              (const TIn*)p.x + row0 * p.ld_x + col0, p.ld_x, p.fuse_first,
                                              sb_of(INV ? m_local - 1 : 0));
            else
                fill_tile<V, NT, TIn>(tile, dl, nr, n_staged, (const TIn*)stage_buf,
                                      (const TIn*)p.x + row0 * p.ld_x + col0, p.ld_x, p.mask);
        } else {
            fill_tile<V, NT, TIn>(tile, dl, nr, n_staged, (const TIn*)stage_buf, (const TIn*)p.x + row0 * p.ld_x + col0,
                                  p.ld_x, p.mask);
        }
        if (!early && step0 < step1) prefetch_first<MASK, V, NT>(p, t_first, qv, dl, rank, w);
        __syncthreads();
        const int64_t t_next = t_idx + t_step;
        if (p.staged_rows && tid == 0 && t_next < p.ntiles && !failed) {
            fence_proxy_async_smem();   // the staging reads above happen before the copies' writes
            issue_tile<TIn>(p, t_next, dl, col0, stage_buf, bar);
        }
        if constexpr (CL == 2) {
            if (!INV) local_stages(qv);
            cluster_sync();             // both slabs of the tile are ready
            cross_stage<INV, NT>((float4*)tile, dl, qv, rank, p.last_blocks);
            cluster_sync();             // the partner's writes into this tile are visible
            if (INV) local_stages(qv);
        } else {
            local_stages(qv);
        }
        if (early && t_next < p.ntiles && step0 < step1)   // the next tile's, in flight during drain and fill
            prefetch_first<MASK, V, NT>(p, t_first, (int)((min((int64_t)R, p.rows - t_next * R) + V - 1) / V), dl,
                                        rank, w);
        if constexpr (std::is_same<TOut, int8_t>::value)
            drain_tile_quant<V, NT>(tile, dl, nr, (int8_t*)p.y + row0 * p.ld_y, p.ld_y, p.mask,
                                    p.scales + row0 * p.ld_s, p.ld_s, p.qlanes);
        else if constexpr (FUSED) {
            if (p.fuse_last)
                drain_tile_fused<NT, TOut, INV>((const float4*)tile, dl, nr, (TOut*)p.y + row0 * p.ld_y + col0,
                                                p.ld_y, p.fuse_last, sb_of(INV ? 0 : m_local - 1));
            else
                drain_tile<V, NT, TOut>(tile, dl, nr, (TOut*)p.y + row0 * p.ld_y + col0, p.ld_y, p.mask);
        } else {
            drain_tile<V, NT, TOut>(tile, dl, nr, (TOut*)p.y + row0 * p.ld_y + col0, p.ld_y, p.mask);
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

// Sub-tiles of one row (V = 1) are needed only when four fp32 rows do not fit in shared
// memory (d > 14524); they are built for the radix sets without 5.
constexpr bool has_row_major_kernel(int mask) { return ((mask >> 5) & 1) == 0; }

// Threads per CTA: 384 (12 warps, at most 168 registers) when every stage splits evenly
// over them without dividing the tile's sub-tiles between items; else 256.
constexpr int kThreadChoices[] = {256, 384};

// Slab-mode kernels exist for the radix sets that contain 2.
constexpr bool has_slab_kernel(int mask) { return ((mask >> 2) & 1) != 0 && mask != 0x1fc; }

template <typename TIn, typename TOut, bool INV, int V, int NT, int CL, int I, bool FUSED = false>
cudaError_t launch_mask(int which, const TiledParams& tp, size_t smem, int grid, cudaStream_t stream) {
    if constexpr (I < kNumMasks) {
        if (which != I) return launch_mask<TIn, TOut, INV, V, NT, CL, I + 1, FUSED>(which, tp, smem, grid, stream);
        if constexpr ((V == 1 && !has_row_major_kernel(kMasks[I])) ||
                      (CL == 2 && (V != 4 || !has_slab_kernel(kMasks[I]) || std::is_same<TOut, int8_t>::value))) {
            return cudaErrorInvalidValue;
        } else {
            auto kern = harp_tiled_kernel<TIn, TOut, INV, kMasks[I], V, NT, CL, FUSED>;
            cudaError_t e = (cudaError_t)harp_set_smem_limit((const void*)kern, (int)smem);
            if (e != cudaSuccess) return e;
            if constexpr (CL == 1) {
                kern<<<(unsigned)grid, NT, smem, stream>>>(tp);
            } else {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3((unsigned)grid);
                cfg.blockDim = dim3(NT);
                cfg.dynamicSmemBytes = smem;
                cfg.stream = stream;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = 2;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                e = cudaLaunchKernelEx(&cfg, kern, tp);
                if (e != cudaSuccess) return e;
            }
            return cudaGetLastError();
        }
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename TIn, typename TOut, bool INV, int V>
cudaError_t launch_nt(int which, int nt, int cl, const TiledParams& tp, size_t smem, int grid, cudaStream_t stream) {
    if constexpr (V == 4) {
        if (tp.fuse_first || tp.fuse_last) {
            if (nt != 256 || cl != 1) return cudaErrorInvalidValue;
            return launch_mask<TIn, TOut, INV, 4, 256, 1, 0, true>(which, tp, smem, grid, stream);
        }
    }
    if (cl == 2) {
        if (nt == 384) return launch_mask<TIn, TOut, INV, V, 384, 2, 0>(which, tp, smem, grid, stream);
        return launch_mask<TIn, TOut, INV, V, 256, 2, 0>(which, tp, smem, grid, stream);
    }
    if (nt == 384) return launch_mask<TIn, TOut, INV, V, 384, 1, 0>(which, tp, smem, grid, stream);
    return launch_mask<TIn, TOut, INV, V, 256, 1, 0>(which, tp, smem, grid, stream);
}

template <typename TIn, typename TOut>
cudaError_t launch(int which, int V, int nt, int cl, bool inverse, const TiledParams& tp, size_t smem, int grid,
                   cudaStream_t stream) {
    if (V == 4)
        return inverse ? launch_nt<TIn, TOut, true, 4>(which, nt, cl, tp, smem, grid, stream)
                       : launch_nt<TIn, TOut, false, 4>(which, nt, cl, tp, smem, grid, stream);
    return inverse ? launch_nt<TIn, TOut, true, 1>(which, nt, cl, tp, smem, grid, stream)
                   : launch_nt<TIn, TOut, false, 1>(which, nt, cl, tp, smem, grid, stream);
}

}  // namespace harp_tiled

// One translation unit per I/O type pair (compiled in parallel).
cudaError_t harp_tiled_launch_bf16(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                   size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_f32(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                  size_t smem, int grid, cudaStream_t stream);
cudaError_t harp_tiled_launch_bf16_f32(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                       size_t smem, int grid, cudaStream_t stream);
// bf16 rows in, int8 codes and per-block fp32 scales out (the fused quantizer epilogue)
cudaError_t harp_tiled_launch_bf16_i8(int which, int V, int nt, int cl, bool inverse, const harp_tiled::TiledParams& tp,
                                      size_t smem, int grid, cudaStream_t stream);
