// Specialized row kernel for the HARP transform at d = 4096, schedule (8,8,8,8),
// bf16 rows, forward direction (HARP technical summary §2.1 Core Architecture,
// §2.2 Hadamard Preconditioning).
//
// Digits: coordinate i = i0 + 8 i1 + 64 i2 + 512 i3.  Stage t mixes digit t.
// Write a = i0 + 8 i1 ("pencil", low digits) and beta = i2 + 8 i3 ("chunk", high
// digits): stages 0,1 act inside each contiguous 64-coordinate chunk beta, stages
// 2,3 inside each stride-64 pencil a.
//
// Work split: a cluster of two CTAs (one per SM) owns a 16-row tile.  CTA r runs
// phase A on chunks beta in [32r, 32r+32) and phase B on pencils a in [32r, 32r+32);
// between the phases each CTA sends the partner its half of the fp32 intermediate
// with one 64 KB bulk copy (TMA engine, shared::cluster) completed on the
// partner's mbarrier.
//
// Inner engine, per phase:
//   * first stage: tensor cores, mma.sync m16n8k8 TF32 with the 16 tile rows as M,
//     the 8 inputs of a group as K and its 8 outputs as N.  fp32 accuracy comes
//     from splitting operands into TF32 hi + lo parts (round to nearest) and
//     summing hi*hi + hi*lo + lo*hi; bf16 input is exact in TF32, so stage 0 needs
//     only hi*hi + hi*lo.  Operand and output slots are permuted so that each lane
//     ends up holding complete groups of the next stage.
//   * second stage: plain fp32 FMA in each lane on the groups it already holds.
// Every shared-memory access pattern below is XOR-swizzled to be bank-conflict
// free; the derivations are next to each index function.
#include <cstdio>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "harp_internal.h"

namespace {

constexpr int kD = 4096;
constexpr int kTile = 16;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kEFloats = 2 * 16 * 32 * 32;   // exchange tile E[half][row][a_local][pos]
constexpr int kSFloats = 16 * 32 * 32;       // send buffer S[row][a_local][pos], reused as bf16 output staging
constexpr int kHalfBytes = kSFloats * 4;     // 65536
constexpr int kXBytes = 16 * 128;            // one 16-row x 64-column bf16 input box per warp
constexpr int kXOffset = (kEFloats + kSFloats) * 4;          // 196608, 1024-aligned
constexpr int kBarOffset = kXOffset + kWarps * kXBytes;      // 229376
constexpr size_t kSmemBytes = (size_t)kBarOffset + 8 * (kWarps + 1) + 1024;   // + alignment slack
constexpr long long kWaitLimit = 1ll << 26;  // mbarrier polls before giving up

struct FastParams {
    __nv_bfloat16* y;
    int64_t rows, ldy;       // ldy in elements
    int ntiles;
    const float2* pk0;       // stage-0 B fragments, [block][lane]
    const float4* pk1;       // stage-1 blocks, lane-interleaved (see pack_interleaved_kernel)
    const float2* pk2;       // stage-2 B fragments
    const float4* pk3;       // stage-3 blocks, lane-interleaved
    int* status;
};

// ----------------------------------------------------------------- PTX ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// x = hi + lo with both parts TF32 (round to nearest): |x - hi - lo| <= 2^-22 |x|
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two independent fp32 fused multiply-adds (round to nearest) on register pairs.
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ unsigned long long pair(float lo, float hi) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ float2 unpair(unsigned long long v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}

// y[o] = sum_l B[o][l] x[l] for the 8 outputs of one block and two rows (A, B), with the
// block read as 16 float4 = (B[2p][2k], B[2p+1][2k], B[2p][2k+1], B[2p+1][2k+1]) at
// cf[(p * 4 + k) * 4] (p = output pair, k = input pair), four lanes apart.  Output pairs
// (2p, 2p+1) accumulate in f32x2 registers; each row's inputs are duplicated once.
__device__ __forceinline__ void block_matvec_2rows(const float4* __restrict__ cf, const float (&xa)[8],
                                                   const float (&xb)[8], float (&ya)[8], float (&yb)[8]) {
    unsigned long long da[8], db[8];
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        da[l] = pair(xa[l], xa[l]);
        db[l] = pair(xb[l], xb[l]);
    }
    float4 cur[4], nxt[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) cur[k] = __ldg(cf + k * 4);
#pragma unroll
    for (int op = 0; op < 4; ++op) {
        if (op < 3) {
#pragma unroll
            for (int k = 0; k < 4; ++k) nxt[k] = __ldg(cf + ((op + 1) * 4 + k) * 4);
        }
        unsigned long long accA = 0ull, accB = 0ull;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const unsigned long long c0 = pair(cur[k].x, cur[k].y);   // (B[2op][2k],   B[2op+1][2k])
            const unsigned long long c1 = pair(cur[k].z, cur[k].w);   // (B[2op][2k+1], B[2op+1][2k+1])
            accA = ffma2(c0, da[2 * k], accA);
            accB = ffma2(c0, db[2 * k], accB);
            accA = ffma2(c1, da[2 * k + 1], accA);
            accB = ffma2(c1, db[2 * k + 1], accB);
        }
        const float2 ra = unpair(accA), rb = unpair(accB);
        ya[2 * op] = ra.x; ya[2 * op + 1] = ra.y;
        yb[2 * op] = rb.x; yb[2 * op + 1] = rb.y;
        if (op < 3) {
#pragma unroll
            for (int k = 0; k < 4; ++k) cur[k] = nxt[k];
        }
    }
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait for the phase with the given parity; returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    for (long long i = 0; i < kWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; "
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

__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst, const void* src, uint32_t bytes,
                                                     uint32_t remote_bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "r"(smem_u32(src)), "r"(bytes), "r"(remote_bar)
        : "memory");
}

// 2-D tiled TMA load of one box into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int col, int row, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(col), "r"(row), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------ shared layouts ---
//
// E[half][beta_local][row][pos]: half = beta >> 5 (the CTA whose chunks produced it),
// beta_local = beta & 31, a_local = pencil index inside the owning CTA (a = 32 r + a_local)
// and pos = a_local ^ swz(row, beta) with swz = ((row & 7) << 2) | (beta & 3).
//  - phase A stores one scalar per lane with beta fixed, row = g (+8), a_local = q + 4s + 8o':
//    a_local ^ (4g + c) has q ^ c in bits 0-1 and g ^ (s + 2o') in bits 2-4, 32 banks.
//  - phase B loads one scalar per lane with a_local fixed, row = g (+8) and beta = q + 8m (+4),
//    so beta & 3 = q: a_local ^ (4g + q) is a permutation of 0..31, 32 banks.
// Each chunk's 16 x 32 block is contiguous (2 KB), so the part of it bound for the partner
// CTA is sent with one bulk copy as soon as the warp has produced it.
__device__ __forceinline__ int e_index(int half, int row, int a_local, int beta) {
    const int swz = ((row & 7) << 2) | (beta & 3);
    return ((half * 32 + (beta & 31)) * 16 + row) * 32 + (a_local ^ swz);
}

__device__ __forceinline__ int s_index(int row, int a_local, int beta) {
    const int swz = ((row & 7) << 2) | (beta & 3);
    return ((beta & 31) * 16 + row) * 32 + (a_local ^ swz);
}

// Output staging O[row][a_local][beta'] (bf16) with beta' = 8 i2 + i3, stored in 16-byte
// chunks indexed by i2 ^ h, h = 2 ((a_local >> 3) & 3) ^ 4 (row & 1).
//  - phase B stores a 16-byte chunk per lane (a_local fixed, i2 = q + 4s, rows 2k and 2k+1
//    in a quarter-warp): the row bit moves the chunk to the other half, 8 distinct chunks.
//  - the store phase loads one word per thread with the row fixed, 8 consecutive beta'
//    pairs and the 4 pencil quarters u = a_local >> 3: chunks (p >> 2) ^ 2u are 8 distinct
//    values and p & 3 selects the word, 32 distinct banks.
__device__ __forceinline__ int o_byte(int row, int a_local, int i2, int i3) {
    const int chunk = i2 ^ ((((a_local >> 3) & 3) << 1) ^ ((row & 1) << 2));
    return ((row * 32 + a_local) * 64 + chunk * 8 + i3) * 2;
}

// Input staging: TMA writes a 16 x 128-byte box with the 128-byte swizzle, i.e. the
// 16-byte chunk c of row r sits at chunk position c ^ (r & 7).  The lane that needs
// elements 8j + 2q, 8j + 2q + 1 of row g reads word q of chunk j ^ g: 32 distinct banks.
__device__ __forceinline__ int x_byte(int row, int j, int q) {
    return row * 128 + ((j ^ (row & 7)) << 4) + 4 * q;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------- kernel ---

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    harp_fast_d4096_fwd_kernel(const __grid_constant__ CUtensorMap tmap_x, FastParams p) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled TMA boxes
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* E = reinterpret_cast<float*>(base);
    float* S = E + kEFloats;
    unsigned char* O = reinterpret_cast<unsigned char*>(S);
    unsigned char* X = base + kXOffset;
    uint64_t* xbar = reinterpret_cast<uint64_t*>(base + kBarOffset);   // one per warp
    uint64_t* bar = xbar + kWarps;                                      // exchange

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int r = (int)cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    unsigned char* Xw = X + warp * kXBytes;

    if (tid == 0) mbar_init(bar, 1);
    if (lane == 0) mbar_init(xbar + warp, 1);
    const uint32_t remote_e = map_to_rank(smem_u32(E + r * kSFloats), (uint32_t)(r ^ 1));   // partner's half r
    const uint32_t remote_bar = map_to_rank(smem_u32(bar), (uint32_t)(r ^ 1));
    cluster_arrive();
    cluster_wait();     // barriers initialised on both CTAs
    cluster_arrive();   // "my E may be written": matched by the wait before the first send

    // first input box of this warp: tile `pair`, task 0
    if (lane == 0 && pair < p.ntiles) {
        mbar_arrive_expect_tx(xbar + warp, kXBytes);
        tma_load_2d(Xw, &tmap_x, 64 * (32 * r + 2 * warp), pair * kTile, xbar + warp);
    }
    uint32_t xparity = 0, parity = 0;

    for (int tile = pair; tile < p.ntiles; tile += npairs) {
        const int64_t row0 = (int64_t)tile * kTile;
        if (tid == 0) mbar_arrive_expect_tx(bar, kHalfBytes);
        cluster_wait();               // the partner has finished reading its E (previous tile)

        // -------------------------------------------------- phase A ---
#pragma unroll 1
        for (int task = 0; task < 2; ++task) {
            const int beta = 32 * r + 2 * warp + task;
            if (!mbar_wait(xbar + warp, xparity) && lane == 0) atomicExch(p.status, 1);
            xparity ^= 1;
            uint32_t w0[8], w1[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // elements 8j + 2q, 8j + 2q + 1 of rows g, g + 8
                w0[j] = *reinterpret_cast<const uint32_t*>(Xw + x_byte(g, j, q));
                w1[j] = *reinterpret_cast<const uint32_t*>(Xw + x_byte(g + 8, j, q));
            }
            // stage 0 on tensor cores: group j = i1, slot q <-> i0 = 2q, slot q+4 <-> i0 = 2q+1;
            // output slot 2q <-> i0 = q, 2q+1 <-> i0 = q + 4.
            float z[8][4];
            float2 bf[8];             // all eight B fragments in flight before the first mma
#pragma unroll
            for (int j = 0; j < 8; ++j) bf[j] = __ldg(p.pk0 + (size_t)(j + 8 * beta) * 32 + lane);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t a[4] = {w0[j] << 16, w1[j] << 16, w0[j] & 0xffff0000u, w1[j] & 0xffff0000u};
                const float2 bb = bf[j];
                uint32_t bh0, bl0, bh1, bl1;
                split_tf32(bb.x, bh0, bl0);
                split_tf32(bb.y, bh1, bl1);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tf32(d, a, bh0, bh1);
                mma_tf32(d, a, bl0, bl1);
#pragma unroll
                for (int e = 0; e < 4; ++e) z[j][e] = d[e];
            }
            // every lane has consumed its words: refill the box with the second chunk of this
            // tile, or the first chunk of the next tile
            __syncwarp();
            if (lane == 0) {
                const int ntile = task == 0 ? tile : tile + npairs;
                if (ntile < p.ntiles) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(xbar + warp, kXBytes);
                    tma_load_2d(Xw, &tmap_x, 64 * (32 * r + 2 * warp + (task ^ 1)), ntile * kTile, xbar + warp);
                }
            }
            // stage 1 in registers: this lane holds i1 = 0..7 of groups i0 = q + 4s for rows g, g+8
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                float xa[8], xb[8], ya[8], yb[8];
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    xa[l] = z[l][s];
                    xb[l] = z[l][s + 2];
                }
                block_matvec_2rows(p.pk1 + (size_t)(beta * 2 + s) * 64 + q, xa, xb, ya, yb);
#pragma unroll
                for (int o = 0; o < 8; ++o) {
                    // coordinate (i0 = q + 4s, i1 = o, beta): pencil a_local = i0 + 8 (o & 3) of CTA o >> 2
                    const int a_local = (q + 4 * s) + 8 * (o & 3);
                    if ((o >> 2) == r) {
                        E[e_index(r, g, a_local, beta)] = ya[o];
                        E[e_index(r, g + 8, a_local, beta)] = yb[o];
                    } else {
                        S[s_index(g, a_local, beta)] = ya[o];
                        S[s_index(g + 8, a_local, beta)] = yb[o];
                    }
                }
            }
            // this chunk's partner-bound 2 KB goes out now, overlapping the rest of phase A
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int off = (beta & 31) * 16 * 32;
                bulk_copy_to_cluster(remote_e + off * 4, S + off, 16 * 32 * 4, remote_bar);
            }
        }

        // --------------------------------------------------- exchange ---
        __syncthreads();              // local E writes of all warps
        if (!mbar_wait(bar, parity) && lane == 0) atomicExch(p.status, 1);   // partner's 32 chunks
        parity ^= 1;
        cluster_arrive();             // both copies have landed: S may be reused
        cluster_wait();

        // --------------------------------------------------- phase B ---
#pragma unroll 1
        for (int task = 0; task < 2; ++task) {
            const int a_local = 2 * warp + task;
            const int a = 32 * r + a_local;
            // stage 2 on tensor cores: group m = i3, slot q <-> i2 = q, slot q+4 <-> i2 = q + 4;
            // output slot 2q <-> i2 = q, 2q+1 <-> i2 = q + 4.
            float z2[8][4];
            float2 bf[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) bf[m] = __ldg(p.pk2 + (size_t)(a + 64 * m) * 32 + lane);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int half = m >> 2;
                const int b0 = q + 8 * m, b1 = q + 4 + 8 * m;
                const float v[4] = {E[e_index(half, g, a_local, b0)], E[e_index(half, g + 8, a_local, b0)],
                                    E[e_index(half, g, a_local, b1)], E[e_index(half, g + 8, a_local, b1)]};
                uint32_t ah[4], al[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) split_tf32(v[e], ah[e], al[e]);
                const float2 bb = bf[m];
                uint32_t bh0, bl0, bh1, bl1;
                split_tf32(bb.x, bh0, bl0);
                split_tf32(bb.y, bh1, bl1);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tf32(d, ah, bh0, bh1);
                mma_tf32(d, ah, bl0, bl1);
                mma_tf32(d, al, bh0, bh1);
#pragma unroll
                for (int e = 0; e < 4; ++e) z2[m][e] = d[e];
            }
            // stage 3 in registers: groups i2 = q + 4s, inputs i3 = 0..7
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int i2 = q + 4 * s;
                float xa[8], xb[8], yA[8], yB[8];
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    xa[l] = z2[l][s];
                    xb[l] = z2[l][s + 2];
                }
                block_matvec_2rows(p.pk3 + (size_t)(a * 2 + s) * 64 + q, xa, xb, yA, yB);
                const uint4 pa = make_uint4(pack_bf16x2(yA[0], yA[1]), pack_bf16x2(yA[2], yA[3]),
                                            pack_bf16x2(yA[4], yA[5]), pack_bf16x2(yA[6], yA[7]));
                const uint4 pb = make_uint4(pack_bf16x2(yB[0], yB[1]), pack_bf16x2(yB[2], yB[3]),
                                            pack_bf16x2(yB[4], yB[5]), pack_bf16x2(yB[6], yB[7]));
                *reinterpret_cast<uint4*>(O + o_byte(g, a_local, i2, 0)) = pa;
                *reinterpret_cast<uint4*>(O + o_byte(g + 8, a_local, i2, 0)) = pb;
            }
        }
        __syncthreads();
        cluster_arrive();             // my E has been read: the partner may send the next tile

        // ------------------------------------------------------ store ---
        // work item (row, p, u): beta' pair p = (2p, 2p+1), pencil quarter u = a_local >> 3.
        // Eight word loads give the 8 pencils of the quarter for both beta'; each becomes a
        // 16-byte piece of a 64-byte output run.  A warp covers one row, 8 pairs, 4 quarters,
        // so each 16-byte store instruction writes 8 whole runs.
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int item = tid + kThreads * it;
            const int row = item >> 7, pp = (item >> 2) & 31, u = item & 3;
            const int64_t grow = row0 + row;
            if (grow < p.rows) {
                const int i2 = pp >> 2, i3 = 2 * (pp & 3);
                uint32_t wv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    wv[k] = *reinterpret_cast<const uint32_t*>(O + o_byte(row, 8 * u + k, i2, i3));
                const uint4 r0 = make_uint4(__byte_perm(wv[0], wv[1], 0x5410), __byte_perm(wv[2], wv[3], 0x5410),
                                            __byte_perm(wv[4], wv[5], 0x5410), __byte_perm(wv[6], wv[7], 0x5410));
                const uint4 r1 = make_uint4(__byte_perm(wv[0], wv[1], 0x7632), __byte_perm(wv[2], wv[3], 0x7632),
                                            __byte_perm(wv[4], wv[5], 0x7632), __byte_perm(wv[6], wv[7], 0x7632));
                __nv_bfloat16* yrow = p.y + grow * p.ldy + 32 * r + 8 * u;
                *reinterpret_cast<uint4*>(yrow + 64 * (i2 + 8 * i3)) = r0;
                *reinterpret_cast<uint4*>(yrow + 64 * (i2 + 8 * (i3 + 1))) = r1;
            }
        }
        __syncthreads();              // O (= S) read before the next tile's phase A writes S
    }
    cluster_wait();                   // matches the last arrive; no bulk copy is in flight
}

// B fragments of a block for mma.m16n8k8 (lane L = 4 g + q):
//   b0 = B[q][g], b1 = B[q + 4][g] with B[k][n] = Blk[out(n)][in(k)],
//   out(n) = n / 2 for even n, n / 2 + 4 for odd n,
//   stage 0: in(q) = 2q, in(q + 4) = 2q + 1;   stage 2: in(k) = k.
__global__ void pack_fragments_kernel(const float* __restrict__ blk, float2* __restrict__ out, int nblocks,
                                      int interleaved_inputs) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nblocks * 32) return;
    const int c = gid >> 5, L = gid & 31;
    const int g = L >> 2, q = L & 3;
    const int o = (g & 1) ? (g >> 1) + 4 : (g >> 1);
    const int k0 = interleaved_inputs ? 2 * q : q;
    const int k1 = interleaved_inputs ? 2 * q + 1 : q + 4;
    const float* b = blk + (size_t)c * 64;
    out[gid] = make_float2(b[o * 8 + k0], b[o * 8 + k1]);
}

// Lane-interleaved copy of the blocks of a register stage, so that the four lanes
// q = 0..3 of a quad, which work on blocks whose index differs by `qstride`, read one
// contiguous 64-byte run per instruction, and each float4 holds two output pairs:
//   out[(((h * 2 + s) * 4 + p) * 4 + k) * 4 + q] =
//       (B[2p][2k], B[2p+1][2k], B[2p][2k+1], B[2p+1][2k+1])   of block
//   c = h * head_mul + (q + 4 s) * qstride   (stage 1: chunk h, c = 8h + i0;  stage 3: pencil h, c = h + 64 i2).
__global__ void pack_interleaved_kernel(const float* __restrict__ blk, float4* __restrict__ out, int nheads,
                                        int head_mul, int qstride) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nheads * 128) return;
    const int q = gid & 3, k = (gid >> 2) & 3, pr = (gid >> 4) & 3, s = (gid >> 6) & 1, h = gid >> 7;
    const int c = h * head_mul + (q + 4 * s) * qstride;
    const float* b = blk + (size_t)c * 64;
    out[gid] = make_float4(b[(2 * pr) * 8 + 2 * k], b[(2 * pr + 1) * 8 + 2 * k], b[(2 * pr) * 8 + 2 * k + 1],
                           b[(2 * pr + 1) * 8 + 2 * k + 1]);
}

struct FastState {
    float2* pk0 = nullptr;
    float2* pk2 = nullptr;
    float4* pk1 = nullptr;
    float4* pk3 = nullptr;
    int max_pairs = 0;
    bool ready = false;
};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool is_d4096_radix8(const harp_plan_s* p) {
    if (p->desc.d != kD || p->desc.m != 4) return false;
    for (int t = 0; t < 4; ++t)
        if (p->desc.st[t].b != 8) return false;
    return true;
}

harp_status prepare(harp_plan_s* p, cudaStream_t stream) {
    FastState* fs = static_cast<FastState*>(p->fast);
    if (fs && fs->ready) return HARP_OK;
    if (!fs) {
        fs = new FastState();
        p->fast = fs;
    }
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        cudaGetLastError();
    });
    if (!g_encode) return harp_fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const int nblocks = kD / 8;
    if ((!fs->pk0 && cudaMalloc((void**)&fs->pk0, sizeof(float2) * nblocks * 32) != cudaSuccess) ||
        (!fs->pk2 && cudaMalloc((void**)&fs->pk2, sizeof(float2) * nblocks * 32) != cudaSuccess) ||
        (!fs->pk1 && cudaMalloc((void**)&fs->pk1, sizeof(float4) * nblocks * 16) != cudaSuccess) ||
        (!fs->pk3 && cudaMalloc((void**)&fs->pk3, sizeof(float4) * nblocks * 16) != cudaSuccess)) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the fragment tables failed");
    }
    const int threads = 256, grid = (nblocks * 32 + threads - 1) / threads;
    const float* blocks = p->d_blocks;
    pack_fragments_kernel<<<grid, threads, 0, stream>>>(blocks + p->desc.st[0].block_off, fs->pk0, nblocks, 1);
    pack_fragments_kernel<<<grid, threads, 0, stream>>>(blocks + p->desc.st[2].block_off, fs->pk2, nblocks, 0);
    // stage 1: block c = i0 + 8 beta, i0 = q + 4s;  stage 3: block c = a + 64 i2, i2 = q + 4s
    pack_interleaved_kernel<<<(64 * 128 + threads - 1) / threads, threads, 0, stream>>>(
        blocks + p->desc.st[1].block_off, fs->pk1, 64, 8, 1);
    pack_interleaved_kernel<<<(64 * 128 + threads - 1) / threads, threads, 0, stream>>>(
        blocks + p->desc.st[3].block_off, fs->pk3, 64, 1, 64);
    cudaError_t e = cudaFuncSetAttribute(harp_fast_d4096_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    int nclusters = 0;
    e = cudaOccupancyMaxActiveClusters(&nclusters, (void*)harp_fast_d4096_fwd_kernel, &cfg);
    if (e != cudaSuccess || nclusters < 1) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no cluster of two fits on this device");
    }
    fs->max_pairs = nclusters;
    e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    fs->ready = true;
    return HARP_OK;
}

}  // namespace

harp_status launch_apply_fast(harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                              int64_t ld_y, harp_dtype in_dtype, harp_dir dir, void* stream_,
                              harp_dtype out_dtype) {
    if (!is_d4096_radix8(p) || in_dtype != HARP_BF16 || out_dtype != HARP_BF16 || dir != HARP_FORWARD)
        return HARP_ERR_UNSUPPORTED;
    // TMA input boxes need 16-byte aligned rows; output runs are 16-byte stores
    if (((uintptr_t)x & 15) || (ld_x & 7) || ((uintptr_t)y & 15) || (ld_y & 7)) return HARP_ERR_UNSUPPORTED;
    if (rows < 32 || rows > 0x7fffffffll) return HARP_ERR_UNSUPPORTED;
    cudaStream_t stream = (cudaStream_t)stream_;
    harp_status st = prepare(p, stream);
    if (st != HARP_OK) return st;
    FastState* fs = static_cast<FastState*>(p->fast);
    const int64_t ntiles = (rows + kTile - 1) / kTile;
    const int pairs = (int)std::min<int64_t>(fs->max_pairs, ntiles);

    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld_x * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box,
                           estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return harp_fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)cr));

    FastParams fp;
    fp.y = reinterpret_cast<__nv_bfloat16*>(y);
    fp.rows = rows;
    fp.ldy = ld_y;
    fp.ntiles = (int)ntiles;
    fp.pk0 = fs->pk0;
    fp.pk1 = fs->pk1;
    fp.pk2 = fs->pk2;
    fp.pk3 = fs->pk3;
    fp.status = p->d_status;
    harp_fast_d4096_fwd_kernel<<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_fast_d4096_fwd_kernel");
    return HARP_OK;
}

void fast_state_free(harp_plan_s* p) {
    FastState* fs = static_cast<FastState*>(p->fast);
    if (!fs) return;
    cudaFree(fs->pk0);
    cudaFree(fs->pk1);
    cudaFree(fs->pk2);
    cudaFree(fs->pk3);
    delete fs;
    p->fast = nullptr;
}
