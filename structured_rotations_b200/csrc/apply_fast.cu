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

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kD = 4096;
constexpr int kTile = 16;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kEFloats = 2 * 16 * 32 * 32;   // exchange tile E[half][row][a_local][pos]
constexpr int kSFloats = 16 * 32 * 32;       // send buffer S[row][a_local][pos], reused as bf16 output staging
constexpr int kHalfBytes = kSFloats * 4;     // 65536
constexpr size_t kSmemBytes = (size_t)(kEFloats + kSFloats) * 4 + 64;
constexpr long long kWaitLimit = 1ll << 26;  // mbarrier polls before giving up

struct FastParams {
    const uint32_t* x;       // bf16 rows viewed as 32-bit words (pairs)
    __nv_bfloat16* y;
    int64_t rows, ldx_w, ldy;  // ldx in 32-bit words, ldy in elements
    int ntiles;
    const float2* pk0;       // stage-0 B fragments, [block][lane]
    const float* blk1;       // stage-1 blocks, row-major [block][8][8]
    const float2* pk2;       // stage-2 B fragments
    const float* blk3;       // stage-3 blocks
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

__device__ __forceinline__ uint32_t ldg_nc_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// ------------------------------------------------------ shared layouts ---
//
// E[half][row][a_local][pos]: half = beta >> 5 (the CTA whose chunks produced it),
// a_local = pencil index inside the owning CTA (a = 32 r + a_local), and
// pos = (beta & 31) ^ swz(row, a_local) with swz = ((row & 7) << 2) | (a_local & 3).
//  - phase A stores one scalar per lane with beta fixed, row = g (+8), a_local & 3 = q:
//    banks (beta ^ (4g + q)) mod 32 are 32 distinct values.
//  - phase B loads one scalar per lane with a_local fixed and beta = q + 8m (+4),
//    row = g (+8): (q + 8m) ^ (4g + c) puts q in bits 0-1 and g in bits 2-4, so
//    the 32 lanes again hit 32 distinct banks.
__device__ __forceinline__ int e_index(int half, int row, int a_local, int beta) {
    const int swz = ((row & 7) << 2) | (a_local & 3);
    return ((half * 16 + row) * 32 + a_local) * 32 + ((beta & 31) ^ swz);
}

__device__ __forceinline__ int s_index(int row, int a_local, int beta) {
    const int swz = ((row & 7) << 2) | (a_local & 3);
    return (row * 32 + a_local) * 32 + ((beta & 31) ^ swz);
}

// Output staging O[row][a_local][beta'] (bf16) with beta' = 8 i2 + i3, stored in 16-byte
// chunks indexed by i2 ^ ((row & 1) << 2): a quarter-warp stores rows g in {2k, 2k+1}
// with i2 = q + 4s, which lands in 8 distinct chunks.
__device__ __forceinline__ int o_byte(int row, int a_local, int i2, int i3) {
    const int chunk = i2 ^ ((row & 1) << 2);
    return ((row * 32 + a_local) * 64 + chunk * 8 + i3) * 2;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------- kernel ---

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    harp_fast_d4096_fwd_kernel(FastParams p) {
    extern __shared__ __align__(128) float smem[];
    float* E = smem;
    float* S = smem + kEFloats;
    unsigned char* O = reinterpret_cast<unsigned char*>(S);
    uint64_t* bar = reinterpret_cast<uint64_t*>(S + kSFloats);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int r = (int)cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (tid == 0) mbar_init(bar, 1);
    // the partner's view of our chunk half of its E, and the partner's barrier
    const uint32_t remote_e = map_to_rank(smem_u32(E + r * kSFloats), (uint32_t)(r ^ 1));
    const uint32_t remote_bar = map_to_rank(smem_u32(bar), (uint32_t)(r ^ 1));
    cluster_arrive();
    cluster_wait();     // barrier initialised on both CTAs
    cluster_arrive();   // "my E may be written": matched by the wait before the first send

    uint32_t parity = 0;
    for (int tile = pair; tile < p.ntiles; tile += npairs) {
        const int64_t row0 = (int64_t)tile * kTile;
        if (tid == 0) mbar_arrive_expect_tx(bar, kHalfBytes);

        // -------------------------------------------------- phase A ---
        const int64_t rA = row0 + g, rB = row0 + g + 8;
        const bool vA = rA < p.rows, vB = rB < p.rows;
#pragma unroll 1
        for (int task = 0; task < 2; ++task) {
            const int beta = 32 * r + 2 * warp + task;
            const uint32_t* xa = p.x + rA * p.ldx_w + 32 * beta + q;
            const uint32_t* xb = p.x + rB * p.ldx_w + 32 * beta + q;
            uint32_t w0[8], w1[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // element 8j + 2q (+1) of the chunk
                w0[j] = vA ? ldg_nc_u32(xa + 4 * j) : 0u;
                w1[j] = vB ? ldg_nc_u32(xb + 4 * j) : 0u;
            }
            // stage 0 on tensor cores: group j = i1, slot q <-> i0 = 2q, slot q+4 <-> i0 = 2q+1;
            // output slot 2q <-> i0 = q, 2q+1 <-> i0 = q + 4.
            float z[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t a[4] = {w0[j] << 16, w1[j] << 16, w0[j] & 0xffff0000u, w1[j] & 0xffff0000u};
                const float2 bb = __ldg(p.pk0 + (size_t)(j + 8 * beta) * 32 + lane);
                uint32_t bh0, bl0, bh1, bl1;
                split_tf32(bb.x, bh0, bl0);
                split_tf32(bb.y, bh1, bl1);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tf32(d, a, bh0, bh1);
                mma_tf32(d, a, bl0, bl1);
#pragma unroll
                for (int e = 0; e < 4; ++e) z[j][e] = d[e];
            }
            // stage 1 in registers: this lane holds i1 = 0..7 of groups i0 = q + 4s for rows g, g+8
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const float* blk = p.blk1 + (size_t)((q + 4 * s) + 8 * beta) * 64;
#pragma unroll
                for (int o = 0; o < 8; ++o) {
                    const float4 c0 = __ldg(reinterpret_cast<const float4*>(blk + o * 8));
                    const float4 c1 = __ldg(reinterpret_cast<const float4*>(blk + o * 8 + 4));
                    const float cf[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    float yA = 0.f, yB = 0.f;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        yA = fmaf(cf[l], z[l][s], yA);
                        yB = fmaf(cf[l], z[l][s + 2], yB);
                    }
                    // coordinate (i0 = q + 4s, i1 = o, beta): pencil a_local = i0 + 8 (o & 3) of CTA o >> 2
                    const int a_local = (q + 4 * s) + 8 * (o & 3);
                    if ((o >> 2) == r) {
                        E[e_index(r, g, a_local, beta)] = yA;
                        E[e_index(r, g + 8, a_local, beta)] = yB;
                    } else {
                        S[s_index(g, a_local, beta)] = yA;
                        S[s_index(g + 8, a_local, beta)] = yB;
                    }
                }
            }
        }

        // --------------------------------------------------- exchange ---
        fence_proxy_async_smem();     // S written through the generic proxy, read by the bulk copy
        __syncthreads();
        cluster_wait();               // the partner has finished reading its E
        if (tid == 0) bulk_copy_to_cluster(remote_e, S, kHalfBytes, remote_bar);
        if (!mbar_wait(bar, parity) && lane == 0) atomicExch(p.status, 1);
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
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int half = m >> 2;
                const int b0 = q + 8 * m, b1 = q + 4 + 8 * m;
                const float v[4] = {E[e_index(half, g, a_local, b0)], E[e_index(half, g + 8, a_local, b0)],
                                    E[e_index(half, g, a_local, b1)], E[e_index(half, g + 8, a_local, b1)]};
                uint32_t ah[4], al[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) split_tf32(v[e], ah[e], al[e]);
                const float2 bb = __ldg(p.pk2 + (size_t)(a + 64 * m) * 32 + lane);
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
                const float* blk = p.blk3 + (size_t)(a + 64 * i2) * 64;
                float yA[8], yB[8];
#pragma unroll
                for (int o = 0; o < 8; ++o) {
                    const float4 c0 = __ldg(reinterpret_cast<const float4*>(blk + o * 8));
                    const float4 c1 = __ldg(reinterpret_cast<const float4*>(blk + o * 8 + 4));
                    const float cf[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    float sa = 0.f, sb = 0.f;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        sa = fmaf(cf[l], z2[l][s], sa);
                        sb = fmaf(cf[l], z2[l][s + 2], sb);
                    }
                    yA[o] = sa;
                    yB[o] = sb;
                }
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
        // thread -> (row, beta' pair); 32 loads of two bf16 (beta' = 2p, 2p+1) across the 32
        // pencils of this CTA, repacked into two 64-byte runs of the output row.
        {
            const int row = tid >> 5, pidx = tid & 31;
            const int64_t grow = row0 + row;
            if (grow < p.rows) {
                const int i2 = pidx >> 2, i3 = 2 * (pidx & 3);
                uint32_t wv[32];
#pragma unroll
                for (int al = 0; al < 32; ++al)
                    wv[al] = *reinterpret_cast<const uint32_t*>(O + o_byte(row, al, i2, i3));
                uint32_t run0[16], run1[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    run0[k] = __byte_perm(wv[2 * k], wv[2 * k + 1], 0x5410);
                    run1[k] = __byte_perm(wv[2 * k], wv[2 * k + 1], 0x7632);
                }
                __nv_bfloat16* yrow = p.y + grow * p.ldy + 32 * r;
                uint4* d0 = reinterpret_cast<uint4*>(yrow + 64 * (i2 + 8 * i3));
                uint4* d1 = reinterpret_cast<uint4*>(yrow + 64 * (i2 + 8 * (i3 + 1)));
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    d0[k] = make_uint4(run0[4 * k], run0[4 * k + 1], run0[4 * k + 2], run0[4 * k + 3]);
                    d1[k] = make_uint4(run1[4 * k], run1[4 * k + 1], run1[4 * k + 2], run1[4 * k + 3]);
                }
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

struct FastState {
    float2* pk0 = nullptr;
    float2* pk2 = nullptr;
    int max_pairs = 0;
    bool ready = false;
};

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
    const int nblocks = kD / 8;
    if (cudaMalloc((void**)&fs->pk0, sizeof(float2) * nblocks * 32) != cudaSuccess ||
        cudaMalloc((void**)&fs->pk2, sizeof(float2) * nblocks * 32) != cudaSuccess) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the fragment tables failed");
    }
    const int threads = 256, grid = (nblocks * 32 + threads - 1) / threads;
    pack_fragments_kernel<<<grid, threads, 0, stream>>>(p->d_blocks + p->desc.st[0].block_off, fs->pk0, nblocks, 1);
    pack_fragments_kernel<<<grid, threads, 0, stream>>>(p->d_blocks + p->desc.st[2].block_off, fs->pk2, nblocks, 0);
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
    // 4-byte aligned input words, 16-byte aligned output runs
    if (((uintptr_t)x & 3) || (ld_x & 1) || ((uintptr_t)y & 15) || (ld_y & 7)) return HARP_ERR_UNSUPPORTED;
    if (rows < 32) return HARP_ERR_UNSUPPORTED;
    cudaStream_t stream = (cudaStream_t)stream_;
    harp_status st = prepare(p, stream);
    if (st != HARP_OK) return st;
    FastState* fs = static_cast<FastState*>(p->fast);
    const int64_t ntiles = (rows + kTile - 1) / kTile;
    if (ntiles > 0x7fffffff) return HARP_ERR_UNSUPPORTED;
    const int pairs = (int)std::min<int64_t>(fs->max_pairs, ntiles);
    FastParams fp;
    fp.x = reinterpret_cast<const uint32_t*>(x);
    fp.y = reinterpret_cast<__nv_bfloat16*>(y);
    fp.rows = rows;
    fp.ldx_w = ld_x / 2;
    fp.ldy = ld_y;
    fp.ntiles = (int)ntiles;
    fp.pk0 = fs->pk0;
    fp.blk1 = p->d_blocks + p->desc.st[1].block_off;
    fp.pk2 = fs->pk2;
    fp.blk3 = p->d_blocks + p->desc.st[3].block_off;
    fp.status = p->d_status;
    harp_fast_d4096_fwd_kernel<<<2 * pairs, kThreads, kSmemBytes, stream>>>(fp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_fast_d4096_fwd_kernel");
    return HARP_OK;
}

void fast_state_free(harp_plan_s* p) {
    FastState* fs = static_cast<FastState*>(p->fast);
    if (!fs) return;
    cudaFree(fs->pk0);
    cudaFree(fs->pk2);
    delete fs;
    p->fast = nullptr;
}
