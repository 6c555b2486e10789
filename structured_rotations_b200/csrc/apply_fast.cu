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
// Inner engine: every stage runs on tensor cores, mma.sync m16n8k8 TF32 with the 16
// tile rows as M, the 8 inputs of a group as K and its 8 outputs as N.  fp32 accuracy
// comes from splitting operands into TF32 hi + lo parts and summing hi*hi + hi*lo +
// lo*hi (bf16 input is exact in TF32, so stage 0 needs only hi*hi + hi*lo).
//
// Coefficients are stationary in tensor memory: each warp always works on the same
// two chunks and two pencils, whose 64 blocks in mma B-fragment form are exactly
// 128 words per lane, i.e. the warp's quarter of its TMEM lane quadrant.  They are
// written once per launch and read with tcgen05.ld, so the coefficients cost no L2
// traffic inside the row loop.
//
// Between the two stages of a phase the mma output (lane q holds two outputs of every
// group) is turned into the next stage's operand (lane q holds two inputs of every
// group) by a 4-lane butterfly: three shfl.xor rounds plus an XOR permutation by the
// lane's quad index (two levels of selects).  The K slots of the second stage
// therefore mean different inputs in different lanes; the packed B fragments
// follow the same lane-dependent order.
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
constexpr size_t kSmemBytes = (size_t)kBarOffset + 8 * (kWarps + 2) + 16 + 1024;   // + TMEM slot, alignment slack
constexpr int kTmemCols = 512;               // the SM's whole tensor memory: 128 columns per warp
constexpr long long kWaitLimit = 1ll << 26;  // mbarrier polls before giving up

struct FastParams {
    __nv_bfloat16* y;
    int64_t rows, ldy;       // ldy in elements
    int ntiles;
    const float4* frag;      // B fragments, [cta rank][warp][column / 4][lane] float4 (see pack kernel)
    int* status;
    int8_t* q;               // quantizing variant: int8 codes, rows of 4096, leading dimension ldq
    int64_t ldq;
    float* scales;           // and one scale per block of QB coordinates, leading dimension lds
    int64_t lds;
};

// ----------------------------------------------------------------- PTX ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Two values split into x = hi + lo for the three-product TF32 scheme.  hi is x truncated to
// 11 significant bits (bits 0-12 of the pattern cleared, one logic instruction), so hi is
// exact in TF32 and |lo| < 2^-10 |x|; lo = x - hi is exact in fp32 (at most 13 significant
// bits), and the tensor core reads its top 11, so |x - hi - lo_tf32| < 2^-21 |x|.  The
// dropped product lo_a lo_b is below 2^-20 |a b|.  Only the subtraction uses the FMA pipe.
__device__ __forceinline__ void split2_tf32(float a, float b, uint32_t& ha, uint32_t& hb, uint32_t& la,
                                            uint32_t& lb) {
    ha = __float_as_uint(a) & 0xffffe000u;
    hb = __float_as_uint(b) & 0xffffe000u;
    la = __float_as_uint(__fsub_rn(a, __uint_as_float(ha)));
    lb = __float_as_uint(__fsub_rn(b, __uint_as_float(hb)));
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

// 2-D tiled TMA load of one box into this CTA's own shared memory.
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
// and pos = a_local ^ swz(row, beta), swz = (row & 7) | (c(beta) << 3) with c = beta & 3 in
// the bf16 variant and c = (beta ^ (beta >> 4)) & 3 in the quantizing one.
//  - phase A stores one scalar per lane with beta fixed, row = g (+8) and a_local = l + 8q:
//    (l + 8q) ^ (g + 8c) has l ^ g in bits 0-2 and q ^ c in bits 3-4, 32 banks.
//  - phase B loads one scalar per lane with a_local fixed, row = g (+8) and
//    beta = q + 8m (+4), so beta & 3 = q and (beta >> 4) & 3 = m >> 1 for the whole
//    instruction: a_local ^ (g + 8 (q ^ const)), 32 banks.
//  - the quantizing variant also stores its outputs back in place (a_local fixed, row = g (+8),
//    beta = l + 16q + 8e for fixed l, e: beta & 3 = l & 3, (beta >> 4) & 3 = q), which the
//    (beta >> 4) term spreads: a_local ^ (g + 8 ((l & 3) ^ q)), 32 banks; its epilogue reads a
//    row with lane = a_local and beta fixed, a permutation of one 32-float run.
// Each chunk's 16 x 32 block is contiguous (2 KB), so the part of it bound for the partner
// CTA is sent with one bulk copy as soon as the warp has produced it.
template <int QB>
__device__ __forceinline__ int swz_of(int row, int beta) {
    if constexpr (QB == 0) return (row & 7) | ((beta & 3) << 3);
    else return (row & 7) | (((beta ^ (beta >> 4)) & 3) << 3);
}

template <int QB>
__device__ __forceinline__ int e_index(int half, int row, int a_local, int beta) {
    return ((half * 32 + (beta & 31)) * 16 + row) * 32 + (a_local ^ swz_of<QB>(row, beta));
}

template <int QB>
__device__ __forceinline__ int s_index(int row, int a_local, int beta) {
    return ((beta & 31) * 16 + row) * 32 + (a_local ^ swz_of<QB>(row, beta));
}

// Output staging O[row][a_local][beta] (bf16), stored in 16-byte chunks of 8 beta values
// (chunk = i3 = beta >> 3, inside the chunk i2 = beta & 7) at chunk position
// i3 ^ h, h = (row & 1) ^ (2 ((a_local >> 3) & 3)).
//  - phase B stores one chunk per lane (a_local fixed, i3 = 2q + e, rows 2k and 2k+1 in a
//    quarter-warp): the row bit moves the chunk to the other parity, 8 distinct chunks.
//  - the store phase loads one word (two beta) per thread with the row fixed, 8
//    consecutive beta pairs and the 4 pencil quarters u: chunks (pp >> 2) ^ 2u ^ c are 8
//    distinct values and pp & 3 selects the word, 32 banks.
__device__ __forceinline__ int o_byte(int row, int a_local, int beta) {
    const int chunk = (beta >> 3) ^ ((row & 1) ^ (((a_local >> 3) & 3) << 1));
    return ((row * 32 + a_local) * 64 + chunk * 8 + (beta & 7)) * 2;
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

// ------------------------------------------------------- tensor memory ---

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------- stage helpers ---

// One stage of 8 groups on tensor cores from fp32 operands: d[l] = A[l] * B_l with the
// A fragments split into hi + lo and the B fragments (two fp32 words per group, from
// TMEM) split likewise; three products per group.
__device__ __forceinline__ void mma_stage_f32(const float (&a)[8][4], const uint32_t (&bw)[16],
                                              float (&d)[8][4]) {
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        uint32_t ah[4], al[4];
        split2_tf32(a[l][0], a[l][1], ah[0], ah[1], al[0], al[1]);
        split2_tf32(a[l][2], a[l][3], ah[2], ah[3], al[2], al[3]);
        uint32_t bh0, bl0, bh1, bl1;
        split2_tf32(__uint_as_float(bw[2 * l]), __uint_as_float(bw[2 * l + 1]), bh0, bh1, bl0, bl1);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tf32(acc, ah, bh0, bh1);
        mma_tf32(acc, ah, bl0, bl1);
        mma_tf32(acc, al, bh0, bh1);
#pragma unroll
        for (int e = 0; e < 4; ++e) d[l][e] = acc[e];
    }
}

__device__ __forceinline__ void cswap(bool p, float& x, float& y) {
    const float a = p ? y : x;
    const float b = p ? x : y;
    x = a;
    y = b;
}

// 4-lane butterfly between the two stages of a phase.
// In:  z[j][e], the mma output of group j (e = s + 2h: output slot s of row half h), where
//      output slot s of lane q is next-stage group c + 4s with c = q.
// Out: a[l][e'], the A fragment of next-stage group l = c + 4s (e' = h + 2t), whose K slot t
//      holds input j = (q ^ c) + 4t: round delta brings j = delta + 4t from lane q ^ delta.
__device__ __forceinline__ void quad_butterfly(const float (&z)[8][4], int q, float (&a)[8][4]) {
    float rr[4][2][2][2];   // [delta][t][s][h]
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                rr[0][t][s][h] = z[4 * t][s + 2 * h];
#pragma unroll
                for (int dl = 1; dl < 4; ++dl)
                    rr[dl][t][s][h] = __shfl_xor_sync(0xffffffffu, z[dl + 4 * t][s + 2 * h], dl);
            }
    // rr[delta] came from lane q ^ delta; reorder so that rr[c] comes from lane c
    const bool b0 = (q & 1) != 0, b1 = (q & 2) != 0;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                cswap(b0, rr[0][t][s][h], rr[1][t][s][h]);
                cswap(b0, rr[2][t][s][h], rr[3][t][s][h]);
                cswap(b1, rr[0][t][s][h], rr[2][t][s][h]);
                cswap(b1, rr[1][t][s][h], rr[3][t][s][h]);
            }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            a[c + 4 * s][0] = rr[c][0][s][0];
            a[c + 4 * s][1] = rr[c][0][s][1];
            a[c + 4 * s][2] = rr[c][1][s][0];
            a[c + 4 * s][3] = rr[c][1][s][1];
        }
}

// Output row `row` of one tile, stored by one warp: item (pp, u) = beta pair (2pp, 2pp+1)
// and pencil quarter u = a_local >> 3, four items per lane.  Eight word loads give the 8
// pencils of the quarter for both beta; each becomes a 16-byte piece of a 64-byte output
// run, so each 16-byte store instruction writes 8 whole runs.  Row w of O occupies exactly
// the bytes of S that warp w writes next (its two chunks' 2 KB blocks), so no other warp
// has to wait for these loads.
__device__ __forceinline__ void store_row(const unsigned char* O, const FastParams& p, int64_t row0, int row,
                                          int r, int lane) {
    const int64_t grow = row0 + row;
    if (grow >= p.rows) return;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int item = lane + 32 * it;
        const int pp = item >> 2, u = item & 3;
        uint32_t wv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            wv[k] = *reinterpret_cast<const uint32_t*>(O + o_byte(row, 8 * u + k, 2 * pp));
        const uint4 r0 = make_uint4(__byte_perm(wv[0], wv[1], 0x5410), __byte_perm(wv[2], wv[3], 0x5410),
                                    __byte_perm(wv[4], wv[5], 0x5410), __byte_perm(wv[6], wv[7], 0x5410));
        const uint4 r1 = make_uint4(__byte_perm(wv[0], wv[1], 0x7632), __byte_perm(wv[2], wv[3], 0x7632),
                                    __byte_perm(wv[4], wv[5], 0x7632), __byte_perm(wv[6], wv[7], 0x7632));
        __nv_bfloat16* yrow = p.y + grow * p.ldy + 32 * r + 8 * u;
        *reinterpret_cast<uint4*>(yrow + 64 * (2 * pp)) = r0;
        *reinterpret_cast<uint4*>(yrow + 64 * (2 * pp + 1)) = r1;
    }
}

// ------------------------------------------------- quantizing epilogue ---
//
// The quantizing variant (QB = 32, 64, 128 or 256, the blockwise int8 quantizer of the fused
// rotate-then-quantize call) leaves each fp32 output in E where phase B read its input (see
// e_index), then warp w quantizes row w of the tile:
//  - lane L holds pencil a_local = L of the row for all 64 beta (64 conflict-free loads); a
//    block of QB coordinates is, in this CTA's view, the pencils of beta >> SH (QB >= 64: the
//    other 32 pencils are the partner's) or of one beta (QB = 32: the block is this CTA's);
//  - block maxima: |y| maximised over the lane's beta of the block, then over the warp
//    (redux.sync on the fp32 bit patterns, which order like the values for |y| >= 0);
//  - QB >= 64: lane kb sends block kb's maximum to the partner's AMX[w][kb] (st.async,
//    completed on the partner's qbar) and takes the larger of its own and the partner's;
//  - s = a / 127 and 127 / a (fp32, round to nearest; 0 for a = 0) for the lane's blocks,
//    the reciprocals passed round by shuffles; codes clamp(rne(y * (127 / a)), -127, 127)
//    go byte by byte into the 32-byte runs CS[w][beta] and leave as 16-byte stores (the run
//    of beta holds coordinates 64 beta + 32 r .. + 31).
// S holds AMX (4 KB) and CS (32 KB) here: S is free from phase B (the partner has
// received this CTA's chunks) until the next tile's phase A, which starts only after every
// thread of both CTAs has passed this epilogue (the tile-end cluster barrier).
constexpr int kAmxOffset = 0, kCsOffset = 4096;

// round to nearest even, saturated to [-128, 127]
__device__ __forceinline__ uint32_t cvt_rni_sat_s8(float x) {
    uint32_t r;
    asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void st_async_b32(uint32_t addr, uint32_t v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
                 "r"(remote_bar)
                 : "memory");
}

template <int QB>
__device__ __forceinline__ void quant_row(const float* E, unsigned char* S, const FastParams& p, int64_t row0, int r,
                                          int w, int lane, uint64_t* qbar, uint32_t qparity, uint32_t remote_s,
                                          uint32_t remote_qbar) {
    constexpr int SH = QB <= 64 ? 0 : (QB == 128 ? 1 : 2);   // block of beta >> SH
    constexpr int NLOC = 64 >> SH;                           // blocks of the row in this CTA's view
    constexpr bool XCH = QB >= 64;                           // blocks span both CTAs
    float v[64];
#pragma unroll
    for (int beta = 0; beta < 64; ++beta) v[beta] = E[e_index<QB>(beta >> 5, w, lane, beta)];
    float own0 = 0.f, own1 = 0.f;   // lane L: the maxima of blocks L and L + 32
#pragma unroll
    for (int kb = 0; kb < NLOC; ++kb) {
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < (1 << SH); ++t) m = fmaxf(m, fabsf(v[(kb << SH) + t]));
        const float wm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
        if (kb < 32) own0 = lane == kb ? wm : own0;
        else own1 = lane == kb - 32 ? wm : own1;
    }
    float a0 = own0, a1 = own1;
    if constexpr (XCH) {
        const uint32_t dst = remote_s + kAmxOffset + (uint32_t)(w * 64 + lane) * 4u;
        if (lane < NLOC) st_async_b32(dst, __float_as_uint(own0), remote_qbar);
        if (NLOC > 32) st_async_b32(dst + 128u, __float_as_uint(own1), remote_qbar);
        if (!mbar_wait(qbar, qparity)) {
            if (lane == 0) atomicExch(p.status, 1);
            mbar_wait(qbar, qparity);   // bounded again: no store may land after exit
        }
        const float* amx = reinterpret_cast<const float*>(S + kAmxOffset) + w * 64;
        if (lane < NLOC) a0 = fmaxf(own0, amx[lane]);
        if (NLOC > 32) a1 = fmaxf(own1, amx[lane + 32]);
    }
    float inv0 = 0.f, inv1 = 0.f;   // lane L: 127 / a of blocks L and L + 32
    const int64_t grow = row0 + w;
#pragma unroll
    for (int h = 0; h < (NLOC > 32 ? 2 : 1); ++h) {
        const int kb = lane + 32 * h;
        if (kb < NLOC) {
            const float a = h ? a1 : a0;
            const float iv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
            if (h) inv1 = iv;
            else inv0 = iv;
            if (grow < p.rows) {
                if constexpr (XCH) {
                    if (r == 0) p.scales[grow * p.lds + kb] = __fdiv_rn(a, 127.f);
                } else {
                    p.scales[grow * p.lds + 2 * kb + r] = __fdiv_rn(a, 127.f);   // block (beta = kb, CTA r)
                }
            }
        }
    }
    // Codes: |y| <= a gives |y * fl(127 / a)| <= 127 (1 + 2^-23), so the round-to-nearest
    // conversion lands in [-127, 127]; the saturating conversion to s8 keeps that bound
    // without a separate clamp.
    unsigned char* cs = S + kCsOffset + w * 2048;
#pragma unroll
    for (int kb = 0; kb < NLOC; ++kb) {
        const float iv = __shfl_sync(0xffffffffu, kb < 32 ? inv0 : inv1, kb & 31);
#pragma unroll
        for (int t = 0; t < (1 << SH); ++t) {
            const int beta = (kb << SH) + t;
            cs[beta * 32 + lane] = (unsigned char)(cvt_rni_sat_s8(v[beta] * iv) & 0xffu);
        }
    }
    __syncwarp();
    if (grow < p.rows) {
        // runs beta = 2 lane and 2 lane + 1: 64 contiguous staging bytes, two 32-byte runs out
        const uint4* src = reinterpret_cast<const uint4*>(cs + 64 * lane);
        int8_t* dst = p.q + grow * p.ldq + 32 * r + 128 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(dst + 64 * (k >> 1) + 16 * (k & 1)) = src[k];
    }
}

// ------------------------------------------------------------- kernel ---

// QB = 0: bf16 rows out.  QB = 32 .. 256: int8 codes and per-block scales out (quant_row).
template <int QB>
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
    uint64_t* qbar = bar + 1;                                           // partner's block maxima
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int r = (int)cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    unsigned char* Xw = X + warp * kXBytes;

    // tensor memory: the whole 512 columns; warp w uses lanes 32 (w & 3).., columns 128 (w >> 2)..
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(qbar, 1);
    }
    if (lane == 0) mbar_init(xbar + warp, 1);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t taddr = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + 128u * (uint32_t)(warp >> 2);
    {
        // this warp's 128 fragment columns: [slot (2 chunks, 2 pencils)][stage][group][word]
        const float4* src = p.frag + ((size_t)(r * kWarps + warp) * 32) * 32 + lane;
#pragma unroll 1
        for (int c16 = 0; c16 < 8; ++c16) {
            uint32_t v[16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 f = __ldg(src + (c16 * 4 + k) * 32);
                v[4 * k] = __float_as_uint(f.x);
                v[4 * k + 1] = __float_as_uint(f.y);
                v[4 * k + 2] = __float_as_uint(f.z);
                v[4 * k + 3] = __float_as_uint(f.w);
            }
            tmem_st16(taddr + 16u * c16, v);
        }
        tmem_wait_st();
    }

    const uint32_t remote_e = map_to_rank(smem_u32(E + r * kSFloats), (uint32_t)(r ^ 1));   // partner's half r
    const uint32_t remote_bar = map_to_rank(smem_u32(bar), (uint32_t)(r ^ 1));
    const uint32_t remote_s = map_to_rank(smem_u32(S), (uint32_t)(r ^ 1));
    const uint32_t remote_qbar = map_to_rank(smem_u32(qbar), (uint32_t)(r ^ 1));
    cluster_arrive();
    cluster_wait();     // barriers initialised on both CTAs
    cluster_arrive();   // "my E may be written": matched by the wait at the top of the first tile

    // first input box of this warp: tile `pair`, task 0
    if (lane == 0 && pair < p.ntiles) {
        mbar_arrive_expect_tx(xbar + warp, kXBytes);
        tma_load_2d(Xw, &tmap_x, 64 * (32 * r + 2 * warp), pair * kTile, xbar + warp);
    }
    uint32_t xparity = 0, parity = 0, qparity = 0;
    int64_t prev_row0 = -1;           // tile whose output still sits in O

    for (int tile = pair; tile < p.ntiles; tile += npairs) {
        const int64_t row0 = (int64_t)tile * kTile;
        if (tid == 0) {
            mbar_arrive_expect_tx(bar, kHalfBytes);
            // the partner's block maxima of this tile (16 rows of 4096 / QB blocks)
            if constexpr (QB >= 64) mbar_arrive_expect_tx(qbar, 16u * (4096u / QB) * 4u);
        }

        // -------------------------------------------------- phase A ---
#pragma unroll 1
        for (int task = 0; task < 2; ++task) {
            const int beta = 32 * r + 2 * warp + task;
            uint32_t bw[16];
            tmem_ld16(taddr + 32u * task, bw);          // stage-0 fragments of this chunk
            if (!mbar_wait(xbar + warp, xparity) && lane == 0) atomicExch(p.status, 1);
            xparity ^= 1;
            uint32_t w0[8], w1[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // elements 8j + 2q, 8j + 2q + 1 of rows g, g + 8
                w0[j] = *reinterpret_cast<const uint32_t*>(Xw + x_byte(g, j, q));
                w1[j] = *reinterpret_cast<const uint32_t*>(Xw + x_byte(g + 8, j, q));
            }
            tmem_wait_ld();
            // stage 0: group j = i1, slot q <-> i0 = 2q, slot q+4 <-> i0 = 2q+1;
            // output slot 2q <-> i0 = q, 2q+1 <-> i0 = q + 4.
            float z[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t a[4] = {w0[j] << 16, w1[j] << 16, w0[j] & 0xffff0000u, w1[j] & 0xffff0000u};
                uint32_t bh0, bl0, bh1, bl1;
                split2_tf32(__uint_as_float(bw[2 * j]), __uint_as_float(bw[2 * j + 1]), bh0, bh1, bl0, bl1);
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
            tmem_ld16(taddr + 32u * task + 16u, bw);    // stage-1 fragments
            float a1[8][4];
            quad_butterfly(z, q, a1);
            tmem_wait_ld();
            // stage 1: group l = i0; output slot 2q <-> i1 = q (pencils of CTA 0),
            // 2q+1 <-> i1 = q + 4 (pencils of CTA 1); both are pencil a_local = l + 8q there.
            float y1[8][4];
            mma_stage_f32(a1, bw, y1);
            if (task == 0) {
                // row `warp` of the previous tile's output leaves O, which aliases the part
                // of S this warp is about to write
                if (QB == 0 && prev_row0 >= 0) store_row(O, p, prev_row0, warp, r, lane);
                __syncwarp();
                cluster_wait();       // the partner has finished reading its E (previous tile)
            }
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                const int a_local = l + 8 * q;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {   // hh = destination CTA
                    const float va = y1[l][hh], vb = y1[l][hh + 2];
                    if (hh == r) {
                        E[e_index<QB>(r, g, a_local, beta)] = va;
                        E[e_index<QB>(r, g + 8, a_local, beta)] = vb;
                    } else {
                        S[s_index<QB>(g, a_local, beta)] = va;
                        S[s_index<QB>(g + 8, a_local, beta)] = vb;
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
        cluster_arrive();             // the partner's copies have landed: its S may be reused

        // --------------------------------------------------- phase B ---
#pragma unroll 1
        for (int task = 0; task < 2; ++task) {
            const int a_local = 2 * warp + task;
            uint32_t bw[16];
            tmem_ld16(taddr + 32u * (2 + task), bw);    // stage-2 fragments of this pencil
            // stage 2: group m = i3, slot q <-> i2 = q, slot q+4 <-> i2 = q + 4;
            // output slot 2q <-> i2 = q, 2q+1 <-> i2 = q + 4.
            float v2[8][4];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int half = m >> 2;
                const int b0 = q + 8 * m, b1 = q + 4 + 8 * m;
                v2[m][0] = E[e_index<QB>(half, g, a_local, b0)];
                v2[m][1] = E[e_index<QB>(half, g + 8, a_local, b0)];
                v2[m][2] = E[e_index<QB>(half, g, a_local, b1)];
                v2[m][3] = E[e_index<QB>(half, g + 8, a_local, b1)];
            }
            tmem_wait_ld();
            float zz2[8][4];
            mma_stage_f32(v2, bw, zz2);
            tmem_ld16(taddr + 32u * (2 + task) + 16u, bw);   // stage-3 fragments
            float a3[8][4];
            quad_butterfly(zz2, q, a3);
            tmem_wait_ld();
            // stage 3: group l = i2; output slot 2q <-> i3 = 2q, 2q+1 <-> i3 = 2q + 1
            float y3[8][4];
            mma_stage_f32(a3, bw, y3);
            if (task == 0) cluster_wait();   // my copies have landed too: O (= S) may be written
            if constexpr (QB == 0) {
                // bf16 runs of 8 consecutive beta (i2 = 0..7) for i3 = 2q + e, rows g and g + 8
#pragma unroll
                for (int e = 0; e < 2; ++e) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int c = e + 2 * hh;
                        const uint4 pk =
                            make_uint4(pack_bf16x2(y3[0][c], y3[1][c]), pack_bf16x2(y3[2][c], y3[3][c]),
                                       pack_bf16x2(y3[4][c], y3[5][c]), pack_bf16x2(y3[6][c], y3[7][c]));
                        *reinterpret_cast<uint4*>(O + o_byte(g + 8 * hh, a_local, 8 * (2 * q + e))) = pk;
                    }
                }
            } else {
                // fp32 outputs back into E where this pencil's inputs were (beta = i2 + 8 i3)
#pragma unroll
                for (int l = 0; l < 8; ++l)
#pragma unroll
                    for (int e = 0; e < 2; ++e)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int beta = l + 8 * (2 * q + e);
                            E[e_index<QB>(beta >> 5, g + 8 * hh, a_local, beta)] = y3[l][e + 2 * hh];
                        }
            }
        }
        __syncthreads();
        if constexpr (QB > 0) {
            quant_row<QB>(E, reinterpret_cast<unsigned char*>(S), p, row0, r, warp, lane, qbar, qparity, remote_s,
                          remote_qbar);
            if constexpr (QB >= 64) qparity ^= 1;
        }
        cluster_arrive();             // my E has been read: the partner may send the next tile

        prev_row0 = row0;             // its output is stored during the next tile's first task
    }
    if (QB == 0 && prev_row0 >= 0) store_row(O, p, prev_row0, warp, r, lane);
    cluster_wait();                   // matches the last arrive; no bulk copy is in flight
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(*tmem_slot, kTmemCols);
}

// B fragments for mma.m16n8k8, packed per (CTA rank r, warp w, lane L = 4g + q) into
// 128 columns: column = slot * 32 + stage * 16 + group * 2 + word, where slots 0, 1 are
// the chunks beta = 32r + 2w + slot (stages 0, 1) and slots 2, 3 the pencils
// a = 32r + 2w + slot - 2 (stages 2, 3).  Word k of group n is B[k-th K slot][g] =
// Blk[out(g)][in]:
//   out(g) = g / 2 (even g), g / 2 + 4 (odd g) for stages 0-2; out(g) = g for stage 3;
//   stage 0, block j + 8 beta:   in = 2q + k
//   stage 1, block l + 8 beta:   in = (q ^ (l & 3)) + 4k
//   stage 2, block a + 64 m:     in = q + 4k
//   stage 3, block a + 64 l:     in = (q ^ (l & 3)) + 4k
// Stored as float4 over 4 consecutive columns: frag[((r * 16 + w) * 32 + col / 4) * 32 + L].
__global__ void pack_fragments_kernel(const float* __restrict__ b0, const float* __restrict__ b1,
                                      const float* __restrict__ b2, const float* __restrict__ b3,
                                      float* __restrict__ frag) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;   // one float per thread
    if (gid >= 2 * kWarps * 128 * 32) return;
    const int comp = gid & 3;
    const int L = (gid >> 2) & 31;
    const int col4 = (gid >> 7) & 31;
    const int w = (gid >> 12) & 15;
    const int r = gid >> 16;
    const int col = col4 * 4 + comp;
    const int slot = col >> 5, stage = (col >> 4) & 1, grp = (col >> 1) & 7, k = col & 1;
    const int g = L >> 2, q = L & 3;
    const int pn = (g & 1) ? (g >> 1) + 4 : (g >> 1);
    float v;
    if (slot < 2) {
        const int beta = 32 * r + 2 * w + slot;
        if (stage == 0) v = b0[(size_t)(grp + 8 * beta) * 64 + pn * 8 + 2 * q + k];
        else            v = b1[(size_t)(grp + 8 * beta) * 64 + pn * 8 + ((q ^ (grp & 3)) + 4 * k)];
    } else {
        const int a = 32 * r + 2 * w + slot - 2;
        if (stage == 0) v = b2[(size_t)(a + 64 * grp) * 64 + pn * 8 + q + 4 * k];
        else            v = b3[(size_t)(a + 64 * grp) * 64 + g * 8 + ((q ^ (grp & 3)) + 4 * k)];
    }
    frag[gid] = v;
}

struct FastState {
    float* frag = nullptr;
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

// The variants: bf16 rows out, then int8 codes for quantizer blocks of 32, 64, 128, 256.
const void* const kKernels[] = {(const void*)harp_fast_d4096_fwd_kernel<0>, (const void*)harp_fast_d4096_fwd_kernel<32>,
                                (const void*)harp_fast_d4096_fwd_kernel<64>, (const void*)harp_fast_d4096_fwd_kernel<128>,
                                (const void*)harp_fast_d4096_fwd_kernel<256>};

// The coefficient table and the launch attributes of the specialized kernel, built once per
// plan by materialization (on the materializing stream): afterwards launches only read
// them, so calls on any number of streams may run at once.
harp_status prepare(harp_plan_s* p, cudaStream_t stream) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        cudaGetLastError();
    });
    if (!g_encode) return harp_fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cudaError_t e = cudaSuccess;
    for (const void* k : kKernels) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    int nclusters = 0;
    for (const void* k : kKernels) {   // the variants' limits (equal in practice: one CTA per SM)
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, k, &cfg);
        if (e != cudaSuccess) break;
        nclusters = k == kKernels[0] ? n : std::min(nclusters, n);
    }
    if (e != cudaSuccess || nclusters < 1) {
        cudaGetLastError();
        return harp_fail(HARP_ERR_CUDA, "no cluster of two fits on this device");
    }
    FastState* fs = new FastState();
    const int nfloat = 2 * kWarps * 128 * 32;
    if (cudaMalloc((void**)&fs->frag, sizeof(float) * nfloat) != cudaSuccess) {
        cudaGetLastError();
        delete fs;
        return harp_fail(HARP_ERR_ALLOC, "cudaMalloc of the fragment table failed");
    }
    const float* blocks = p->d_blocks;
    pack_fragments_kernel<<<(nfloat + 255) / 256, 256, 0, stream>>>(
        blocks + p->desc.st[0].block_off, blocks + p->desc.st[1].block_off, blocks + p->desc.st[2].block_off,
        blocks + p->desc.st[3].block_off, fs->frag);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        cudaFree(fs->frag);
        delete fs;
        return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    fs->max_pairs = nclusters;
    fs->ready = true;
    p->fast = fs;
    return HARP_OK;
}

}  // namespace

namespace {

// Encodes the input map and launches variant QB (0: bf16 rows to fp.y; else the quantizer).
harp_status launch_variant(harp_plan_s* p, const void* x, int64_t rows, int64_t ld_x, FastParams fp, int qb,
                           cudaStream_t stream) {
    const FastState* fs = static_cast<const FastState*>(p->fast);
    if (!fs || !fs->ready) return HARP_ERR_UNSUPPORTED;   // no table: the plan was not eligible or it failed
    const int64_t ntiles = (rows + kTile - 1) / kTile;
    const int pairs = (int)std::min<int64_t>(fs->max_pairs, ntiles);

    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld_x * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    const cuuint32_t estride[2] = {1, 1};
    auto encode = [&] {
        return g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    };
    CUresult cr = encode();
    if (cr == CUDA_ERROR_INVALID_CONTEXT) {
        // a host thread whose first CUDA call this is has no current context yet: bind the
        // plan's device (the runtime's primary context) and encode again
        if (cudaSetDevice(p->device) != cudaSuccess) cudaGetLastError();
        cr = encode();
    }
    if (cr != CUDA_SUCCESS) return harp_fail(HARP_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)cr));

    fp.rows = rows;
    fp.ntiles = (int)ntiles;
    fp.frag = reinterpret_cast<const float4*>(fs->frag);
    fp.status = p->d_status;
    switch (qb) {
        case 0: harp_fast_d4096_fwd_kernel<0><<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp); break;
        case 32: harp_fast_d4096_fwd_kernel<32><<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp); break;
        case 64: harp_fast_d4096_fwd_kernel<64><<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp); break;
        case 128: harp_fast_d4096_fwd_kernel<128><<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp); break;
        case 256: harp_fast_d4096_fwd_kernel<256><<<2 * pairs, kThreads, kSmemBytes, stream>>>(tmap, fp); break;
        default: return HARP_ERR_UNSUPPORTED;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_fast_d4096_fwd_kernel");
    return HARP_OK;
}

}  // namespace

harp_status launch_apply_fast(harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                              int64_t ld_y, harp_dtype in_dtype, harp_dir dir, void* stream,
                              harp_dtype out_dtype) {
    if (!is_d4096_radix8(p) || in_dtype != HARP_BF16 || out_dtype != HARP_BF16 || dir != HARP_FORWARD)
        return HARP_ERR_UNSUPPORTED;
    // TMA input boxes need 16-byte aligned rows; output runs are 16-byte stores
    if (((uintptr_t)x & 15) || (ld_x & 7) || ((uintptr_t)y & 15) || (ld_y & 7)) return HARP_ERR_UNSUPPORTED;
    if (rows < 32 || rows > 0x7fffffffll) return HARP_ERR_UNSUPPORTED;
    FastParams fp = {};
    fp.y = reinterpret_cast<__nv_bfloat16*>(y);
    fp.ldy = ld_y;
    return launch_variant(p, x, rows, ld_x, fp, 0, (cudaStream_t)stream);
}

harp_status launch_apply_fast_quant(harp_plan_s* p, const void* x, int64_t rows, int64_t ld_x, int8_t* q,
                                    int64_t ld_q, float* scales, int64_t ld_s, int qblock, harp_dir dir,
                                    void* stream) {
    if (!is_d4096_radix8(p) || dir != HARP_FORWARD) return HARP_ERR_UNSUPPORTED;
    if (qblock != 32 && qblock != 64 && qblock != 128 && qblock != 256) return HARP_ERR_UNSUPPORTED;
    // TMA input boxes: 16-byte aligned rows; codes leave as 16-byte stores; scales as floats
    if (((uintptr_t)x & 15) || (ld_x & 7) || ((uintptr_t)q & 15) || (ld_q & 15) || ((uintptr_t)scales & 3))
        return HARP_ERR_UNSUPPORTED;
    if (rows < 32 || rows > 0x7fffffffll) return HARP_ERR_UNSUPPORTED;
    FastParams fp = {};
    fp.q = q;
    fp.ldq = ld_q;
    fp.scales = scales;
    fp.lds = ld_s;
    return launch_variant(p, x, rows, ld_x, fp, qblock, (cudaStream_t)stream);
}

void fast_prepare(harp_plan_s* p, void* stream) {
    if (p->fast || !is_d4096_radix8(p)) return;
    if (prepare(p, (cudaStream_t)stream) != HARP_OK) harp_clear_error();   // the plan runs on the tiled kernel
}

void fast_state_free(harp_plan_s* p) {
    FastState* fs = static_cast<FastState*>(p->fast);
    if (!fs) return;
    cudaFree(fs->frag);
    delete fs;
    p->fast = nullptr;
}
