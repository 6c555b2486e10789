// Column passes of the two-sided rotation (HARP abstract: a rotation on each side of a
// weight matrix): every column of an fp32 matrix X with d rows takes T or T^T of one
// plan, with the result written in place or rounded to the output type.
//
// Stage t mixes the rows {lo + s_t (k + b_t hi)} of X with block B_{t,c}, the same
// b_t x b_t block for every column.  So a block serves all 64 columns of a tile (the 32
// lanes of a warp hold two columns each and load the block's coefficients with
// warp-uniform addresses, a broadcast), and the columns never need a transpose.  A CTA
// (one per SM) runs through a contiguous range of tiles, column tile after column tile of
// one row tile, so the row tile's blocks are staged in shared memory once for all its
// column tiles.  When two tiles' data fit in shared memory next to the blocks, the next
// tile's data arrive (cp.async into a second buffer) while this tile's stages run; the
// large shapes (a 448-row problem of 64 columns is 112 KB) load, compute and store in turn.
//
// The stages split at t* into two passes over X (P = s_{t*} = prod_{t<t*} b_t, Q = d / P):
//  - pass A, stages t >= t*: for fixed p in [0, P) the rows {p + P v : v < Q} form a
//    Q-coordinate problem in v, where stage t has stride s_t / P and the block of local
//    index c_v is c = p + P c_v.  A tile holds PB consecutive p values, PB*Q rows.
//  - pass B, stages t < t*: a slab of P contiguous rows; the block of local index c_l
//    in slab n is c = n (P / b_t) + c_l.
// The inverse runs pass A (stages m-1 .. t*) then pass B (t*-1 .. 0) with transposed
// blocks; the forward direction runs pass B (0 .. t*-1) then pass A (t* .. m-1).
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace {

constexpr int kCols = 64;          // columns per tile: two per lane
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemBudget = 200 * 1024;

struct ColsParams {
    PlanDesc pd;
    const float* blocks;   // row-major [stage][c][k][l]
    float* x;              // d rows, leading dimension ld_x (fp32)
    void* y;               // output rows (== x for in place), leading dimension ld_y
    int64_t ld_x, ld_y;
    int ncols;
    int pass_a;            // 1: row sets {p + P v}; 0: slabs of P rows
    int P, Q, PB, SB;      // PB p values per pass-A tile, SB slabs per pass-B tile
    int t_first, t_last, t_step;   // stages t_first, t_first + t_step, ..., t_last
    int inverse;
    int out_bf16;
    int col_tiles;         // tiles across the columns
    int64_t ntiles;        // row tiles x col_tiles, tile = row tile * col_tiles + column tile
    int nbuf;              // 2: the next tile's data loads while this one computes; 1: in turn
};

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
    return (uint32_t)__cvta_generic_to_shared(ptr);
}

// Asynchronous global -> shared copies (no register staging), grouped per tile.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// every group but the newest has landed
__device__ __forceinline__ void cp_async_wait_but_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ int tile_row_global(const ColsParams& p, int tile_r, int i) {
    // pass A: tile tile_r covers p = tile_r * PB + pb, its row i = pb * Q + v;
    // pass B: tile tile_r covers slabs tile_r * SB ..., contiguous rows
    if (p.pass_a) {
        const int pb = i / p.Q, v = i - pb * p.Q;
        return tile_r * p.PB + pb + p.P * v;
    }
    return tile_r * p.SB * p.P + i;
}

// One group of b rows of the lane's column; the block comes from the row tile's copy in
// shared memory (every lane reads the same address: a broadcast).
template <int B>
__device__ __forceinline__ void apply_group(float* __restrict__ tile, const ColsParams& p, const float* blk,
                                            const int (&rows)[B], int lane) {
    float w[B * B];
    if constexpr ((B * B) % 4 == 0) {
#pragma unroll
        for (int q = 0; q < B * B / 4; ++q) {
            const float4 v = ((const float4*)blk)[q];
            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < B * B; ++e) w[e] = blk[e];
    }
    float2* t2 = reinterpret_cast<float2*>(tile);
    float2 xv[B];
#pragma unroll
    for (int l = 0; l < B; ++l) xv[l] = t2[rows[l] * (kCols / 2) + lane];
    float2 yv[B];
#pragma unroll
    for (int k = 0; k < B; ++k) yv[k] = make_float2(0.f, 0.f);
    // every output sums over l = 0..b-1 in order
#pragma unroll
    for (int l = 0; l < B; ++l)
#pragma unroll
        for (int k = 0; k < B; ++k) {
            const float c = p.inverse ? w[l * B + k] : w[k * B + l];
            yv[k].x = fmaf(c, xv[l].x, yv[k].x);
            yv[k].y = fmaf(c, xv[l].y, yv[k].y);
        }
#pragma unroll
    for (int k = 0; k < B; ++k) t2[rows[k] * (kCols / 2) + lane] = yv[k];
}

template <int B>
__device__ __forceinline__ void run_stage(float* tile, const float* coef, const ColsParams& p, const StageDesc& sd,
                                          int warp, int lane) {
    // local stride and block count of one problem (a p value in pass A, the slab in B)
    const int sl = p.pass_a ? (int)(sd.s / p.P) : (int)sd.s;
    const int n_local = (p.pass_a ? p.Q : p.P) / B;          // blocks of one problem
    const int n_items = (p.pass_a ? p.PB : p.SB) * n_local;
    for (int item = warp; item < n_items; item += kWarps) {
        const int pb = item / n_local, cl = item - pb * n_local;   // problem, local block
        const int lo = cl % sl, hi = cl / sl;
        const int base = pb * (p.pass_a ? p.Q : p.P) + lo + sl * B * hi;
        int rows[B];
#pragma unroll
        for (int k = 0; k < B; ++k) rows[k] = base + sl * k;
        apply_group<B>(tile, p, coef + item * (B * B), rows, lane);
    }
}

// Items of one stage in a tile: (problem pb, local block cl), item = pb * n_local + cl;
// the global block index of an item.
__device__ __forceinline__ int64_t item_block(const ColsParams& p, const StageDesc& sd, int tile_r, int item) {
    const int n_local = (p.pass_a ? p.Q : p.P) / sd.b;
    const int pb = item / n_local, cl = item - pb * n_local;
    return p.pass_a ? (int64_t)(tile_r * p.PB + pb) + (int64_t)p.P * cl
                    : (int64_t)(tile_r * p.SB + pb) * (p.P / sd.b) + cl;
}

__device__ __forceinline__ int stage_items(const ColsParams& p, const StageDesc& sd) {
    return (p.pass_a ? p.PB * p.Q : p.SB * p.P) / sd.b;
}

// The blocks of every stage of this pass that row tile tile_r's groups use, stage after
// stage (each stage's part starts on a 16-byte boundary), item order.
__device__ __forceinline__ void issue_coefs(const ColsParams& p, float* coef, int tile_r) {
    int off = 0;
    for (int t = p.t_first;; t += p.t_step) {
        const StageDesc& sd = p.pd.st[t];
        const int bb = sd.b * sd.b, n = stage_items(p, sd) * bb;
        if ((bb & 3) == 0 && (sd.block_off & 3) == 0) {   // whole 16-byte pieces
            const int bb4 = bb / 4;
            for (int e = threadIdx.x; e < n / 4; e += kThreads) {
                const int item = e / bb4, k = e - item * bb4;
                cp_async16(coef + off + 4 * e, p.blocks + sd.block_off + item_block(p, sd, tile_r, item) * bb + 4 * k);
            }
        } else {
            for (int e = threadIdx.x; e < n; e += kThreads) {
                const int item = e / bb, k = e - item * bb;
                cp_async4(coef + off + e, p.blocks + sd.block_off + item_block(p, sd, tile_r, item) * bb + k);
            }
        }
        off += (n + 3) & ~3;
        if (t == p.t_last) break;
    }
}

// A tile's data (8 float4 per row): cp.async for whole tiles, plain loads (zero past the last
// column) for the ragged last column tile.
__device__ __forceinline__ void issue_tile(const ColsParams& p, float* buf, int64_t tile, int rows_per_tile) {
    const int tile_r = (int)(tile / p.col_tiles);
    const int col0 = (int)(tile - (int64_t)tile_r * p.col_tiles) * kCols;
    const bool full = col0 + kCols <= p.ncols;
    for (int e = threadIdx.x; e < rows_per_tile * (kCols / 4); e += kThreads) {
        const int i = e / (kCols / 4), cq = e - i * (kCols / 4);
        const float* src = p.x + (int64_t)tile_row_global(p, tile_r, i) * p.ld_x + col0 + 4 * cq;
        if (full) {
            cp_async16((float4*)buf + e, src);
        } else {
            const int c = col0 + 4 * cq;
            float4 v;
            v.x = c < p.ncols ? src[0] : 0.f;
            v.y = c + 1 < p.ncols ? src[1] : 0.f;
            v.z = c + 2 < p.ncols ? src[2] : 0.f;
            v.w = c + 3 < p.ncols ? src[3] : 0.f;
            ((float4*)buf)[e] = v;
        }
    }
}

// Persistent over a contiguous range of tiles (so consecutive tiles mostly share their row
// tile, whose blocks then stay in shared memory).  With two data buffers the next tile's
// copies are in flight while this tile's stages run and its results leave.
__global__ void __launch_bounds__(kThreads, 1) harp_cols_kernel(const __grid_constant__ ColsParams p) {
    extern __shared__ __align__(16) float smem[];
    const int rows_per_tile = p.pass_a ? p.PB * p.Q : p.SB * p.P;
    const int tile_floats = rows_per_tile * kCols;
    float* coef = smem + p.nbuf * tile_floats;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t per = (p.ntiles + gridDim.x - 1) / gridDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * per, t1 = min(p.ntiles, t0 + per);
    if (t0 >= t1) return;
    int loaded_r = -1;   // the row tile whose blocks are in `coef`
    if (p.nbuf == 2) {
        issue_tile(p, smem + (int)(t0 & 1) * tile_floats, t0, rows_per_tile);   // tile j uses buffer j & 1
        cp_async_commit();
    }
    for (int64_t j = t0; j < t1; ++j) {
        const int tile_r = (int)(j / p.col_tiles);
        const int col0 = (int)(j - (int64_t)tile_r * p.col_tiles) * kCols;
        float* buf = smem + (p.nbuf == 2 ? (int)(j & 1) : 0) * tile_floats;
        if (tile_r != loaded_r) {
            // a new row tile: its blocks, waited for at once (at most a few times per CTA);
            // the previous tile's stages are done (the barrier that ended its iteration)
            issue_coefs(p, coef, tile_r);
            cp_async_commit();
            cp_async_wait_all();
            loaded_r = tile_r;
        }
        if (p.nbuf == 2) {
            if (j + 1 < t1) issue_tile(p, smem + (int)((j + 1) & 1) * tile_floats, j + 1, rows_per_tile);
            cp_async_commit();
            cp_async_wait_but_one();   // this tile's copies (and any before them) have landed
        } else {
            issue_tile(p, buf, j, rows_per_tile);
            cp_async_commit();
            cp_async_wait_all();
        }
        __syncthreads();
        int off = 0;
        for (int t = p.t_first;; t += p.t_step) {
            const StageDesc& sd = p.pd.st[t];
            const float* cs = coef + off;
            switch (sd.b) {
                case 2: run_stage<2>(buf, cs, p, sd, warp, lane); break;
                case 3: run_stage<3>(buf, cs, p, sd, warp, lane); break;
                case 4: run_stage<4>(buf, cs, p, sd, warp, lane); break;
                case 5: run_stage<5>(buf, cs, p, sd, warp, lane); break;
                case 6: run_stage<6>(buf, cs, p, sd, warp, lane); break;
                case 7: run_stage<7>(buf, cs, p, sd, warp, lane); break;
                case 8: run_stage<8>(buf, cs, p, sd, warp, lane); break;
                default: break;
            }
            off += (stage_items(p, sd) * sd.b * sd.b + 3) & ~3;
            __syncthreads();
            if (t == p.t_last) break;
        }
        // store: fp32 (16 bytes per thread) or bf16 (8 bytes)
        const bool full = col0 + kCols <= p.ncols;
        for (int e = tid; e < rows_per_tile * (kCols / 4); e += kThreads) {
            const int i = e / (kCols / 4), cq = e - i * (kCols / 4);
            const int64_t row = tile_row_global(p, tile_r, i);
            const int c = col0 + 4 * cq;
            const float4 v = ((const float4*)buf)[e];
            if (p.out_bf16) {
                __nv_bfloat16* dst = (__nv_bfloat16*)p.y + row * p.ld_y + c;
                if (full) {
                    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
                    uint2 u;
                    u.x = *(const uint32_t*)&a;
                    u.y = *(const uint32_t*)&b;
                    *(uint2*)dst = u;
                } else {
                    const float f[4] = {v.x, v.y, v.z, v.w};
                    for (int k = 0; k < 4; ++k)
                        if (c + k < p.ncols) dst[k] = __float2bfloat16_rn(f[k]);
                }
            } else {
                float* dst = (float*)p.y + row * p.ld_y + c;
                if (full) {
                    *(float4*)dst = v;
                } else {
                    const float f[4] = {v.x, v.y, v.z, v.w};
                    for (int k = 0; k < 4; ++k)
                        if (c + k < p.ncols) dst[k] = f[k];
                }
            }
        }
        __syncthreads();   // this buffer's reads are done before the next copies into it
    }
}

}  // namespace

// Column transform of an fp32 matrix x (d rows of ncols, leading dimension ld_x) by
// the plan's T (forward) or T^T (inverse); the result goes to y (fp32 with ld_y, which
// may be x itself, or bf16).  Two passes, each a kernel launch on `stream` with one
// persistent CTA per SM.
harp_status launch_cols(const harp_plan_s* pl, float* x, int64_t ld_x, int64_t ncols, void* y, int64_t ld_y,
                        harp_dtype out_dtype, harp_dir dir, void* stream_) {
    const PlanDesc& pd = pl->desc;
    const int64_t d = pd.d;
    if (pl->composite) return HARP_ERR_UNSUPPORTED;   // the split below needs s_t = prod_{j<t} b_j
    if (pd.m < 2 || ncols <= 0 || ncols > (int64_t)1 << 30) return HARP_ERR_UNSUPPORTED;
    for (int t = 0; t < pd.m; ++t)
        if (pd.st[t].b > 8) return HARP_ERR_UNSUPPORTED;
    if (((uintptr_t)x & 15) || (ld_x & 3) || ((uintptr_t)y & 15) || (ld_y & 3)) return HARP_ERR_UNSUPPORTED;
    // Split t*: a tile row costs nbuf x 256 bytes of data (nbuf data buffers of 64 columns) plus
    // 4 sum_t b_t bytes of the blocks of its pass's stages; pick the split whose larger problem
    // (P or Q rows) is smallest, with two data buffers if some split fits with them.
    const int64_t data_row = kCols * 4;
    auto coef_row = [&](int t0, int t1) {   // bytes of blocks per tile row, stages [t0, t1)
        int64_t s4 = 0;
        for (int t = t0; t < t1; ++t) s4 += 4 * pd.st[t].b + 16;
        return s4;
    };
    int best = -1, nbuf = 2;
    int64_t best_size = 0;
    for (; nbuf >= 1 && best < 0; --nbuf) {
        for (int t = 1; t < pd.m; ++t) {
            const int64_t P = pd.st[t].s, Q = d / P;
            if (P * (nbuf * data_row + coef_row(0, t)) > kSmemBudget ||
                Q * (nbuf * data_row + coef_row(t, pd.m)) > kSmemBudget)
                continue;
            const int64_t size = std::max(P, Q);
            if (best < 0 || size < best_size) best = t, best_size = size;
        }
        if (best >= 0) break;
    }
    if (best < 0) return HARP_ERR_UNSUPPORTED;
    const int P = (int)pd.st[best].s, Q = (int)(d / P);
    const int64_t row_a = nbuf * data_row + coef_row(best, pd.m), row_b = nbuf * data_row + coef_row(0, best);
    int PB = (int)std::min<int64_t>(P, kSmemBudget / (Q * row_a));
    while (P % PB) --PB;
    int SB = (int)std::min<int64_t>(Q, kSmemBudget / (P * row_b));
    while (Q % SB) --SB;
    const int col_tiles = (int)((ncols + kCols - 1) / kCols);
    cudaStream_t stream = (cudaStream_t)stream_;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || nsm <= 0) {
        cudaGetLastError();
        nsm = 1;
    }

    ColsParams cp;
    cp.pd = pd;
    cp.blocks = pl->d_blocks;
    cp.x = x;
    cp.ld_x = ld_x;
    cp.ncols = (int)ncols;
    cp.P = P;
    cp.Q = Q;
    cp.PB = PB;
    cp.SB = SB;
    cp.inverse = dir == HARP_INVERSE;
    cp.col_tiles = col_tiles;
    cp.nbuf = nbuf;
    const bool inv = dir == HARP_INVERSE;
    for (int pass = 0; pass < 2; ++pass) {
        // inverse: A (m-1 .. t*) then B (t*-1 .. 0); forward: B (0 .. t*-1) then A (t* .. m-1)
        const bool a = inv ? pass == 0 : pass == 1;
        cp.pass_a = a;
        if (a) {
            cp.t_first = inv ? pd.m - 1 : best;
            cp.t_last = inv ? best : pd.m - 1;
        } else {
            cp.t_first = inv ? best - 1 : 0;
            cp.t_last = inv ? 0 : best - 1;
        }
        cp.t_step = inv ? -1 : 1;
        const bool last = pass == 1;
        cp.y = last ? y : (void*)x;
        cp.ld_y = last ? ld_y : ld_x;
        cp.out_bf16 = last && out_dtype == HARP_BF16;
        const int row_tiles = a ? P / PB : Q / SB;
        cp.ntiles = (int64_t)row_tiles * col_tiles;
        const size_t smem = (size_t)(a ? PB * Q * row_a : SB * P * row_b);
        cudaError_t e = (cudaError_t)harp_set_smem_limit((const void*)harp_cols_kernel, (int)smem);
        if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
        const int grid = (int)std::min<int64_t>(cp.ntiles, nsm);   // persistent CTAs, one per SM
        harp_cols_kernel<<<(unsigned)grid, kThreads, smem, stream>>>(cp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    }
    harp_set_last_kernel("harp_cols_kernel");
    return HARP_OK;
}
