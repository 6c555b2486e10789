// Host side of the cluster row kernel (device code and layouts in apply_cluster.cuh; HARP
// technical summary §2.1 Core Architecture).  At materialization a plan that qualifies gets a
// split (stage t*, cluster size CL) and its cluster table: for every cluster rank, the blocks
// that rank applies, per stage in its local block order, lane-interleaved in groups of 32, so a
// rank's blocks are one contiguous segment that a single bulk copy stages in shared memory.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "apply_cluster.cuh"
#include "harp_internal.h"

int harp_cluster_max_active(int which, int cl, size_t smem);   // apply_cluster_bf16.cu

namespace {

using harp_cluster::ClusterParams;
using harp_tiled::FastDiv;

constexpr int64_t kSmemBudget = 227 * 1024 - 128;
constexpr int kMaxTileRows = 32;

FastDiv fast_div(int n) {
    FastDiv f;
    int l = 0;
    while ((1ll << l) < n) ++l;
    f.l = l;
    f.n = n;
    f.m = (uint32_t)(((1ull << (32 + l)) + (uint64_t)n - 1) / (uint64_t)n - (1ull << 32));
    return f;
}

// The multiply-shift quotient (Granlund and Montgomery's round-up method) checked at the
// edges of the range the kernel divides (x < 2^21).
bool fast_div_ok(const FastDiv& f) {
    auto q = [&](uint64_t x) { return (uint32_t)(((((uint64_t)x * f.m) >> 32) + x) >> f.l); };
    const uint64_t n = (uint64_t)f.n;
    const uint64_t xs[] = {0, 1, n - 1, n, n + 1, 2 * n - 1, ((uint64_t)1 << 21) - 1};
    for (uint64_t x : xs)
        if (q(x) != x / n) return false;
    return true;
}

// The split a plan takes (stage t*, cluster size) and the sizes that follow from it.
struct Split {
    int which = 0;                 // radix-set instantiation
    int cl = 0, t_split = 0, dl = 0, S = 0, P = 0;
    int64_t seg_floats = 0;
    int64_t stage_off[HARP_MAX_STAGES] = {};
    int r_max = 0;                 // rows per tile the shared-memory budget allows
    int max_clusters = 0;          // clusters resident at once (the persistent grid)
};

struct ClusterState : Split {
    float* table = nullptr;
    cudaEvent_t built = nullptr;   // recorded after the table's build
    std::atomic<bool> done{false}; // `built` has completed
};

// Shared memory of a CTA: its blocks, two buffers of R rows, one mbarrier per stage and one
// for the exchange.
size_t smem_bytes(int64_t seg_floats, int R, int dl) {
    return (size_t)seg_floats * 4 + 2 * (size_t)R * dl * 4 + 8 * (HARP_MAX_STAGES + 1);
}

int64_t stage_floats(int64_t nb_loc, int b) { return (nb_loc + 31) / 32 * 32 * b * b; }

// Rank r's local blocks of stage t, lane-interleaved: local block c_l of phase A is global
// block c_l + r nb_loc; of phase B (local order l = j P + p), global block r P + c_l % P +
// S (c_l / P).
__global__ void cluster_table_kernel(const float* __restrict__ blocks, float* __restrict__ table, int64_t seg,
                                     int64_t off, int cl, int nb_loc, int bb, int phase_a, int P, int S) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)cl * nb_loc * bb;
    if (idx >= total) return;
    const int e = (int)(idx % bb);
    const int c_loc = (int)((idx / bb) % nb_loc);
    const int r = (int)(idx / ((int64_t)bb * nb_loc));
    const int64_t c = phase_a ? (int64_t)c_loc + (int64_t)r * nb_loc : (int64_t)r * P + c_loc % P + (int64_t)S * (c_loc / P);
    const int group = c_loc >> 5, lane = c_loc & 31;
    const int64_t to = (bb % 4 == 0) ? (((int64_t)group * (bb / 4) + e / 4) * 32 + lane) * 4 + (e & 3)
                                     : ((int64_t)group * bb + e) * 32 + lane;
    table[(int64_t)r * seg + off + to] = blocks[c * bb + e];
}

int radix_set(const PlanDesc& pd) {
    int mask = 0;
    for (int t = 0; t < pd.m; ++t) {
        if (pd.st[t].b > 8) return -1;
        mask |= 1 << pd.st[t].b;
    }
    int which = 0;
    while (which < harp_tiled::kNumMasks && (harp_tiled::kMasks[which] & mask) != mask) ++which;
    return which == harp_tiled::kNumMasks ? -1 : which;
}

}  // namespace

void cluster_prepare(harp_plan_s* p, void* stream) {
    if (p->cluster || p->composite) return;
    const PlanDesc& pd = p->desc;
    const int64_t d = pd.d;
    const int which = radix_set(pd);
    if (which < 0 || d % 8 || pd.m < 2) return;
    Split best;
    for (int cl : {16, 8, 4, 2}) {
        for (int ts = 1; ts < pd.m; ++ts) {
            const int64_t S = pd.st[ts].s, N = d / S;
            if (S % cl || N % cl || (S / cl) % 8) continue;
            Split c;
            c.which = which;
            c.cl = cl;
            c.t_split = ts;
            c.dl = (int)(d / cl);
            c.S = (int)S;
            c.P = (int)(S / cl);
            int64_t off = 0;
            for (int t = 0; t < pd.m; ++t) {
                c.stage_off[t] = off;
                off += stage_floats(c.dl / pd.st[t].b, pd.st[t].b);
            }
            c.seg_floats = off;
            const int64_t per_row = 2 * (int64_t)c.dl * 4;
            c.r_max = (int)std::min<int64_t>(
                kMaxTileRows, (kSmemBudget - c.seg_floats * 4 - 8 * (HARP_MAX_STAGES + 1)) / per_row / 4 * 4);
            if (c.r_max < 4) continue;
            if (c.P > best.P || best.cl == 0) best = c;   // within one CL, the longest output runs
        }
        if (best.cl == 0) continue;
        best.max_clusters = harp_cluster_max_active(best.which, best.cl, smem_bytes(best.seg_floats, best.r_max, best.dl));
        if (best.max_clusters >= 1) break;
        best = Split();   // this cluster size does not fit on the device: try a smaller one
    }
    if (best.cl == 0) return;
    ClusterState* cs = new ClusterState();
    static_cast<Split&>(*cs) = best;
    const size_t bytes = (size_t)cs->cl * cs->seg_floats * sizeof(float);
    if (cudaMalloc((void**)&cs->table, bytes) != cudaSuccess) {
        cudaGetLastError();
        delete cs;
        return;
    }
    cudaStream_t s = (cudaStream_t)stream;
    cudaMemsetAsync(cs->table, 0, bytes, s);
    for (int t = 0; t < pd.m; ++t) {
        const int b = pd.st[t].b;
        const int nb_loc = cs->dl / b;
        const int64_t n = (int64_t)cs->cl * nb_loc * b * b;
        cluster_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
            p->d_blocks + pd.st[t].block_off, cs->table, cs->seg_floats, cs->stage_off[t], cs->cl, nb_loc, b * b,
            t < cs->t_split ? 1 : 0, cs->P, cs->S);
    }
    if (cudaGetLastError() != cudaSuccess ||
        cudaEventCreateWithFlags(&cs->built, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(cs->built, s) != cudaSuccess) {
        cudaGetLastError();
        if (cs->built) cudaEventDestroy(cs->built);
        cudaFree(cs->table);
        delete cs;
        return;
    }
    p->cluster = cs;
}

void cluster_state_free(harp_plan_s* p) {
    ClusterState* cs = static_cast<ClusterState*>(p->cluster);
    if (!cs) return;
    cudaFree(cs->table);
    if (cs->built) cudaEventDestroy(cs->built);
    delete cs;
    p->cluster = nullptr;
}

harp_status launch_apply_cluster(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                                 int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir, void* stream) {
    ClusterState* cs = static_cast<ClusterState*>(p->cluster);
    if (!cs) return HARP_ERR_UNSUPPORTED;
    if (in_dtype == HARP_F32 && out_dtype == HARP_BF16) return HARP_ERR_UNSUPPORTED;
    const int64_t es_in = in_dtype == HARP_F32 ? 4 : 2, es_out = out_dtype == HARP_F32 ? 4 : 2;
    if (((uintptr_t)x & 15) || ((uintptr_t)y & 15) || ((ld_x * es_in) & 15) || ((ld_y * es_out) & 15))
        return HARP_ERR_UNSUPPORTED;
    const PlanDesc& pd = p->desc;
    ClusterParams cp;
    cp.pd = pd;
    cp.table = cs->table;
    cp.seg_floats = cs->seg_floats;
    for (int t = 0; t < HARP_MAX_STAGES; ++t) cp.stage_off[t] = cs->stage_off[t];
    for (int t = 0; t < pd.m; ++t) {
        cp.ls[t] = (int)(t < cs->t_split ? pd.st[t].s : pd.st[t].s / cs->cl);
        cp.nb_div[t] = fast_div(cs->dl / pd.st[t].b);
        cp.s_div[t] = fast_div(cp.ls[t]);
        if (!fast_div_ok(cp.nb_div[t]) || !fast_div_ok(cp.s_div[t])) return HARP_ERR_UNSUPPORTED;
    }
    cp.t_split = cs->t_split;
    cp.cl = cs->cl;
    cp.dl = cs->dl;
    cp.S = cs->S;
    cp.P = cs->P;
    cp.S_div = fast_div(cs->S);
    cp.P_div = fast_div(cs->P);
    cp.dl_div = fast_div(cs->dl);
    if (!fast_div_ok(cp.S_div) || !fast_div_ok(cp.P_div) || !fast_div_ok(cp.dl_div)) return HARP_ERR_UNSUPPORTED;
    cp.x = x;
    cp.y = y;
    cp.rows = rows;
    cp.ld_x = ld_x;
    cp.ld_y = ld_y;
    cp.R = (int)std::min<int64_t>(cs->r_max, (rows + 3) / 4 * 4);
    cp.status = p->d_status;
    if (!cs->done.load(std::memory_order_acquire)) {
        // the table's build has finished once its event has (a poll, no wait)
        const cudaError_t q = cudaEventQuery(cs->built);
        if (q == cudaSuccess) cs->done.store(true, std::memory_order_release);
        else if (q != cudaErrorNotReady) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(q));
    }
    cp.early = cs->done.load(std::memory_order_acquire) ? 1 : 0;
    const int64_t ntiles = (rows + cp.R - 1) / cp.R;
    const size_t smem = smem_bytes(cs->seg_floats, cp.R, cs->dl);
    const int grid = (int)(std::min<int64_t>(ntiles, cs->max_clusters) * cs->cl);   // persistent clusters
    cudaStream_t s = (cudaStream_t)stream;
    const bool inv = dir == HARP_INVERSE;
    cudaError_t e;
    if (in_dtype == HARP_BF16 && out_dtype == HARP_BF16)
        e = harp_cluster_launch_bf16(cs->which, cs->cl, inv, cp, smem, grid, s);
    else if (in_dtype == HARP_F32)
        e = harp_cluster_launch_f32(cs->which, cs->cl, inv, cp, smem, grid, s);
    else
        e = harp_cluster_launch_bf16_f32(cs->which, cs->cl, inv, cp, smem, grid, s);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_cluster_kernel");
    return HARP_OK;
}
