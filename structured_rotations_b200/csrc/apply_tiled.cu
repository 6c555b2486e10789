// Host launcher of the general tiled row kernel (kernel and layout in apply_tiled.cuh;
// HARP technical summary §2.1 Core Architecture).  Picks the rows per tile R from the
// shared-memory budget, the radix-set instantiation that covers the schedule, and one
// persistent CTA per SM.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "apply_tiled.cuh"
#include "harp_internal.h"

namespace {

harp_tiled::FastDiv make_fast_div(int n) {
    harp_tiled::FastDiv f;
    int l = 0;
    while ((1ll << l) < n) ++l;
    f.l = l;
    f.n = n;
    f.m = (uint32_t)(((1ull << (32 + l)) + (uint64_t)n - 1) / (uint64_t)n - (1ull << 32));
    return f;
}

// Granlund and Montgomery's round-up method ("Division by invariant integers using
// multiplication", 1994, section 4) makes the quotient exact for every 32-bit x when the
// 33-bit sum umulhi(x, m) + x is kept; the kernel divides only x < 2^21, so the sum fits in
// 32 bits.  A cheap check at the edges guards the constants.
bool fast_div_ok(const harp_tiled::FastDiv& f) {
    auto q = [&](uint64_t x) { return (uint32_t)(((((uint64_t)x * f.m) >> 32) + x) >> f.l); };
    const uint64_t n = (uint64_t)f.n;
    const uint64_t xs[] = {0, 1, n - 1, n, n + 1, 2 * n - 1, ((uint64_t)1 << 21) - 1};
    for (uint64_t x : xs)
        if (q(x) != x / n) return false;
    return true;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 1;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

// Test hook (harp_test_inject_wait_timeout): the poll limit and over-declared bytes of the
// next tiled launches on this host thread.
thread_local long long g_inject_limit = 0;
thread_local uint32_t g_inject_extra = 0;

}  // namespace

extern "C" harp_status harp_test_inject_wait_timeout(int64_t poll_limit, uint32_t extra_bytes) {
    harp_clear_error();
    // the barrier's transaction count holds less than 2^20 bytes: the staged rows (under
    // 227 KiB) plus at most 4 KiB stay below it
    if (poll_limit < 0 || (extra_bytes != 0 && poll_limit == 0) || extra_bytes > 4096)
        return harp_fail(HARP_ERR_INVALID_ARG, "poll_limit >= 1 with 1..4096 extra bytes, or (0, 0) to clear");
    g_inject_limit = extra_bytes ? poll_limit : 0;
    g_inject_extra = extra_bytes;
    return HARP_OK;
}

harp_status launch_apply_tiled(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                               int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir,
                               void* stream, const QuantOut* quant) {
    using namespace harp_tiled;
    const int64_t d = p->desc.d;
    if (d % 8 != 0) return HARP_ERR_UNSUPPORTED;
    int mask = 0;
    for (int t = 0; t < p->desc.m; ++t) {
        if (p->desc.st[t].b > 8) return HARP_ERR_UNSUPPORTED;
        mask |= 1 << p->desc.st[t].b;
    }
    if (in_dtype == HARP_F32 && out_dtype == HARP_BF16) return HARP_ERR_UNSUPPORTED;
    if (quant && in_dtype != HARP_BF16) return HARP_ERR_UNSUPPORTED;
    const int64_t es_in = in_dtype == HARP_F32 ? 4 : 2;
    const int64_t es_out = quant ? 1 : out_dtype == HARP_F32 ? 4 : 2;
    if (((uintptr_t)x & 15) || ((uintptr_t)y & 15) || ((ld_x * es_in) & 15) || ((ld_y * es_out) & 15))
        return HARP_ERR_UNSUPPORTED;
    int which = 0;
    while (which < kNumMasks && (kMasks[which] & mask) != mask) ++which;
    if (which == kNumMasks) return HARP_ERR_UNSUPPORTED;

    // Rows per tile R = V Q for a CTA holding dl coordinates of each row: as many sub-tiles
    // of V = 4 rows (fp32, 16 dl bytes each) as fit, then as many of the next tile's raw
    // rows as fit in the rest go to a staging area (bulk copies overlap the arithmetic; the
    // other rows are read directly).  One sub-tile fewer when that would stage fewer than
    // half the rows.  Sub-tiles of one row when not even one 4-row sub-tile fits.
    const int64_t budget = kSmemOptIn - 64;
    struct Shape {
        int V;
        int64_t R, staged;
    };
    auto shape_for = [&](int64_t dl) -> Shape {
        auto staged_for = [&](int64_t r) {
            return std::max<int64_t>(0, std::min<int64_t>(r, (budget - r * dl * 4) / (dl * es_in)));
        };
        Shape sh{4, 0, 0};
        int64_t Q = std::min<int64_t>(budget / (16 * dl), kMaxTileRows / 4);
        if (Q > 1 && staged_for(4 * Q) < 2 * Q) --Q;
        if (Q < 1) {
            sh.V = 1;
            Q = std::min<int64_t>(budget / (4 * dl), kMaxTileRows);
        }
        Q = std::min<int64_t>(Q, (rows + sh.V - 1) / sh.V);
        sh.R = sh.V * Q;
        sh.staged = sh.R > 0 ? std::min<int64_t>(staged_for(sh.R), rows) : 0;
        return sh;
    };
    // Slab mode (a cluster of two CTAs, each with half of every row) for schedules whose
    // last radix is 2, when it doubles the rows per tile.  Opt-in (HARP_TILED_SLAB=1): it
    // halves the coefficient stream per row but measured no faster than whole rows on
    // B200 (d = 8192: equal; d = 5120: slower), whose limit here is issue rate.
    const PlanDesc& pd = p->desc;
    int cl = 1;
    Shape sh = shape_for(d);
    {
        const char* env = std::getenv("HARP_TILED_SLAB");
        bool ok = !quant && !p->composite && env && !std::strcmp(env, "1") && pd.m >= 2 && pd.st[pd.m - 1].b == 2 && d % 16 == 0 &&
                  has_slab_kernel(kMasks[which]) && (pd.st[pd.m - 1].block_off & 3) == 0;
        for (int t = 0; ok && t < pd.m - 1; ++t) ok = ((d / 2) / pd.st[t].b) % 32 == 0;
        if (ok) {
            const Shape s2 = shape_for(d / 2);
            if (s2.V == 4 && s2.R >= 2 * sh.R) {
                sh = s2;
                cl = 2;
            }
        }
    }
    // Small batches (decode-shaped): 4-row sub-tiles would pad rows with zeros and leave
    // most SMs idle, so one-row sub-tiles spread the rows over as many SMs as possible.
    if (cl == 1 && sh.V == 4 && rows < 4 * (int64_t)sm_count() && has_row_major_kernel(kMasks[which])) {
        const char* env = std::getenv("HARP_TILED_SMALL");
        if (!(env && !std::strcmp(env, "0"))) {
            const int64_t r1 = std::min<int64_t>((rows + sm_count() - 1) / sm_count(), budget / (4 * d));
            if (r1 >= 1) {
                sh.V = 1;
                sh.R = r1;
                sh.staged = std::max<int64_t>(0, std::min<int64_t>(r1, (budget - r1 * d * 4) / (d * es_in)));
            }
        }
    }
    const int V = sh.V;
    const int64_t R = sh.R, staged = sh.staged, dl = d / cl;
    if (R < 1 || (V == 1 && !has_row_major_kernel(kMasks[which]))) return HARP_ERR_UNSUPPORTED;

    TiledParams tp;
    tp.pd = pd;
    tp.scales = quant ? quant->scales : nullptr;
    tp.ld_s = quant ? quant->ld_s : 0;
    tp.qlanes = quant ? quant->qblock / 8 : 1;
    tp.lanes = p->d_blocks_lanes;
    for (int t = 0; t < HARP_MAX_STAGES; ++t) tp.lane_off[t] = p->lane_off[t];
    tp.x = x;
    tp.y = y;
    tp.rows = rows;
    tp.ld_x = ld_x;
    tp.ld_y = ld_y;
    tp.ntiles = (rows + R - 1) / R;
    tp.R = (int)R;
    tp.staged_rows = (int)staged;
    tp.mask = (dl % 32 == 0) ? 0x18 : 0;
    tp.status = p->d_status;
    // stages applied while filling / draining: radix 8 at stride 1, radix 2 at stride d / 2
    // (whole rows in 4-row sub-tiles; the quantizer's drain keeps its stage).  Only when a tile
    // is a single sub-tile (d = 8192: R = 4), where a pass over the tile is the largest share of
    // the work: the fused fill and drain need 256 threads (more registers than a 384-thread CTA
    // allows), which measured slower than the passes they save at d = 5120 (R = 8) and equal at
    // d = 4096 (B200: d = 8192 forward 2.36 -> 2.12 ms, d = 5120 forward 1.24 -> 1.33 ms).
    {
        auto kind_of = [&](int t) {
            const StageDesc& sd = pd.st[t];
            if (sd.b == 8 && sd.s == 1) return (int)kFuseS1R8;
            if (sd.b == 2 && 2 * sd.s == d) return (int)kFuseH2R2;
            return (int)kFuseNone;
        };
        const bool can = sh.V == 4 && sh.R == 4 && cl == 1 && !std::getenv("HARP_TILED_NOFUSE");
        const bool inv = dir == HARP_INVERSE;
        tp.fuse_first = can ? kind_of(inv ? pd.m - 1 : 0) : kFuseNone;
        tp.fuse_last = can && !quant && pd.m >= 2 ? kind_of(inv ? 0 : pd.m - 1) : kFuseNone;
    }
    tp.wait_limit = g_inject_extra ? g_inject_limit : kWaitLimit;
    tp.extra_tx = g_inject_extra;
    tp.last_blocks = p->d_blocks + pd.st[pd.m - 1].block_off;
    for (int t = 0; t < pd.m; ++t) {
        tp.nb_div[t] = make_fast_div((int)(dl / pd.st[t].b));
        tp.s_div[t] = make_fast_div((int)pd.st[t].s);
        if (!fast_div_ok(tp.nb_div[t]) || !fast_div_ok(tp.s_div[t])) return HARP_ERR_UNSUPPORTED;
    }
    const size_t smem = (size_t)R * dl * 4 + (size_t)staged * dl * es_in + 16;
    const int grid = cl * (int)std::min<int64_t>(tp.ntiles, sm_count() / cl);
    int nt = kThreadChoices[1];
    {
        const int qv = (int)((std::min<int64_t>(R, rows) + V - 1) / V);
        for (int t = 0; t < pd.m - (cl == 2 ? 1 : 0); ++t)
            if (stage_groups((int)(dl / pd.st[t].b), qv, kThreadChoices[1]) > 1) nt = kThreadChoices[0];
        // the fused fill / drain need more than the 168 registers a 384-thread CTA allows
        if (tp.fuse_first || tp.fuse_last) nt = kThreadChoices[0];
    }
    cudaStream_t s = (cudaStream_t)stream;
    const bool inv = dir == HARP_INVERSE;
    cudaError_t e;
    if (quant)
        e = harp_tiled_launch_bf16_i8(which, V, nt, cl, inv, tp, smem, grid, s);
    else if (in_dtype == HARP_BF16 && out_dtype == HARP_BF16)
        e = harp_tiled_launch_bf16(which, V, nt, cl, inv, tp, smem, grid, s);
    else if (in_dtype == HARP_F32)
        e = harp_tiled_launch_f32(which, V, nt, cl, inv, tp, smem, grid, s);
    else
        e = harp_tiled_launch_bf16_f32(which, V, nt, cl, inv, tp, smem, grid, s);
    if (e != cudaSuccess) return harp_fail(HARP_ERR_CUDA, cudaGetErrorString(e));
    harp_set_last_kernel("harp_tiled_kernel");
    return HARP_OK;
}
