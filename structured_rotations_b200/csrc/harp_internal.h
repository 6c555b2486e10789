// Internal declarations shared by the host plan code and the CUDA launchers.
#pragma once

#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "harp.h"

struct StageDesc {
    int32_t b;          // radix b_t
    int32_t p;          // parameters per block (1 for b=2, b(b-1)/2 otherwise)
    int64_t s;          // stride s_t = prod_{j<t} b_j
    int64_t nblocks;    // d / b_t
    int64_t theta_off;  // first parameter of the stage
    int64_t block_off;  // first float of the stage's blocks (nblocks * b * b floats)
    int32_t mixer_off;  // first double of G_{b_t} in the packed mixer table
};

struct PlanDesc {       // passed by value to kernels
    int64_t d;
    int32_t m;
    StageDesc st[HARP_MAX_STAGES];
};

struct harp_plan_s {
    PlanDesc desc;
    harp_theta_kind kind;
    std::vector<float> theta_f32;
    std::vector<int8_t> theta_i8;
    std::vector<float> scales;
    uint64_t sign_seed = 0, qr_seed = 0;
    std::vector<int8_t> signs;                  // +1 / -1, length d
    std::vector<double> mixers;                 // packed G_b, row-major
    std::map<int, int> mixer_index;             // radix -> offset into mixers
    int64_t theta_total = 0;
    int64_t block_floats = 0;
    // Lane-interleaved copy of the blocks for the tiled kernel: per stage, blocks in groups
    // of 32 consecutive c; inside a group, 16-byte piece q of block c at
    // (group * (b*b/4) + q) * 32 + (c % 32) (in float4 units) when b*b % 4 == 0, else
    // float e of block c at (group * b*b + e) * 32 + (c % 32).  A warp whose lanes take 32
    // consecutive blocks then reads 512 (128) contiguous bytes per load.
    int64_t lane_off[HARP_MAX_STAGES] = {0};
    int64_t lane_floats = 0;

    // device side (owned)
    int device = -1;
    // Set last by materialization, once the blocks (and every table a kernel reads) are
    // built; atomic so that a call that sees it set also sees the finished device state.
    std::atomic<bool> materialized{false};
    std::mutex materialize_mu;        // explicit and implicit (int8) materialization take turns
    bool composite = false;           // built by harp_plan_compose: stages of several plans in a row
    float* d_blocks = nullptr;        // signed blocks, [stage][c][k][l]
    float* d_blocks_lanes = nullptr;  // the same, lane-interleaved (see lane_off)
    void* d_theta = nullptr;          // float or int8 codes, as stored
    float* d_scales = nullptr;
    double* d_mixers = nullptr;
    int8_t* d_signs = nullptr;
    int* d_status = nullptr;          // device error word (bounded waits)
    void* fast = nullptr;             // fast-path state (see apply_fast.cu)
    void* cluster = nullptr;          // cluster-kernel split and table (see apply_cluster.cu)
    void* host_io = nullptr;          // streams and staging buffers of harp_apply_host (host_io.cu)
    std::mutex host_io_mu;            // harp_apply_host calls on this plan take turns
};

// true if the byte ranges [a, a + na) and [b, b + nb) share a byte (api.cu)
bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb);

// error reporting (plan.cpp)
harp_status harp_fail(harp_status s, const std::string& msg);
void harp_clear_error();
void harp_set_last_kernel(const char* name);
// Raises a kernel's dynamic shared-memory limit (cudaFuncAttributeMaxDynamicSharedMemorySize)
// to at least `bytes` on the current device; the runtime call is made only the first time a
// kernel needs more than before, since it costs microseconds on every launch otherwise.
int harp_set_smem_limit(const void* kernel, int bytes);

// device helpers (materialize.cu)
harp_status harp_device_free(harp_plan_s* p);
// HARP_OK if the plan is materialized.  An int8 plan that is not is materialized here on
// `stream`, which is then synchronized before the plan is marked ready, so that a call
// from another stream or thread that finds it ready reads finished blocks.  Other plans
// return HARP_ERR_NOT_MATERIALIZED.
harp_status harp_require_materialized(harp_plan_s* p, void* stream);

// launchers (apply_simple.cu / transpose.cu)
harp_status launch_apply_simple(const harp_plan_s* p, const void* x, void* y, int64_t rows,
                                int64_t ld_x, int64_t ld_y, harp_dtype in_dtype,
                                harp_dtype out_dtype, harp_dir dir, void* stream);
harp_status launch_transpose(const void* src, void* dst, int64_t rows, int64_t cols,
                             int64_t ld_src, int64_t ld_dst, harp_dtype in_dtype,
                             harp_dtype out_dtype, void* stream);

// fast path (apply_fast.cu): returns HARP_ERR_UNSUPPORTED when the shape has no
// specialized kernel, in which case the caller uses the simple kernel.
harp_status launch_apply_fast(harp_plan_s* p, const void* x, void* y, int64_t rows,
                              int64_t ld_x, int64_t ld_y, harp_dtype in_dtype, harp_dir dir,
                              void* stream, harp_dtype out_dtype);
void fast_state_free(harp_plan_s* p);
// Chooses the cluster kernel's split for plans it covers and builds their cluster table on
// `stream` (apply_cluster.cu); a no-op for other plans, which then never take that kernel.
void cluster_prepare(harp_plan_s* p, void* stream);
void cluster_state_free(harp_plan_s* p);
// Cluster row kernel (apply_cluster.cu): HARP_ERR_UNSUPPORTED for plans without a cluster
// table, unaligned rows and fp32-in / bf16-out.
harp_status launch_apply_cluster(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                                 int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir,
                                 void* stream);
// Builds the specialized kernel's coefficient table (and its launch attributes) on
// `stream` for plans it covers; a no-op for other plans.  Called by materialization, so
// every later launch only reads the table.  A plan whose table cannot be built (no
// cluster fits, no tensor-map encoder) is left without one and runs on the other kernels.
// The specialized kernel with the blockwise quantizer as its epilogue (harp_apply_quant on a
// d = 4096 (8,8,8,8) plan, forward); HARP_ERR_UNSUPPORTED for anything else.
harp_status launch_apply_fast_quant(harp_plan_s* p, const void* x, int64_t rows, int64_t ld_x, int8_t* q,
                                    int64_t ld_q, float* scales, int64_t ld_s, int qblock, harp_dir dir,
                                    void* stream);
void fast_prepare(harp_plan_s* p, void* stream);
void host_io_free(harp_plan_s* p);

// the row kernels in order of preference (api.cu)
harp_status run_rows(harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x, int64_t ld_y,
                     harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir, void* stream);

// Column transform for the two-sided rotation (cols.cu): every column of an fp32 matrix
// x (d rows) takes T (forward) or T^T (inverse); result to y (fp32, may be x, or bf16).
// HARP_ERR_UNSUPPORTED for schedules it does not cover (radix > 8, one stage, ...).
harp_status launch_cols(const harp_plan_s* p, float* x, int64_t ld_x, int64_t ncols, void* y, int64_t ld_y,
                        harp_dtype out_dtype, harp_dir dir, void* stream);

// Int8 output of the tiled kernel (the fused quantizer epilogue): y receives int8 codes,
// `scales` one fp32 scale per block of `qblock` coordinates (row stride ld_s floats).
struct QuantOut {
    float* scales;
    int64_t ld_s;
    int qblock;
};

// General tiled row kernel (apply_tiled.cu): radices 2..8, d % 8 == 0, 16-byte aligned
// rows.  Returns HARP_ERR_UNSUPPORTED for other shapes.
harp_status launch_apply_tiled(const harp_plan_s* p, const void* x, void* y, int64_t rows, int64_t ld_x,
                               int64_t ld_y, harp_dtype in_dtype, harp_dtype out_dtype, harp_dir dir,
                               void* stream,
                               const struct QuantOut* quant = nullptr);
