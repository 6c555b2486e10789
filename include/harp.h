/*
 * harp.h — C ABI of libharp, a B200 (sm_100a) implementation of the HARP
 * stride-staged block-orthogonal rotation.
 *
 * The operation (HARP technical summary, gist.science, "Technical Summary: HARP
 * (Hadamard-Preconditioned Adaptive Rotation Processor)"):
 *   §2.1 Core Architecture — a mixed-radix schedule b = (b_0, ..., b_{m-1}) with
 *        prod b_t = d; stage t applies a block-diagonal orthogonal matrix to
 *        groups of b_t coordinates separated by a stride permutation.
 *   §2.2 Hadamard Preconditioning — each block is B_{t,c}(theta) = Q_{t,c}(theta)
 *        G_{b_t}; G is the normalized Sylvester Hadamard for power-of-two radices
 *        and a QR fallback of a fixed Gaussian matrix otherwise; Q is a Givens
 *        rotation for b_t = 2 and a Cayley map for b_t > 2; theta = 0 recovers
 *        the fixed randomized Hadamard transform.
 *   §2.4 Deployment Efficiency — theta may be stored as int8.
 *   Abstract — a two-sided processor: a rotation on each side of a weight matrix.
 *
 * Conventions fixed by this library (the pages leave them open):
 *   strides      s_t = prod_{j<t} b_j; index i = sum_t i_t s_t, digit 0 least
 *                significant; stage t mixes digit t.  The group of stage t that
 *                holds block c = lo + s_t*hi (0 <= lo < s_t) is the b_t coordinates
 *                lo + s_t*(k + b_t*hi), k = 0..b_t-1.
 *   transform    T = M_{m-1} ... M_1 M_0 S, where S = diag(+-1) and
 *                (M_t x)[lo + s_t(k + b_t hi)] = sum_l B_{t,c}[k][l] x[lo + s_t(l + b_t hi)].
 *   signs        s_i = -1 if bit 63 of the i-th SplitMix64 output of sign_seed is
 *                set, +1 otherwise (SplitMix64: state += 0x9E3779B97F4A7C15, then
 *                the published 64-bit finalizer).
 *   mixers       power of two: G[k][l] = (-1)^popcount(k&l) / sqrt(b).  Otherwise
 *                one matrix per radix value: b*b standard normals, row-major, from
 *                the SplitMix64 stream seeded with (qr_seed ? qr_seed :
 *                0x4841525000000000) + b, two outputs per entry, U = (u >> 11) 2^-53,
 *                g = sqrt(-2 ln(1 - U1)) cos(2 pi U2); G = Q diag(sign(R_kk)) from the
 *                Householder QR M = QR (sign(0) = +1).
 *   theta layout stages t = 0..m-1 in order; within a stage, blocks c = 0..d/b_t-1;
 *                per block p_t parameters: p_t = 1 (Givens angle) if b_t = 2, else
 *                b_t(b_t-1)/2 entries of the strict upper triangle of A in
 *                row-major order ((0,1), (0,2), ..., (0,b-1), (1,2), ...), with
 *                A[j][i] = -A[i][j] and Q = (I - A)^{-1} (I + A).
 *                Givens: Q = [[cos, -sin], [sin, cos]].
 *   int8 theta   theta = q * scales[t] for every parameter of stage t.
 *
 * Memory and streams:
 *   * Every pointer named "host" is host memory; every activation/weight/output
 *     pointer is device memory owned by the caller.  The plan owns copies of theta,
 *     the signs, the mixers and the materialized blocks.
 *   * All device work is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Argument errors are returned synchronously and leave
 *     the stream untouched.  Launch errors return HARP_ERR_CUDA; faults of earlier
 *     work surface at the next synchronizing call.
 *   * Rows are dense vectors of length d; row r starts at x + r*ld elements.
 *     ld >= d.  bf16 rows must start on 16-byte boundaries for the vectorized paths
 *     (the library falls back to a scalar kernel otherwise, never to the CPU).
 */
#ifndef HARP_H_
#define HARP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HARP_API __attribute__((visibility("default")))
#else
#define HARP_API
#endif

#define HARP_MAX_STAGES 16
#define HARP_MAX_RADIX 16
#define HARP_MAX_DIM 32768

typedef struct harp_plan_s* harp_plan_t;

typedef enum {
    HARP_OK = 0,
    HARP_ERR_INVALID_ARG = 1,     /* null pointer, bad size, bad stride, partial aliasing */
    HARP_ERR_SCHEDULE = 2,        /* prod b_t != d, radix outside [2, 16], too many stages */
    HARP_ERR_UNSUPPORTED = 3,     /* dtype / direction value not known */
    HARP_ERR_NOT_MATERIALIZED = 4,/* harp_apply before harp_materialize_blocks (float theta) */
    HARP_ERR_ALLOC = 5,           /* device or host allocation failed */
    HARP_ERR_CUDA = 6,            /* a CUDA runtime call or launch failed */
    HARP_ERR_TIMEOUT = 7,         /* a bounded device-side wait gave up */
    HARP_ERR_WRONG_DEVICE = 8     /* plan materialized on another device */
} harp_status;

typedef enum { HARP_THETA_F32 = 0, HARP_THETA_I8 = 1 } harp_theta_kind;
typedef enum { HARP_F32 = 0, HARP_BF16 = 1 } harp_dtype;
/* FORWARD: y = T x.  INVERSE: y = T^T x (exact inverse; T is orthogonal). */
typedef enum { HARP_FORWARD = 0, HARP_INVERSE = 1 } harp_dir;

/*
 * harp_plan_create — validate a schedule and build the host side of a plan
 * (§2.1 schedule, §2.2 blocks).  Host only: no CUDA call is made.
 *   out        receives the new plan (unchanged on error).
 *   d          dimension, 2 <= d <= HARP_MAX_DIM.
 *   radices    host array of m radices, each in [2, HARP_MAX_RADIX], product d.
 *   m          number of stages, 1 <= m <= HARP_MAX_STAGES.
 *   kind       HARP_THETA_F32: theta is a host float array; HARP_THETA_I8: theta
 *              is a host int8 array of codes and `scales` holds m floats.
 *   theta      harp_theta_count(radices, m) parameters in the layout above; NULL
 *              means all zeros (the fixed randomized Hadamard transform).
 *   scales     m per-stage scales for HARP_THETA_I8, ignored (may be NULL) for F32.
 *   sign_seed  seed of the sign diagonal S.
 *   qr_seed    0 selects the default seed base for the non-power-of-two mixers.
 * Returns HARP_ERR_SCHEDULE / HARP_ERR_INVALID_ARG on bad input, HARP_ERR_ALLOC if
 * host memory runs out.  The plan copies everything it needs.
 */
HARP_API harp_status harp_plan_create(harp_plan_t* out, int64_t d, const int32_t* radices, int32_t m,
                             harp_theta_kind kind, const void* theta, const float* scales,
                             uint64_t sign_seed, uint64_t qr_seed);

/*
 * harp_materialize_blocks — upload theta (as stored: float or int8 codes plus
 * scales), signs and mixers to the current device and build every block
 * B_{t,c} = Q_{t,c}(theta) G_{b_t} on the device (§2.2; int8 codes are
 * dequantized inside the kernel, §2.4).  Blocks are computed in double and stored
 * as float32; the sign diagonal is folded into the stage-0 blocks.  Allocates
 * device memory owned by the plan on first use.  Idempotent; a second call on
 * another device returns HARP_ERR_WRONG_DEVICE.  Also builds, on `stream`, the
 * coefficient table of the specialized d = 4096 (8,8,8,8) kernel for plans it covers,
 * so that applies only read plan state.  Calls on one plan from several host threads
 * take turns (a lock of the plan's).
 */
HARP_API harp_status harp_materialize_blocks(harp_plan_t plan, void* stream);

/*
 * harp_apply — y_r = T x_r (FORWARD) or y_r = T^T x_r (INVERSE) for rows r < rows
 * (§2.1 stages, §2.2 blocks; the inverse is the exact change of basis back).
 *   x, y        device pointers, element type `dtype` (HARP_F32: float,
 *               HARP_BF16: bfloat16 bits); y may equal x (in place); any other
 *               overlap of the two row ranges returns HARP_ERR_INVALID_ARG.
 *   rows        number of rows; 0 is a no-op returning HARP_OK.
 *   ld_x, ld_y  leading dimensions in elements, >= d.
 * Arithmetic: inputs widened to fp32, every stage accumulated in fp32 with fused
 * multiply-adds (the specialized d = 4096 kernel forms the products on tensor cores from
 * TF32 hi/lo splits of both operands, three passes, fp32 accumulation), the output
 * rounded to `dtype` to nearest even.
 * Concurrency: a plan is immutable once materialized (every table a kernel reads is
 * built by harp_materialize_blocks), so calls on different streams or host threads may
 * run at once; order them after the materialization (same stream, an event or a
 * synchronize).
 * Materialization: a HARP_THETA_F32 plan that was not materialized returns
 * HARP_ERR_NOT_MATERIALIZED.  A HARP_THETA_I8 plan materializes implicitly on its first
 * call (its int8 codes are dequantized by the block-building kernel on the call's stream,
 * which that call then synchronizes; concurrent first calls take turns on a lock of the
 * plan and only one builds).  The same holds for every entry point below that takes a
 * plan.
 */
HARP_API harp_status harp_apply(harp_plan_t plan, const void* x, void* y, int64_t rows,
                       int64_t ld_x, int64_t ld_y, harp_dtype dtype, harp_dir dir,
                       void* stream);

/*
 * harp_apply_ex — harp_apply with separate input and output types (for example bf16 rows
 * in, fp32 rows out, to keep an intermediate unrounded).  y may equal x only when the two
 * types are equal.  Everything else as harp_apply.
 */
HARP_API harp_status harp_apply_ex(harp_plan_t plan, const void* x, void* y, int64_t rows,
                                   int64_t ld_x, int64_t ld_y, harp_dtype in_dtype,
                                   harp_dtype out_dtype, harp_dir dir, void* stream);

/*
 * harp_apply_host — harp_apply between host buffers, copies included: y_r = T x_r
 * (FORWARD) or T^T x_r (INVERSE) for rows in host memory.  The rows pass through the GPU in
 * chunks of about 32 MiB on three streams owned by the plan, so that host-to-device copies,
 * kernels and device-to-host copies overlap (page-locked host memory is needed for the
 * overlap; pageable memory works, the copies then serialize).  Synchronous: returns when y
 * holds the result.  Runs on the current device, which must be the plan's.  The plan keeps
 * the streams and six device buffers of one chunk until harp_plan_destroy; calls on one
 * plan from several host threads take turns (a lock of the plan's).
 *   x, y        host pointers, element type dtype; y may equal x (then ld_x == ld_y); any
 *               other overlap returns HARP_ERR_INVALID_ARG.
 *   rows, ld_x, ld_y, dtype, dir   as harp_apply.
 */
HARP_API harp_status harp_apply_host(harp_plan_t plan, const void* x, void* y, int64_t rows,
                                     int64_t ld_x, int64_t ld_y, harp_dtype dtype, harp_dir dir);

/*
 * harp_apply_quant — the row transform with a fused blockwise quantizer on its output
 * (the rotated rows feed a blockwise quantizer: §2.4, a drop-in preprocessing step in
 * front of the quantizer backend).  For every row r and every aligned block of `qblock`
 * coordinates of y_r = T x_r (FORWARD) or T^T x_r (INVERSE), computed in fp32 as in
 * harp_apply:
 *   s = a / 127, a = max |y| over the block    (fp32, round to nearest; 0 for a zero block)
 *   q = clamp(round_half_even(y * (127 / a)), -127, 127)
 *                                              (int8; the reciprocal and the product rounded
 *                                               to nearest in fp32; 0 where a = 0)
 * so y is approximately q * s.  y itself is never written: one pass reads x and writes
 * the codes and scales.
 *   x        device bf16 rows, leading dimension ld_x >= d.
 *   q        device int8 codes, rows of d, leading dimension ld_q >= d.
 *   scales   device float, rows of d / qblock scales, leading dimension ld_s >= d / qblock.
 *   qblock   32, 64, 128 or 256, dividing d; else HARP_ERR_INVALID_ARG.
 * x, q and scales must not overlap.  Runs on the specialized d = 4096 (8,8,8,8) kernel for
 * that schedule, forward, from 32 rows up, else on the general tiled kernel: radices <= 8,
 * d % 8 == 0, x and q rows 16-byte aligned (ld_q a multiple of 16), scales 4-byte aligned;
 * otherwise HARP_ERR_UNSUPPORTED.  rows = 0 is a no-op.  Asynchronous on `stream`.
 */
HARP_API harp_status harp_apply_quant(harp_plan_t plan, const void* x, int64_t rows, int64_t ld_x,
                                      harp_dtype in_dtype, int8_t* q, int64_t ld_q, float* scales,
                                      int64_t ld_s, int32_t qblock, harp_dir dir, void* stream);

/*
 * harp_apply_columns — every column of an fp32 matrix takes T (FORWARD) or T^T
 * (INVERSE): for j < ncols, y[:, j] = T x[:, j] with x of d = plan dimension rows.  The
 * column side of a two-sided rotation, applied in place without a transpose (HARP
 * abstract: a rotation on each side of a weight matrix).
 *   x        device fp32 matrix, d rows of ncols, leading dimension ld_x >= ncols,
 *            16-byte aligned, ld_x a multiple of 4.  Overwritten (it holds an
 *            intermediate between the kernel's two passes).
 *   y        result, d rows of ncols, leading dimension ld_y (a multiple of 4 elements),
 *            16-byte aligned, element type out_dtype; y may equal x for HARP_F32.
 * Returns HARP_ERR_UNSUPPORTED for plans the column kernel does not take (a single
 * stage, a radix above 8, a schedule without a split whose tiles fit in shared memory)
 * and for unaligned arguments.
 */
HARP_API harp_status harp_apply_columns(harp_plan_t plan, float* x, int64_t ld_x, int64_t ncols,
                                        void* y, int64_t ld_y, harp_dtype out_dtype, harp_dir dir,
                                        void* stream);

/*
 * harp_two_sided_workspace_bytes — device workspace that harp_apply_two_sided
 * needs for an n_out x n_in weight (two fp32 copies of it, 256-byte aligned).
 */
HARP_API size_t harp_two_sided_workspace_bytes(int64_t n_out, int64_t n_in);

/*
 * harp_apply_two_sided — W_out = T_U^T W T_V (HARP abstract: a two-sided
 * processor; U acts on the output side, V on the input side of W).
 *   planU       plan with d = n_out (rotation of the columns of W).
 *   planV       plan with d = n_in (rotation of the rows of W).
 *   W, W_out    device pointers, n_out rows of n_in elements, leading dimension
 *               ld >= n_in, element type `dtype`.  W_out may equal W.
 *   workspace   device memory of at least harp_two_sided_workspace_bytes(),
 *               256-byte aligned; intermediates are kept in fp32 there.
 * Rows of W take T_V^T, columns take T_U^T; the result is rounded once, at the end.
 * The original weight is W = T_U W_out T_V^T.
 */
HARP_API harp_status harp_apply_two_sided(harp_plan_t planU, harp_plan_t planV, const void* W,
                                 void* W_out, int64_t n_out, int64_t n_in, int64_t ld,
                                 harp_dtype dtype, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * harp_apply_two_sided_noalloc — the same W_out = T_U^T W T_V as
 * harp_apply_two_sided, for callers that cannot allocate device memory when they
 * rotate a weight (code that runs inside a memory pool or arena it does not own,
 * inside a capture region, or in a host runtime that exposes no allocator to
 * plugins).  It needs no workspace argument: the two fp32 intermediates live in a
 * fixed array of HARP_NOALLOC_SCRATCH_BYTES inside the library's device image,
 * which every GPU that loads the library holds until the process exits.  The
 * paper has no counterpart of this entry point; it exists for such callers only.
 *   Limit: n_out * n_in <= HARP_NOALLOC_SCRATCH_BYTES / 8 elements (4,194,304),
 *          else HARP_ERR_INVALID_ARG and nothing is launched.
 *   First call on a device: looks up the array's device address
 *          (cudaGetSymbolAddress) with that device current and keeps it for the
 *          life of the process; make that first call before any stream capture.  The
 *          kept address does not survive cudaDeviceReset: do not call this entry point
 *          again after resetting the device in the same process.
 *   Sides: each row pass holds one fp32 row in shared memory, so max(n_out, n_in) * 4
 *          bytes must fit the device's opt-in shared memory per block (227 KiB on
 *          B200), else HARP_ERR_UNSUPPORTED before anything is launched.
 *   Sharing: all calls use the same array; calls whose work overlaps on the GPU
 *          (different streams or host threads) race on it and must be serialized
 *          by the caller.  No part of the array needs to start at zero.
 *   It calls no cudaMalloc, cudaFree or other allocating routine.  Other arguments
 *   and errors are those of harp_apply_two_sided.
 */
#define HARP_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
HARP_API harp_status harp_apply_two_sided_noalloc(harp_plan_t planU, harp_plan_t planV,
                                                  const void* W, void* W_out, int64_t n_out,
                                                  int64_t n_in, int64_t ld, harp_dtype dtype,
                                                  void* stream);

/* harp_noalloc_scratch_bytes — size of that static array (HARP_NOALLOC_SCRATCH_BYTES). */
HARP_API size_t harp_noalloc_scratch_bytes(void);

/*
 * harp_grad_workspace_bytes — device workspace that harp_grad_theta needs for this plan:
 * one float accumulator per block entry (4 d sum_t b_t bytes, each stage padded to 16
 * bytes).  0 for a NULL plan.
 */
HARP_API size_t harp_grad_workspace_bytes(harp_plan_t plan);

/*
 * harp_grad_theta — calibration backward (§2.3 Optimization Objective: theta is fitted
 * per layer from calibration data): dtheta = dL/dtheta for L = sum_r g_r . (T x_r), i.e.
 * the gradient of a loss through the forward transform given the upstream gradients
 * g_r = dL/dy_r.  (dL/dx_r = T^T g_r is harp_apply with HARP_INVERSE.)
 *   x, g        device pointers, rows of d elements of type dtype (both the same type),
 *               leading dimensions ld_x, ld_g >= d.
 *   rows        number of rows; 0 writes dtheta = 0.
 *   dtheta      device float array of the plan's theta count, overwritten, in the theta
 *               layout of harp_plan_create (stages in order, blocks in c order, the
 *               block's parameters contiguous).  For int8 plans it is the gradient with
 *               respect to the dequantized values q * scale_t.
 *   workspace   device memory of at least harp_grad_workspace_bytes(plan) bytes,
 *               16-byte aligned; overwritten.
 * Arithmetic: fp32 in the stage chain and the per-tile sums, fp32 atomic additions across
 * tiles (the order of those additions varies between runs, so the last bits of dtheta
 * may too), double in the map from block gradients to theta.
 * Returns HARP_ERR_UNSUPPORTED for radices above 8 and for rows too long for two fp32 rows
 * in shared memory (d above 29,056); asynchronous on `stream` like harp_apply.
 */
HARP_API harp_status harp_grad_theta(harp_plan_t plan, const void* x, const void* g, int64_t rows,
                                     int64_t ld_x, int64_t ld_g, harp_dtype dtype, float* dtheta,
                                     void* workspace, size_t ws_bytes, void* stream);

/*
 * harp_off_block_energy — the block-diagonality term of the fit (§2.3 Optimization
 * Objective: R_bd(Theta_V), the Hessian energy that falls outside the quantizer's blocks
 * after the input-side rotation).  For a square matrix h of n x n (normally the rotated
 * Hessian proxy H' = T_V^T H T_V, which is harp_apply_two_sided(planV, planV, H)):
 *   out[0] = sum of h_ij^2 over i / q != j / q     (outside the q x q diagonal blocks)
 *   out[1] = sum of all h_ij^2
 * so R_bd = out[0] / out[1].  Squares and sums in double (fp32 and bf16 squares are exact
 * there); the CTAs' partial sums are added with double atomics, so the last bits vary
 * between runs.
 *   h        device matrix, element type dtype, leading dimension ld >= n.
 *   q        block size, q > 0 dividing n.
 *   out      device array of 2 doubles, overwritten (zeroed on `stream` first); must not
 *            overlap h.
 * Asynchronous on `stream`; HARP_ERR_INVALID_ARG for bad sizes or NULL pointers.
 */
HARP_API harp_status harp_off_block_energy(const void* h, int64_t n, int64_t ld, harp_dtype dtype, int32_t q,
                                           double* out, void* stream);

/*
 * harp_l_diag — the diagonal-weighted quantization error of the fit (§2.3 Optimization
 * Objective: L_diag, the quantizer's error on the rotated weight weighted by the rotated
 * Hessian's diagonal):
 *   out[0] = sum_j h_jj sum_r (w_rj - Q(w)_rj)^2
 * with Q the blockwise round-to-nearest int8 quantizer along the rows of w (per aligned
 * block of qblock columns: s = max|w| / 127, code = clamp(round_half_even(w / s), -127,
 * 127), Q(w) = code * s; a zero block is exact).  The quantizer's arithmetic is double
 * (the same operations as its float64 definition, so its codes match that definition's
 * for the same w); the sums are double with atomic adds across CTAs.
 *   w        device rotated weight W' = T_U^T W T_V (harp_apply_two_sided), rows x cols,
 *            element type dtype, leading dimension ld_w >= cols.
 *   h        device float rotated Hessian proxy H' (cols x cols, leading dimension ld_h >=
 *            cols); only its diagonal is read.
 *   qblock   32, 64, 128 or 256, dividing cols.
 *   out      device double, overwritten (zeroed on `stream` first); must not overlap w or h.
 * rows = 0 writes 0.  Asynchronous on `stream`.
 */
HARP_API harp_status harp_l_diag(const void* w, int64_t rows, int64_t cols, int64_t ld_w, harp_dtype dtype,
                                 const float* h, int64_t ld_h, int32_t qblock, double* out, void* stream);

/*
 * harp_moment_check — the check that picks how many composed passes a batch needs (the
 * RHT-composition results quoted with the HARP pages propose a linear-time check on the
 * input's moments that adapts the number of randomized Hadamard passes at run time, without
 * giving the statistic or its thresholds).  Per row r of x:
 *   moments[3r .. 3r+2] = (sum x^2, sum |x|^3, sum x^4)          (double)
 *   passes[r] = 1 if kappa <= tau1, 2 if kappa <= tau2, else 3,   kappa = m4 / m2^2
 * kappa is 1/d for a flat row and 1 for a one-hot row (0 for a zero row, which takes 1 pass);
 * the Berry-Esseen ratio m3 / m2^1.5 follows from the moments.  Compose that many plans
 * (harp_plan_compose) for the batch.
 *   x         device rows, element type dtype, leading dimension ld >= d.
 *   moments   device double array of 3 rows entries, or NULL.
 *   passes    device int32 array of rows entries, or NULL (not both NULL).
 * tau1 <= tau2, else HARP_ERR_INVALID_ARG; the outputs must not overlap x or each other.
 * rows = 0 is a no-op.  Asynchronous on `stream`.
 */
HARP_API harp_status harp_moment_check(const void* x, int64_t rows, int64_t d, int64_t ld, harp_dtype dtype,
                                       double tau1, double tau2, double* moments, int32_t* passes, void* stream);

/*
 * harp_plan_compose — one plan for the composition T = T_{k-1} ... T_1 T_0 of k plans of
 * the same dimension (plans[0] acts first): k independent rotations in one pass over the
 * rows (composing two or three randomized Hadamard transforms brings every input's
 * coordinates close to the behaviour of a uniform random rotation, the RHT-composition
 * results the HARP pages quote).  The composite copies the plans' device blocks (the
 * plans may be destroyed afterwards) and is materialized on the current device; every
 * plan must be materialized there, and the stages must number at most HARP_MAX_STAGES in
 * all (HARP_ERR_SCHEDULE otherwise).  The composite works with harp_apply, harp_apply_ex,
 * harp_apply_host, harp_apply_quant (INVERSE gives T^T = T_0^T ... T_{k-1}^T) and as a side
 * of harp_apply_two_sided; harp_apply_columns, harp_grad_theta, harp_plan_signs and
 * harp_plan_base_mixer return HARP_ERR_UNSUPPORTED for it.  Destroy with
 * harp_plan_destroy.  The copies run on `stream` and the call returns when they are done
 * (not allowed inside a stream capture).
 */
HARP_API harp_status harp_plan_compose(harp_plan_t* out, const harp_plan_t* plans, int32_t k, void* stream);

/* harp_plan_device_status — synchronizes the plan's device and reports whether any
 * bounded device-side wait of a kernel launched with this plan gave up since the
 * last call: HARP_ERR_TIMEOUT if one did (the flag is then cleared), HARP_OK if
 * not, HARP_ERR_NOT_MATERIALIZED before materialization. */
HARP_API harp_status harp_plan_device_status(harp_plan_t plan);

/* harp_plan_destroy — free the plan and its device memory (synchronizes the
 * device that owns it).  NULL is accepted. */
HARP_API harp_status harp_plan_destroy(harp_plan_t plan);

/* harp_status_string — static, human-readable name of a status code. */
HARP_API const char* harp_status_string(harp_status s);

/* harp_last_kernel — name of the last kernel this host thread launched through
 * harp_apply / harp_apply_two_sided (static per-thread buffer). */
HARP_API const char* harp_last_kernel(void);

/* harp_last_error — detail of the last failing call on this host thread (static
 * per-thread buffer, valid until the next call). */
HARP_API const char* harp_last_error(void);

/*
 * harp_test_inject_wait_timeout — test hook for the bounded device waits (the paper has no
 * counterpart).  Until it is called again with (0, 0), every general tiled-kernel launch
 * from this host thread tells its row-staging barriers to expect `extra_bytes` more than it
 * copies and polls them only `poll_limit` times, so the first wait of each staged tile runs
 * out: the kernel then sets the plan's status word (harp_plan_device_status reports
 * HARP_ERR_TIMEOUT), retires the extra bytes itself, waits (bounded as usual) for the copies
 * it really issued, and finishes with correct output.  No copy is left in flight and no
 * wait is unbounded.  poll_limit >= 1 and 1 <= extra_bytes <= 4096, or both 0 to clear;
 * else HARP_ERR_INVALID_ARG.
 */
HARP_API harp_status harp_test_inject_wait_timeout(int64_t poll_limit, uint32_t extra_bytes);

/* ------------------------------------------------------------------------- */
/* Host-side introspection: no device work, usable without a GPU.            */
/* ------------------------------------------------------------------------- */

/* Number of parameters of a schedule: sum_t (d/b_t) p_t; -1 if the schedule is
 * invalid. */
HARP_API int64_t harp_theta_count(const int32_t* radices, int32_t m);

/* The first n outputs of SplitMix64 started at `seed` (host array out[n]). */
HARP_API harp_status harp_splitmix64(uint64_t seed, int64_t n, uint64_t* out);

/* The plan's base mixer G_radix in double, row-major, into host out[radix*radix];
 * HARP_ERR_INVALID_ARG if no stage of the plan uses that radix. */
HARP_API harp_status harp_plan_base_mixer(harp_plan_t plan, int32_t radix, double* out);

/* The plan's sign diagonal as +1/-1 into host out[d]. */
HARP_API harp_status harp_plan_signs(harp_plan_t plan, int8_t* out);

/* Dimension, stage count and radices of a plan (radices: host out[HARP_MAX_STAGES]). */
HARP_API harp_status harp_plan_shape(harp_plan_t plan, int64_t* d, int32_t* m, int32_t* radices);

#ifdef __cplusplus
}
#endif

#endif /* HARP_H_ */
