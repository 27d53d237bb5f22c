/*
 * fp8train.h — C ABI of the B200 (sm_100a) FP8 delayed-scaling Linear step and fused AdamW.
 *
 * One Linear layer's training step, HYBRID recipe, per-tensor delayed scaling:
 *
 *   cast X, W (E4M3) and dY (E5M2)      fp8_cast_transpose_amax   (x3)
 *   Y  = X  . W        (fprop)          fp8_gemm
 *   dX = dY . W^T      (dgrad)          fp8_gemm
 *   dW = X^T . dY      (wgrad)          fp8_gemm
 *   amax history roll + next scales     fp8_scale_update
 *   unscale, clip, AdamW, BF16 weight   fused_adamw_multi_tensor
 *
 * and the same step in three launches:
 *
 *   casts of X and dY + the scale update of X, W, dY    fp8_cast_transpose_amax_update_multi
 *   fprop, dgrad, wgrad (+ sum of dW^2)                 fp8_gemm_multi_sumsq
 *   AdamW on that sum + cast of the next step's W       fused_adamw_multi_tensor_presummed
 *
 * plus current scaling (fp8_cast_transpose_amax_current_multi) and MXFP8 block scaling
 * (fp8_mx_cast_multi, fp8_mx_gemm_multi).
 *
 * Sources, cited by page title and section:
 *   [P1] "算子与编译器：FP8 训练与优化器 Kernel" (charles2530.github.io)
 *   [P2] "FP8 混合精度训练工程实践：从 H100 到大模型训练的范式跃迁" (ybb.press)
 *   [P3] "LLM FP8 微调上线生产实战：用 Amax Scaling、层级白名单与 BF16 回退守住收敛" (oh-bug.com)
 *
 * Conventions shared by every entry point
 *   - Every pointer argument whose name starts with d_, and every tensor argument, is DEVICE
 *     memory on the current CUDA device, owned by the caller. The library allocates no device
 *     memory and keeps no pointer after a call returns.
 *   - All matrices are row-major and contiguous. BF16 is stored as uint16 bit patterns, FP8 as
 *     one byte per element (E4M3: 1-4-3 bits, bias 7, max 448; E5M2: 1-5-2 bits, bias 15,
 *     max 57344 [P2 §一]).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream). Scalars that the GPU produces (scales, amax, norms) travel by
 *     device pointer, so a step never synchronises with the host.
 *   - Arguments are validated on the host before anything is launched. An invalid argument
 *     returns an error status and launches nothing. A launch failure returns FP8T_ERR_CUDA;
 *     fp8t_last_error_message() describes the last failure on the calling thread.
 *   - Waits inside kernels are bounded in time. When one expires the kernel records it in a
 *     device error word and returns early; fp8t_check_device_error() reports it. The word is
 *     for reporting only: what a fused call does about an expired wait (keep the scales, report
 *     a NaN sum of squares) depends on that call's own launches, never on the word, so a stale
 *     entry from an unrelated call changes nothing.
 */
#ifndef FP8TRAIN_H
#define FP8TRAIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp8t_status {
    FP8T_OK = 0,
    FP8T_ERR_INVALID_ARG = 1,       /* NULL pointer, non-positive size, unknown enum value     */
    FP8T_ERR_UNSUPPORTED_SHAPE = 2, /* a dimension is not a multiple of 16 (128 for MX) or too big */
    FP8T_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned                          */
    FP8T_ERR_UNSUPPORTED_DEVICE = 4,/* the current device is not sm_100                         */
    FP8T_ERR_CUDA = 5,              /* a CUDA runtime or driver call failed                      */
    FP8T_ERR_TIMEOUT = 6            /* a bounded wait inside a kernel expired                    */
} fp8t_status;

typedef enum fp8t_format {
    FP8T_E4M3 = 0, /* forward tensors X and W under HYBRID [P3 核心原理, E4M3 与 E5M2 承担不同职责] */
    FP8T_E5M2 = 1  /* the output gradient dY under HYBRID                                        */
} fp8t_format;

typedef enum fp8t_amax_algo {
    FP8T_AMAX_MAX = 0,         /* representative amax = largest entry of the history window  */
    FP8T_AMAX_MOST_RECENT = 1  /* representative amax = the newest entry                       */
} fp8t_amax_algo;             /* [P3 核心原理, Delayed Scaling 用历史换取稳定性, strategy table] */

/*
 * fp8_cast_transpose_amax — quantise one BF16 matrix to FP8 with a given per-tensor scale,
 * emit it row-major and transposed, and measure its amax.
 *
 * Defines: the saturating quantise q = sat(x * scale) of the FP8Tensor quantize step
 * [P2 §四, Delayed Scaling 核心逻辑], the amax = max|x| statistic it records [same], and the
 * zero-fraction / saturation / non-finite counts of [P3 工程落地, 第四步 metrics table].
 *
 *   x_bf16          rows x cols BF16, row-major (input).
 *   rows, cols      > 0, multiples of 16, rows*cols < 2^40.
 *   fmt             FP8T_E4M3 or FP8T_E5M2.
 *   d_scale         1 float: the scale to apply (delayed scaling: produced by the previous
 *                   fp8_scale_update). Read only.
 *   q_rowmajor      rows x cols FP8 bytes, row-major, or NULL to skip.
 *   q_transposed    cols x rows FP8 bytes (q^T, row-major), or NULL to skip.
 *   d_amax_inout    1 float, MAX-ACCUMULATED like the counters: it becomes the larger of its
 *                   previous content and max|x| over the BF16 input (NaN if any input is NaN),
 *                   compared as non-negative f32 bit patterns. Start it at 0; fp8_scale_update
 *                   resets each amax it consumes to 0, so a training step needs no memset.
 *   d_scale_inv_out 1 float, overwritten with 1/scale (IEEE division), or NULL to skip.
 *   d_counters      3 x uint64, or NULL: ADDED to [0] #saturated (|f32(x*scale)| > FP8 max),
 *                   [1] #zero codes (q is +0 or -0), [2] #non-finite inputs.
 *   Element rule:   q = encode_fmt(f32(x) * scale), one IEEE f32 multiply rounded to nearest,
 *                   then round-to-nearest-even to the format with saturation to +-max (an
 *                   infinite product saturates too); a NaN input gives the byte 0x7F.
 *   Pointers must be 16-byte aligned (except d_* scalars, 4- or 8-byte aligned).
 */
fp8t_status fp8_cast_transpose_amax(const void* x_bf16, int64_t rows, int64_t cols, fp8t_format fmt,
                                    const float* d_scale, void* q_rowmajor, void* q_transposed,
                                    float* d_amax_inout, float* d_scale_inv_out,
                                    unsigned long long* d_counters, void* stream);

/* One tensor of fp8_cast_transpose_amax_multi: the arguments of fp8_cast_transpose_amax. */
typedef struct fp8t_cast_tensor {
    const void* x_bf16;
    int64_t rows, cols;
    fp8t_format fmt;
    const float* d_scale;
    void* q_rowmajor;                  /* may be NULL */
    void* q_transposed;                /* may be NULL */
    float* d_amax_inout;
    float* d_scale_inv_out;            /* may be NULL */
    unsigned long long* d_counters;    /* may be NULL */
} fp8t_cast_tensor;

/*
 * fp8_cast_transpose_amax_multi — fp8_cast_transpose_amax for several tensors in one launch
 * (the X, W and dY casts of a step, for instance), with the same per-tensor semantics and
 * validation. Up to 8 tensors share a launch; longer lists are split into several launches.
 *   tensors     HOST array of n_tensors descriptors (read during the call only).
 *   n_tensors   1 .. 4096.
 */
fp8t_status fp8_cast_transpose_amax_multi(const fp8t_cast_tensor* tensors, int32_t n_tensors,
                                          void* stream);

/*
 * fp8_cast_transpose_amax_current_multi — current ("just-in-time") scaling: each tensor's scale
 * is derived from its own amax before it is cast, instead of from the history of earlier steps
 * [P2 §四 FP8Tensor.quantize measures amax = max|x| of the tensor it quantises; P3 核心原理 gives
 * scale = (FP8_MAX / amax) / 2^margin]. Per group of up to 8 tensors one amax launch reads the
 * tensors, and its last CTA writes scale = (FP8_MAX / amax) * 2^-margin IN PLACE into
 * tensors[i].d_scale (amax 0 gives 1; a NaN or infinite amax keeps the previous scale; an
 * overflow gives FLT_MAX; FP8_MAX 448 for E4M3, 57344 for E5M2); then the cast of
 * fp8_cast_transpose_amax_multi runs with that scale, with all its outputs (the amax slot
 * max-accumulates as usual).
 *   margin        0 .. 126.
 *   d_workspace   FP8T_CURRENT_WORKSPACE_BYTES of device memory, 4-byte aligned, ZERO-FILLED
 *                 before its first use and left zero by every call; concurrent calls need
 *                 their own.
 * Traffic: 2 B/element more than the delayed cast (the amax read).
 */
#define FP8T_CURRENT_WORKSPACE_BYTES 64
fp8t_status fp8_cast_transpose_amax_current_multi(const fp8t_cast_tensor* tensors,
                                                  int32_t n_tensors, int32_t margin,
                                                  unsigned int* d_workspace, void* stream);

/* The scale state fp8_cast_transpose_amax_update_multi updates for one tensor. */
typedef struct fp8t_cast_update {
    float* d_amax_history;     /* history_len floats of this tensor, entry 0 newest (in/out) */
    float* d_scale_inv_next;   /* 1 float: receives 1 / next scale; must not be the cast's
                                  d_scale_inv_out, which keeps 1 / the scale the cast used */
} fp8t_cast_update;

/*
 * fp8_cast_transpose_amax_update_multi — the casts of fp8_cast_transpose_amax_multi followed,
 * inside the same launch, by the delayed-scaling update of fp8_scale_update for the same
 * tensors [P3 核心原理, Delayed Scaling: the scale for the next iteration comes from the amax
 * history; the scale kernel is one of the extra launches 实践建议 warns about]. The CTA that
 * finishes last rolls each tensor's history (amax pushed at entry 0), picks the representative
 * amax (algo), writes the next scale IN PLACE into tensors[i].d_scale (declared const there
 * because the cast only reads it; this call overwrites it after every read of it is done),
 * writes 1/next scale to updates[i].d_scale_inv_next and resets tensors[i].d_amax_inout to 0.
 * FP8 max is 448 for E4M3 tensors and 57344 for E5M2 ones. The result is bit-identical to
 * fp8_cast_transpose_amax_multi then fp8_scale_update with the same arguments.
 *   updates       HOST array of n_tensors entries.
 *   history_len   1 .. 65536 (the same for every tensor of the call).
 *   algo, margin  as in fp8_scale_update.
 *   d_ticket      1 device uint32, zero before the first call; each launch leaves it zero.
 *                 Calls that may run at the same time (other streams) need their own tickets.
 * An entry with x_bf16 = NULL, rows = cols = 0 and no outputs or counters is UPDATE ONLY: its
 * amax slot was filled by another call (the weight cast inside
 * fused_adamw_multi_tensor_presummed of the previous step) and only the update runs for it.
 * If a bounded wait of this launch expires (FP8T_ERR_TIMEOUT pending in the device error word),
 * the scale state is left unchanged; the CTAs report it to the last one through the ticket. Argument errors as in the two calls it combines, plus
 * FP8T_ERR_INVALID_ARG for a NULL or shared scale-inverse pointer.
 */
fp8t_status fp8_cast_transpose_amax_update_multi(const fp8t_cast_tensor* tensors,
                                                 const fp8t_cast_update* updates, int32_t n_tensors,
                                                 int32_t history_len, fp8t_amax_algo algo,
                                                 int32_t margin, unsigned int* d_ticket,
                                                 void* stream);

/*
 * fp8_gemm — per-tensor scaled FP8 GEMM, FP32 accumulation, BF16 output, "TN" layout:
 *
 *   D[i][j] = bf16_rn( (sum_k A[i][k] * B[j][k]) * (a_scale_inv * b_scale_inv) )
 *
 * Defines: the FP8 GEMM of the recipe table with an FP32 accumulator and a 16-bit output
 * [P2 §三, 标准 FP8 Training Recipe], dequantised by the per-tensor scales [P2 §四, dequantize;
 * P2 §五, per-tensor mode of the FP8 GEMM table: FP8 x FP8, FP32 accumulate, BF16 out].
 * The three GEMMs of the step are all of this form (W stored in x out):
 *   fprop  Y  = X.W     : A = Xq   (T x in),   B = Wq^T  (out x in), M=T,  N=out, K=in
 *   dgrad  dX = dY.W^T  : A = dYq  (T x out),  B = Wq    (in x out), M=T,  N=in,  K=out
 *   wgrad  dW = X^T.dY  : A = Xq^T (in x T),   B = dYq^T (out x T),  M=in, N=out, K=T
 *
 *   A               M x K FP8 bytes, row-major (K contiguous), format a_fmt.
 *   B               N x K FP8 bytes, row-major (K contiguous), format b_fmt.
 *   M, N, K         > 0, multiples of 16, each < 2^31.
 *   d_a_scale_inv, d_b_scale_inv   1 float each (device); their f32 product scales the sum.
 *   D_bf16          M x N BF16, row-major (output, overwritten).
 *   A, B, D must be 16-byte aligned. The accumulation order over k is unspecified; the result is
 *   within 2 BF16 ulp + 1e-5 * sum_k |A[i][k] B[j][k]| * scale of the exact value.
 */
fp8t_status fp8_gemm(const void* A, fp8t_format a_fmt, const void* B, fp8t_format b_fmt,
                     int64_t M, int64_t N, int64_t K,
                     const float* d_a_scale_inv, const float* d_b_scale_inv,
                     void* D_bf16, void* stream);

/* How an operand of fp8_gemm_multi is stored. The 5th-generation tensor cores read 8-bit
 * operands in either order, so no transposed copy is needed for the wgrad or fprop operands. */
typedef enum fp8t_layout {
    FP8T_K_MAJOR = 0,   /* A stored M x K row-major (B: N x K), the layout of fp8_gemm        */
    FP8T_MN_MAJOR = 1   /* A stored K x M row-major (B: K x N): e.g. Xq itself for wgrad     */
} fp8t_layout;

/* One GEMM of fp8_gemm_multi: the arguments of fp8_gemm plus the operands' layouts (zero =
 * K-major, so a descriptor filled like fp8_gemm's arguments computes the same product). */
typedef struct fp8t_gemm_desc {
    const void* A;
    fp8t_format a_fmt;
    const void* B;
    fp8t_format b_fmt;
    int64_t M, N, K;
    const float* d_a_scale_inv;
    const float* d_b_scale_inv;
    void* D_bf16;
    fp8t_layout a_layout;
    fp8t_layout b_layout;
} fp8t_gemm_desc;

/*
 * fp8_gemm_multi — several independent fp8_gemm problems in one persistent launch (the fprop,
 * dgrad and wgrad of a step, or those of several layers), same per-problem semantics and
 * validation. One launch holds up to 24 problems; tiles are taken problem by problem, so the
 * whole group shares one tile schedule (no gap between problems, balanced last wave).
 *   gemms     HOST array of n_gemms descriptors (read during the call only).
 *   n_gemms   1 .. 4096.
 */
fp8t_status fp8_gemm_multi(const fp8t_gemm_desc* gemms, int32_t n_gemms, void* stream);

/*
 * fp8_gemm_multi_sumsq — fp8_gemm_multi that also returns, for the problems selected by
 * sumsq_of, S = sum over their D elements of f32(D)^2, accumulated in FP64: the gradient
 * sum of squares the AdamW global-norm clip needs [P1 FP8 训练主路径图 (unscale and clip before
 * the optimizer); P1 Fused Optimizer 的意义 (read the gradient once)], formed while the wgrad
 * output is still on chip. The summation order is fixed (per-warp partials in a workspace, then
 * one pass in index order), so S is the same on every run; it may differ from a sequential
 * FP64 sum in the last bits.
 *   sumsq_of        HOST array of n_gemms int32: nonzero = include this problem's D.
 *   d_sumsq_out     1 double (device), overwritten; NaN if a bounded wait of this call expired.
 *   d_workspace     device scratch of fp8_gemm_sumsq_workspace_bytes() bytes, 256-byte aligned,
 *                   ZERO-FILLED before its first use (it holds a ticket counter and the call's
 *                   abort word, which every call leaves at zero). Calls that may run at the
 *                   same time need their own.
 * Errors as in fp8_gemm_multi, plus FP8T_ERR_INVALID_ARG for NULL/misaligned S or workspace,
 * no selected problem, or a workspace that is too small.
 */
fp8t_status fp8_gemm_multi_sumsq(const fp8t_gemm_desc* gemms, int32_t n_gemms,
                                 const int32_t* sumsq_of, double* d_sumsq_out, void* d_workspace,
                                 size_t workspace_bytes, void* stream);

/* Scratch bytes fp8_gemm_multi_sumsq needs (0 on invalid input or no selected problem). */
size_t fp8_gemm_sumsq_workspace_bytes(const fp8t_gemm_desc* gemms, int32_t n_gemms,
                                      const int32_t* sumsq_of);

/*
 * MXFP8 block scaling [P2 §九, Blackwell microscaling: 32 values share one 8-bit E8M0 scale,
 * each stored as FP8; P2 §三: micro scaling with E4M3 elements]. For every block of 32 values
 * the shared exponent is X = floor(log2(amax)) - emax, emax = 8 for E4M3 (448 = 1.75 * 2^8)
 * and 15 for E5M2, clamped to [-127, 127] (amax 0: -127; infinite amax: 127); the scale code is
 * X + 127 (0xFF if the block holds a NaN, whose elements are then encoded at unit scale), and
 * every element is q = encode_fmt(f32(x) * 2^-X) with the rounding and saturation of
 * fp8_cast_transpose_amax.
 *
 * Scale layout ("atoms"): for an operand with MN rows (M for A, N for B) and K columns of the
 * contraction, the scales are stored as [MN/128][K/128] atoms of 512 bytes; inside an atom,
 * byte (i % 32) * 16 + (i / 32) * 4 + kb holds the scale of row i (0..127) and K-block kb
 * (0..3, 32 values each). This is the order in which the tensor cores' scale copy reads them.
 */
typedef struct fp8t_mx_cast_tensor {
    const void* x_bf16;      /* rows x cols BF16, row-major; rows, cols multiples of 128     */
    int64_t rows, cols;
    fp8t_format fmt;
    void* q_row;             /* rows x cols codes, blocks along each row (K = cols), or NULL  */
    void* scales_row;        /* atoms [rows/128][cols/128] (MN = rows, K = cols)              */
    void* q_col;             /* rows x cols codes, blocks down each column (K = rows), or NULL */
    void* scales_col;        /* atoms [cols/128][rows/128] (MN = cols, K = rows)              */
} fp8t_mx_cast_tensor;

/*
 * fp8_mx_cast_multi — MX quantisation of several BF16 matrices, each into its row-wise copy
 * (the K-major GEMM operand: Xq for fprop, dYq for dgrad, W for dgrad's B) and/or its
 * column-wise copy (the MN-major operand: W for fprop's B, X and dY for wgrad), both in x's own
 * row-major layout with their scale atoms. At least one copy per tensor. Up to 8 tensors share
 * a launch. All pointers 16-byte aligned. Errors: INVALID_ARG, UNSUPPORTED_SHAPE (dimensions
 * not multiples of 128), MISALIGNED, CUDA.
 */
fp8t_status fp8_mx_cast_multi(const fp8t_mx_cast_tensor* tensors, int32_t n_tensors, void* stream);

/* One block-scaled GEMM of fp8_mx_gemm_multi: D = bf16(sum_k a_k b_k 2^(Xa + Xb)). */
typedef struct fp8t_mx_gemm_desc {
    const void* A;           /* M x K (K-major) or K x M (MN-major) codes                       */
    const void* A_scales;    /* atoms [M/128][K/128]                                            */
    fp8t_format a_fmt;
    fp8t_layout a_layout;
    const void* B;           /* N x K (K-major) or K x N (MN-major) codes                       */
    const void* B_scales;    /* atoms [N/128][K/128]                                            */
    fp8t_format b_fmt;
    fp8t_layout b_layout;
    int64_t M, N, K;         /* positive multiples of 128                                       */
    void* D_bf16;            /* M x N BF16, row-major                                           */
} fp8t_mx_gemm_desc;

/*
 * fp8_mx_gemm_multi — several MXFP8 GEMMs in one persistent launch on the block-scaled tensor
 * cores (FP32 accumulation, BF16 output, no per-tensor scale). HOST array of n_gemms (1..4096)
 * descriptors. Errors as fp8_gemm_multi; dimensions must be multiples of 128. The call runs
 * 256 x 384 output tiles when every N is at least 512, else 256 x 256 tiles; the results do not
 * depend on the choice.
 */
fp8t_status fp8_mx_gemm_multi(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms, void* stream);

/*
 * fp8_mx_gemm_multi_sumsq — fp8_mx_gemm_multi that also leaves in *d_sumsq_out the FP64 sum of
 * f32(D)^2 over the problems whose sumsq_of entry is nonzero (the wgrad outputs of a step, so
 * AdamW's global norm needs no pass over the gradients [P1 Fused Optimizer 的意义; 优化器 kernel
 * 的带宽账]), with the same fixed summation order, workspace rules, zero-on-entry / zero-on-exit
 * ticket words and NaN result on an expired wait as fp8_gemm_multi_sumsq.
 *   sumsq_of         HOST array of n_gemms int32 flags.
 *   d_sumsq_out      1 double (device), written by the launch that finishes the call.
 *   d_workspace      device scratch of fp8_mx_gemm_sumsq_workspace_bytes, 256-byte aligned,
 *                    zero-filled once before its first use (the call leaves it zero again).
 */
fp8t_status fp8_mx_gemm_multi_sumsq(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms,
                                    const int32_t* sumsq_of, double* d_sumsq_out,
                                    void* d_workspace, size_t workspace_bytes, void* stream);

/* Scratch bytes fp8_mx_gemm_multi_sumsq needs (0 on invalid input or no problem selected). */
size_t fp8_mx_gemm_sumsq_workspace_bytes(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms,
                                         const int32_t* sumsq_of);

/*
 * fp8_scale_update — roll each tensor's amax history and compute the next scale
 * [P3 核心原理, Scale 决定数值是否进入可表示区间 (scale = (FP8_MAX / amax) / 2^margin) and
 *  Delayed Scaling 用历史换取稳定性 (history window; max / most_recent; used next iteration)].
 *
 * For each tensor t in [0, n_tensors):
 *   history row t is shifted by one (entry H-1 is dropped) and entry 0 becomes d_amax[t],
 *   after which d_amax[t] is reset to 0 (ready for the next step's max-accumulating casts);
 *   rep   = max over the row of |h| (NaN if any entry is NaN)   for FP8T_AMAX_MAX,
 *           |h[0]|                                              for FP8T_AMAX_MOST_RECENT;
 *   scale = (d_fp8_max[t] / rep) * 2^-margin   (IEEE f32 division, then an exact power-of-two
 *           multiply; +inf becomes FLT_MAX)     if rep is finite and > 0,
 *           1.0                                 if rep == 0,
 *           unchanged                           if rep is NaN or inf;
 *   scale_inv = 1 / scale (IEEE f32 division).
 *
 *   n_tensors       1 .. 65535.
 *   d_amax          n floats (input; reset to 0 on return).
 *   d_amax_history  n x history_len floats, row-major, index 0 = newest (in/out).
 *   history_len     1 .. 65536.
 *   d_fp8_max       n floats: 448 for E4M3 tensors, 57344 for E5M2 tensors (input).
 *   margin          0 .. 126.
 *   d_scale, d_scale_inv   n floats each (in/out, out).
 */
fp8t_status fp8_scale_update(int32_t n_tensors, float* d_amax, float* d_amax_history,
                             int32_t history_len, const float* d_fp8_max, fp8t_amax_algo algo,
                             int32_t margin, float* d_scale, float* d_scale_inv, void* stream);

/* One parameter tensor of the multi-tensor AdamW: device pointers, 16-byte aligned. */
typedef struct fp8t_adamw_tensor {
    float* master;          /* FP32 master weight, numel (in/out)                 */
    float* m;               /* FP32 first moment, numel (in/out)                  */
    float* v;               /* FP32 second moment, numel (in/out)                 */
    const void* grad_bf16;  /* BF16 gradient of the loss-scaled loss, numel (in)  */
    void* weight_bf16;      /* BF16 copy of the updated master, numel (out)       */
    int64_t numel;          /* > 0                                                */
} fp8t_adamw_tensor;

/*
 * fused_adamw_multi_tensor — one fused AdamW step over many tensors [P1 Fused Optimizer 的意义
 * (read grad, update first/second moments, bias correction, weight decay, parameter update in
 * one kernel); P1 FP8 训练主路径图 (unscale / clip before the optimizer); P2 §四, precision flow
 * (gradient un-scaling by the loss scale, FP32 AdamW)].
 *
 *   norm  = sqrt(sum over all tensors of f32(g)^2, accumulated in FP64) / loss_scale
 *   If norm is not finite nothing is updated and *d_skipped_out = 1; otherwise *d_skipped_out = 0,
 *   coef  = (max_grad_norm > 0 && norm > max_grad_norm) ? max_grad_norm / norm : 1
 *   and each element, in f32 with every operation rounded separately (no fused multiply-add):
 *     g = f32(grad) * (coef * (1/loss_scale))
 *     m = beta1*m + (1-beta1)*g ;  v = beta2*v + (1-beta2)*g*g
 *     p = p * (1 - lr*wd)                                           (decoupled weight decay)
 *     p = p - (lr / (1-beta1^step)) * (m / (sqrt(v) / sqrt(1-beta2^step) + eps))
 *     weight_bf16 = bf16_rne(p)
 *   where 1-beta1, 1-beta2, 1-lr*wd, lr/(1-beta1^step) and sqrt(1-beta2^step) are computed
 *   in double on the host and rounded once to f32.
 *
 *   tensors         HOST array of n_tensors descriptors (read during the call only).
 *   n_tensors       1 .. 1<<20.
 *   step            >= 1 (bias-correction step count); used when d_step_inout is NULL.
 *   d_step_inout    1 int64 in device memory holding the number of completed steps, or NULL.
 *                   When given, `step` is ignored: the call performs step counter+1 and stores
 *                   that back into the counter unless the update is skipped, so a CUDA graph that
 *                   captured the call advances the optimizer on every replay. lr/(1-beta1^t) and
 *                   sqrt(1-beta2^t) are then formed on the device, in double with the same
 *                   formulas (a one-ulp difference from host-formed ones is possible).
 *   loss_scale      > 0 and finite.  max_grad_norm <= 0 disables clipping.
 *   d_grad_norm_out 1 float (device) or NULL: the unscaled global norm.
 *   d_skipped_out   1 int32 (device) or NULL.
 *   d_workspace     device scratch of at least fused_adamw_workspace_bytes() bytes, 16-byte
 *                   aligned; its contents on entry are ignored.
 */
fp8t_status fused_adamw_multi_tensor(const fp8t_adamw_tensor* tensors, int32_t n_tensors,
                                     float lr, float beta1, float beta2, float eps,
                                     float weight_decay, int64_t step, int64_t* d_step_inout,
                                     float loss_scale, float max_grad_norm,
                                     float* d_grad_norm_out, int32_t* d_skipped_out,
                                     void* d_workspace, size_t workspace_bytes, void* stream);

/* Scratch bytes fused_adamw_multi_tensor needs for these tensors (0 on invalid input). */
size_t fused_adamw_workspace_bytes(const fp8t_adamw_tensor* tensors, int32_t n_tensors);

/*
 * The FP8 cast of a tensor's NEW BF16 weight, done by the AdamW update that produces it: the
 * cast of fp8_cast_transpose_amax applied to weight_bf16 viewed as rows x cols (row-major),
 * with the same element rule, row-major codes and amax accumulation (no transposed copy: the
 * GEMMs read the weight codes MN-major where they need the transpose). Under delayed scaling
 * the scale for the next step's weight cast is known once the scale update of the current step
 * has run, so the next step need not read the weight again [P1 优化器 kernel 的带宽账: every
 * extra kernel re-reads the parameters; P3 核心原理: delayed scaling uses the previous scale].
 * rows = cols = 0 means no cast for this tensor.
 */
typedef struct fp8t_adamw_cast {
    int64_t rows, cols;             /* rows*cols == numel, multiples of 16 (or both 0)        */
    fp8t_format fmt;
    const float* d_scale;           /* 1 float: the scale of the next step's weight cast       */
    void* q_rowmajor;               /* rows x cols FP8 bytes, or NULL                          */
    float* d_amax_inout;            /* max-accumulated with max|new weight|                    */
    float* d_scale_inv_out;         /* 1/scale, or NULL                                        */
} fp8t_adamw_cast;

/*
 * fused_adamw_multi_tensor_presummed — fused_adamw_multi_tensor without its norm pass: the sum
 * of f32(g)^2 over all gradients is read from *d_grad_sumsq (for example from
 * fp8_gemm_multi_sumsq over the wgrad problems that produced them), so each gradient is read
 * once, by the update itself [P1 Fused Optimizer 的意义; 优化器 kernel 的带宽账]. Everything else,
 * including the skip on a non-finite norm, is as in fused_adamw_multi_tensor.
 *   casts           NULL, or a HOST array of n_tensors fp8t_adamw_cast: the tensors with
 *                   rows > 0 also get their new weight cast. On a skipped step their weight is
 *                   left unchanged and cast again with the given scale, so codes, amax and
 *                   scale inverse always describe the weight the next step uses.
 *   d_grad_sumsq    1 double (device), read.
 *   d_ticket        1 device uint32, zero before the first call and left zero; needed when
 *                   d_step_inout is given (the counter is advanced by the CTA that finishes
 *                   last), may be NULL otherwise. Concurrent calls need their own.
 */
fp8t_status fused_adamw_multi_tensor_presummed(const fp8t_adamw_tensor* tensors,
                                               const fp8t_adamw_cast* casts, int32_t n_tensors,
                                               float lr, float beta1, float beta2, float eps,
                                               float weight_decay, int64_t step,
                                               int64_t* d_step_inout, float loss_scale,
                                               float max_grad_norm, const double* d_grad_sumsq,
                                               float* d_grad_norm_out, int32_t* d_skipped_out,
                                               unsigned int* d_ticket, void* stream);

/* Size of the scratch array built into the library for fused_adamw_multi_tensor_noalloc. */
#define FP8T_NOALLOC_SCRATCH_BYTES 65536

/*
 * fused_adamw_multi_tensor_noalloc — the same AdamW step as fused_adamw_multi_tensor (same
 * arguments, same results), for callers that have no way to give the library scratch memory.
 * The pages have no counterpart to this entry point; it only changes where the scratch lives.
 *
 * Who needs it: a plugin or extension that receives the parameter, moment and gradient buffers
 * from a host framework but has no handle on that framework's device allocator, and code that
 * must not allocate once it is running because all device memory was reserved up front by a
 * pool. Neither can call cudaMalloc for the few kilobytes of per-block norm partials.
 *
 * Scratch: a file-scope device array of FP8T_NOALLOC_SCRATCH_BYTES (64 KiB) inside the library;
 * every GPU that loads the library keeps it until the process exits. It holds 8191 norm
 * partials and one step slot: any call with up to 3328 tensors fits, and larger calls fit when
 * their tensors are small. A call that needs more (fused_adamw_workspace_bytes() > FP8T_NOALLOC_SCRATCH_BYTES)
 * returns FP8T_ERR_UNSUPPORTED_SHAPE with a message and launches nothing.
 * Set-up: the first call on each device looks up the array's device address (with that device
 * current); make that first call before any stream capture on the device.
 * Sharing: every call uses the same array, which keeps the last call's contents. Each call
 * writes every slot it reads before reading it, so nothing has to be cleared, but two calls
 * whose kernels overlap on the GPU (different streams with no ordering between them) race on it.
 * It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
fp8t_status fused_adamw_multi_tensor_noalloc(const fp8t_adamw_tensor* tensors, int32_t n_tensors,
                                             float lr, float beta1, float beta2, float eps,
                                             float weight_decay, int64_t step,
                                             int64_t* d_step_inout, float loss_scale,
                                             float max_grad_norm, float* d_grad_norm_out,
                                             int32_t* d_skipped_out, void* stream);

/* Synchronise `stream`, then read and clear the device error word: FP8T_ERR_TIMEOUT if a bounded
 * wait in any kernel expired since the last check, FP8T_ERR_CUDA if the stream reports an error. */
fp8t_status fp8t_check_device_error(void* stream);

/* Override the time limit of the bounded waits in the GEMM (nanoseconds; 0 restores the default
 * of 2 s). Meant for tests of the timeout path; takes effect for launches after the call. */
fp8t_status fp8t_set_wait_timeout_ns(uint64_t ns);

/* Test hook for failure detection: mode 1 makes every bounded wait inside the cast and GEMM
 * kernels behave as if its barrier were never signalled, so each runs out its time limit and
 * the kernel takes its abort path (FP8T_ERR_TIMEOUT); mode 2 does this for the GEMM epilogue's
 * waits only, so loads and MMAs are in flight when the kernel drains them; 0 turns it off.
 * The drains of work already issued are never affected. Takes effect for later launches. */
fp8t_status fp8t_debug_expire_waits(int32_t mode);

/* Human-readable name of a status code; never NULL. */
const char* fp8t_status_string(fp8t_status status);

/* Message describing the last failure on the calling thread ("" if none). */
const char* fp8t_last_error_message(void);

/* ABI version of this header: 2 (fp8t_gemm_desc carries the operand layouts). */
int32_t fp8t_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8TRAIN_H */
