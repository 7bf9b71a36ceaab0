/*
 * zq.h -- C ABI of the B200 (sm_100a) ZeroQuant-style W8A8 linear library.
 *
 * The hot path of W8A8 post-training-quantized inference, as three fused
 * steps:
 *   1. LayerNorm (or bias + GeLU) fused with dynamic per-token symmetric
 *      INT8 quantization of the activations;
 *   2. an INT8 x INT8 -> INT32 GEMM against weights quantized in groups of
 *      contiguous output rows;
 *   3. a dequantization epilogue fused into the GEMM:
 *      y[t, o] = s_tok[t] * s_grp[o / G] * acc[t, o] + bias[o]
 *      (+ GeLU, + per-token requantization for the next layer).
 *
 * Sources (web pages):
 *   [ZQ]   "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
 *          Quantization for Large-Scale Transformers": group-wise weight
 *          quantization; token-wise activation quantization; the fused
 *          kernel flowcharts "LN/GeLU + Quantize" and "GEMM + DeQuantize".
 *   [TS36] "探秘Transformer系列之（36）— 大模型量化方案": §1.1.2 absmax
 *          quantization to [-127, 127] and vector-wise scales; §1.2.2
 *          per-token dynamic activation quantization fused with LayerNorm,
 *          INT32 accumulators scaled by both scales before the next op,
 *          group-wise weight quantization.
 *   [IQ]   "Integer Quantization: Deep Dive": quantization formula with
 *          clamp; dequantization x = s * x_int (zero-point 0 here).
 *
 * Numerics fixed by this library where the pages are silent:
 *   scale = absmax / 127 (fp32 IEEE division); code = clamp(rint(v * (127 /
 *   absmax)), -127, 127) with ties to even; an all-zero row or group has
 *   scale 0 and codes 0; LayerNorm uses the biased variance, eps inside the
 *   square root; GeLU is the erf form; bias is added after dequantization.
 *
 * Conventions for every entry point:
 *   - Matrices are dense row-major; the leading dimension equals the row
 *     length.  Activations are [T, K] (T tokens); weights are [N, K]
 *     (N output features, the nn.Linear layout).
 *   - Every pointer except where stated is a DEVICE pointer owned by the
 *     caller; the library keeps no reference after the call returns and
 *     allocates no device memory.  Scratch memory is passed in explicitly
 *     as (workspace, workspace_bytes).
 *   - Tensor pointers (x, q, Wq, W, y, workspace, gamma, beta) must be 16-byte
 *     aligned; scale and bias vectors 4-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL means the legacy default stream).  They return a zq_status.
 *     Arguments are validated on the host before anything is enqueued; a
 *     call that returns an error has launched nothing.  No call aborts,
 *     traps or prints.
 *   - Device-side waits inside the GEMM are bounded.  If one expires the
 *     kernel records the fact in a device flag and returns early (output
 *     undefined); zq_device_status() reports it as ZQ_ERR_TIMEOUT.
 *   - NaN or Inf inputs are outside the contract (not checked on device).
 *   - Hot-path kernels are launched with programmatic dependent launch:
 *     a kernel may start while the previous kernel on the stream finishes
 *     and waits (griddepcontrol.wait) before it reads activations or writes
 *     outputs.  The W8A8 linear starts streaming its weights (Wq, s_grp,
 *     bias) before that wait, so the weights must not be written by a kernel
 *     that lets its successors start early (none of this library's kernels
 *     does; zq_quantize_weights and zq_smooth_weights finish first).  Set
 *     ZQ_NO_PDL in the environment to launch every kernel in plain stream
 *     order.
 *   - The SmoothQuant entry points (zq_smooth_calibrate, zq_smooth_weights)
 *     cover [TS36] §1.3 and "SmoothQuant技术解析：大模型INT8量化的突破与实践";
 *     see their declarations.
 */
#ifndef ZQ_H_
#define ZQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
enum zq_status {
    ZQ_OK = 0,
    ZQ_ERR_NULL = 1,      /* a required pointer is NULL                         */
    ZQ_ERR_SHAPE = 2,     /* dimension <= 0, not a multiple of 16, N % G != 0,
                             or beyond a documented maximum                     */
    ZQ_ERR_ALIGN = 3,     /* pointer misaligned (see conventions)               */
    ZQ_ERR_OVERFLOW = 4,  /* K > ZQ_MAX_K: 127*127*K could leave int32          */
    ZQ_ERR_DTYPE = 5,     /* unknown dtype / activation / output-kind enum      */
    ZQ_ERR_CUDA = 6,      /* CUDA runtime/driver error; see zq_last_cuda_error  */
    ZQ_ERR_TIMEOUT = 7,   /* a bounded device-side wait expired                 */
    ZQ_ERR_WORKSPACE = 8, /* workspace NULL or smaller than required            */
    ZQ_ERR_DEVICE = 9,    /* current device is not sm_100 (B200 class)          */
    ZQ_ERR_SCRATCH = 10   /* problem larger than the fixed scratch array of
                             zq_w8a8_linear_requant_noalloc                      */
};

/* ---- enums --------------------------------------------------------------- */
enum zq_dtype { ZQ_F32 = 0, ZQ_BF16 = 1 };            /* activation input types */
enum zq_act { ZQ_ACT_NONE = 0, ZQ_ACT_GELU = 1 };     /* GeLU = erf form        */
enum zq_out_kind {
    ZQ_OUT_F32 = 0,        /* y fp32 [T, N]                                        */
    ZQ_OUT_BF16 = 1,       /* y bf16 [T, N], rounded to nearest even from fp32     */
    ZQ_OUT_I8_REQUANT = 2, /* y int8 [T, N] + s_tok_out fp32 [T]: the epilogue
                              output (after act) is quantized per token again      */
    ZQ_OUT_I32_RAW = 3     /* y int32 [T, N]: the raw accumulators (debug/parity)  */
};

/* 127*127*K must stay inside int32: K <= floor((2^31-1)/16129). */
#define ZQ_MAX_K 133144
/* Longest row the fused LayerNorm/act quantizer keeps on chip. */
#define ZQ_MAX_H 65536

/* ---- offline weight quantization ----------------------------------------
 * [ZQ] group-wise quantization; [TS36] §1.2.2 and §1.1.2 (absmax rule).
 * W     : fp32 [N, K] device, row-major.
 * group_rows (G) : rows per group; group g = rows g*G .. g*G+G-1, all K
 *         columns, one scale per group.  N % G == 0.  G = 1 gives per-row
 *         (vector-wise) scales, G = N a single per-tensor scale.
 * Wq    : int8 [N, K] device (output).
 * s_grp : fp32 [N / G] device (output): absmax_g / 127.
 * Constraints: K % 16 == 0.  Errors: NULL, SHAPE, ALIGN, CUDA, DEVICE. */
int zq_quantize_weights(const float* W, int64_t N, int64_t K, int64_t group_rows,
                        int8_t* Wq, float* s_grp, void* stream);

/* ---- fused LayerNorm + per-token quantization ----------------------------
 * [ZQ] "LN + Quantize" fused kernel; [TS36] §1.2.2 (quantization fused with
 * the preceding LayerNorm, one dynamic scale per token).
 * x      : [T, H] device, dtype x_dtype (ZQ_F32 or ZQ_BF16).
 * gamma, beta : fp32 [H] device.  eps : added to the variance.
 * q      : int8 [T, H] device (output); s_tok : fp32 [T] device (output).
 * y = (x - mean) / sqrt(var + eps) * gamma + beta per row (fp32), then
 * s_tok = absmax(y)/127, q = clamp(rint(y * 127/absmax(y))).
 * Constraints: H % 16 == 0, H <= ZQ_MAX_H.  Errors: NULL, SHAPE, ALIGN,
 * DTYPE, CUDA, DEVICE. */
int zq_ln_quant(const void* x, int x_dtype, int64_t T, int64_t H,
                const float* gamma, const float* beta, float eps,
                int8_t* q, float* s_tok, void* stream);

/* ---- fused (bias +) activation + per-token quantization ------------------
 * [ZQ] "GeLU + Quantize" fused kernel.  y = act(x + bias) per element in
 * fp32 (bias optional: NULL skips it; act ZQ_ACT_NONE or ZQ_ACT_GELU), then
 * the per-token quantizer of zq_ln_quant.  With no bias and no act the codes
 * and scales are exactly those of the quantizer applied to fp32(x).
 * Shapes, outputs, constraints and errors as zq_ln_quant. */
int zq_act_quant(const void* x, int x_dtype, int64_t T, int64_t H,
                 const float* bias, int act, int8_t* q, float* s_tok, void* stream);

/* ---- W8A8 linear: INT8 GEMM + fused dequantization epilogue --------------
 * [ZQ] "GEMM + DeQuantize"; [TS36] §1.2.2 (INT32 accumulators scaled by the
 * weight and activation scales before the write to the next op) and §1.1.2
 * (denormalisation by the outer product of row and column scales).
 * xq     : int8 [T, K] device;  s_tok : fp32 [T] device.
 * Wq     : int8 [N, K] device;  s_grp : fp32 [N / G] device.
 * bias   : fp32 [N] device or NULL.  act : applied after the bias.
 * out_kind selects y's type (see zq_out_kind).  s_tok_out : fp32 [T] device,
 *          written only for ZQ_OUT_I8_REQUANT (else may be NULL).
 * acc[t, o] = sum_k xq[t, k] * Wq[o, k] (exact int32, tcgen05 INT8 MMA);
 * y[t, o] = act(s_tok[t] * s_grp[o / G] * acc[t, o] + bias[o]) in fp32.
 * ZQ_OUT_I32_RAW stores acc itself and requires act == ZQ_ACT_NONE and
 * bias == NULL.
 * workspace : device scratch of zq_w8a8_linear_workspace(...) bytes (may
 *          be NULL when that is 0), 16-byte aligned when not NULL.  Its
 *          contents on entry do not matter; it is clobbered.
 *          ZQ_OUT_I8_REQUANT requires it: with T > 64 and at most one column
 *          tile of 256 per SM of the current device a word per token and per
 *          128-token block (the fused kernels), else the fp32 output plus a
 *          word per token.  For the other kinds it is optional: with
 *          T <= 64 and at least as many 128-row weight tiles as SMs, the
 *          query returns the size of the int32 partial sums (a 128 x 64
 *          block and a flag per SM) that let every SM take an equal share
 *          of the (weight tile, k-block) iterations; given fewer bytes the
 *          call splits K over thread-block clusters instead, with the same
 *          results.  The environment variable ZQ_EVEN_SPLIT = off | on
 *          (read on every call) turns that choice off, or on for every
 *          T <= 64.  The query reads the current device's SM count; with
 *          no usable device it returns the requantizing kinds' larger size
 *          and 0 for the others.
 * Constraints: K % 16 == 0, N % 16 == 0, N % G == 0, K <= ZQ_MAX_K.
 * Errors: NULL, SHAPE, ALIGN, OVERFLOW, DTYPE, WORKSPACE, CUDA, DEVICE. */
size_t zq_w8a8_linear_workspace(int64_t T, int64_t K, int64_t N, int out_kind);
int zq_w8a8_linear(const int8_t* xq, const float* s_tok, int64_t T, int64_t K,
                   const int8_t* Wq, const float* s_grp, int64_t N, int64_t group_rows,
                   const float* bias, int act, int out_kind,
                   void* y, float* s_tok_out,
                   void* workspace, size_t workspace_bytes, void* stream);

/* ---- one quantized linear layer from floating-point activations ----------
 * [ZQ] fused flowchart, both kernels: x -> [LN + Quantize] -> [GEMM +
 * DeQuantize].  gamma != NULL: zq_ln_quant(x, gamma, beta, eps); gamma ==
 * NULL: zq_act_quant(x, NULL, ZQ_ACT_NONE) (beta and eps ignored).  Then
 * zq_w8a8_linear with the remaining arguments.  The quantized activations
 * live in the workspace (zq_linear_block_workspace bytes).
 * Errors: the union of the two calls'. */
size_t zq_linear_block_workspace(int64_t T, int64_t K, int64_t N, int out_kind);
int zq_linear_block(const void* x, int x_dtype, int64_t T, int64_t K,
                    const float* gamma, const float* beta, float eps,
                    const int8_t* Wq, const float* s_grp, int64_t N, int64_t group_rows,
                    const float* bias, int act, int out_kind, void* y, float* s_tok_out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ---- requantizing linear without caller scratch ---------------------------
 * No counterpart on the source pages: this entry point exists for callers,
 * not for the method.  It computes what zq_w8a8_linear computes with
 * out_kind = ZQ_OUT_I8_REQUANT, through the same kernels and with the same
 * results, but takes no workspace and allocates nothing.
 *
 * Who needs it: callers that cannot obtain device memory themselves -- code
 * running inside a host framework that owns every device allocation and
 * gives its plugins no workspace, or latency-critical serving loops in which
 * a cudaMalloc (it may synchronize the device) is not allowed once serving
 * has started.
 *
 * Scratch: one array of ZQ_NOALLOC_SCRATCH_BYTES in device memory, owned by
 * the library.  Every GPU that loads the library holds it until the process
 * exits.  What a call needs of it depends on the kernel the shape takes:
 * nothing for T > 64 and N <= 4096 (the row absmax is exchanged inside a
 * thread-block cluster); 4 * (T + ceil(T / 128)) bytes, rounded up to 256,
 * for T > 64 and wider rows (per-token absmax words and per-row-block
 * counters); round_up(4*T*N, 256) + round_up(4*T, 256) bytes otherwise (at
 * most 64 tokens, or rows of more column tiles of 256 than the GPU has SMs:
 * the fp32 output and the absmax words).  A call that needs more than the
 * array returns ZQ_ERR_SCRATCH before anything is enqueued.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it for the life
 * of the process; make that first call before any stream capture.  Do not
 * call this entry point on a device after cudaDeviceReset of that device:
 * the module is then loaded again and the kept address may be stale.
 * Sharing: all calls on a device use the same array and it keeps the last
 * call's contents (each call clears what must start at zero).  Calls whose
 * GPU work overlaps -- on different streams, or from different threads --
 * race on the array and give wrong results; order them on one stream.
 * Arguments, layouts and the other errors as zq_w8a8_linear: y is int8
 * [T, N], s_tok_out fp32 [T]; both outputs are required. */
#define ZQ_NOALLOC_SCRATCH_BYTES (64u << 20)
int zq_w8a8_linear_requant_noalloc(const int8_t* xq, const float* s_tok, int64_t T, int64_t K,
                                   const int8_t* Wq, const float* s_grp, int64_t N,
                                   int64_t group_rows, const float* bias, int act,
                                   int8_t* y, float* s_tok_out, void* stream);

/* ---- SmoothQuant smoothing (offline) ------------------------------------
 * [TS36] §1.3 SmoothQuant; "SmoothQuant技术解析：大模型INT8量化的突破与实践"
 * §2.2, §3.  Y = (X diag(s)^-1)(diag(s) W) is the same output; a per-channel
 * s chosen offline makes the activation channels' maxima alike, so per-token
 * activation quantization loses less to outlier channels.  The activation
 * side is folded into the LayerNorm feeding the linear, so the online calls
 * (zq_ln_quant, zq_w8a8_linear) run unchanged on the smoothed parameters.
 *
 * zq_smooth_calibrate: running per-channel absmax of the linear's input over
 * calibration batches.  The activation is a = LayerNorm(x; gamma, beta, eps)
 * (as zq_ln_quant computes it, beta may be NULL for 0) when gamma is
 * non-NULL, else a = x.  amax[j] = max(amax[j], max_t |a[t, j]|).
 * x      : [T, H] device, dtype x_dtype (ZQ_F32 or ZQ_BF16).
 * amax   : fp32 [H] device, in/out; fill it with zeros before the first
 *          batch; it must hold values >= 0.
 * Constraints: H % 16 == 0, H <= 32768.  Errors: NULL, SHAPE, ALIGN,
 * DTYPE, CUDA, DEVICE. */
int zq_smooth_calibrate(const void* x, int x_dtype, int64_t T, int64_t H,
                        const float* gamma, const float* beta, float eps,
                        float* amax, void* stream);

/* zq_smooth_weights: the factors and the fold.
 *   wmax_j = max_o |W[o, j]|;
 *   s_j    = amax_j^alpha / wmax_j^(1 - alpha), at least 1e-5 (powers in
 *            double, rounded once to fp32); s_j = 1 where amax_j or wmax_j
 *            is 0 (the SmoothQuant paper's rule; the pages name the paper
 *            but not its formula);
 *   W_out[o, j] = W[o, j] * s_j;  gamma_out_j = gamma_j / s_j;
 *   beta_out_j = beta_j / s_j   (each one IEEE fp32 rounding).
 * W      : fp32 [N, K] device (output rows o, input channels j);
 * amax   : fp32 [K] device, from zq_smooth_calibrate;
 * alpha  : migration strength in [0, 1] (0.5 balances the activation and
 *          weight maxima, 1 makes every activation channel's max 1);
 * gamma, beta : fp32 [K] device or NULL (then not folded);
 * W_out  : fp32 [N, K] device (may be W); gamma_out, beta_out : fp32 [K]
 *          (may alias gamma, beta; required when those are given);
 * s      : fp32 [K] device (output; also used as scratch during the call).
 * Quantize W_out with zq_quantize_weights and pass gamma_out/beta_out to
 * zq_ln_quant.  Constraints: K % 16 == 0.  Errors: NULL, SHAPE, ALIGN,
 * DTYPE (alpha outside [0, 1]), CUDA, DEVICE. */
int zq_smooth_weights(const float* W, int64_t N, int64_t K, const float* amax, float alpha,
                      const float* gamma, const float* beta, float* W_out,
                      float* gamma_out, float* beta_out, float* s, void* stream);

/* ---- LLM.int8() mixed-precision decomposition ----------------------------
 * [TS36] §1.1 (LLM.int8()): the input columns holding a value above the
 * threshold alpha (6.0 on the pages) form the outlier set O; X[:, O] and the
 * matching weight columns are multiplied in FP16, the other columns run
 * through the INT8 path, and the two results are added.  Here, for a linear
 * fed by a LayerNorm:
 *   1. zq_smooth_calibrate(x, gamma, beta) gives the per-column absmax of
 *      the LayerNorm output over the batch (zero-filled amax first);
 *   2. zq_llmint8_select picks O = {j : amax_j >= threshold}, the lowest
 *      ZQ_LLMINT8_MAX_OUTLIERS of them, and writes gamma/beta with zeros on
 *      those columns;
 *   3. zq_ln_quant(x, gamma_m, beta_m) quantizes the other columns per token
 *      (the decomposed columns become zero codes and do not set the scale);
 *   4. zq_llmint8_outlier_act and zq_llmint8_outlier_weights gather the
 *      decomposed columns of the LayerNorm output and of the fp32 weights as
 *      fp16 (round to nearest even), [T, 8] and [N, 8], zeros past the count;
 *   5. zq_w8a8_linear_llmint8 runs the W8A8 GEMM (weights group-quantized
 *      offline over all columns) whose epilogue adds sum_k xo[t,k] wo[o,k]
 *      (exact fp16 products, fp32 accumulation) before bias and activation.
 * idx: int32 [ZQ_LLMINT8_MAX_OUTLIERS] device (-1 past the count);
 * count: int32 [1] device, the total number of columns >= threshold (it may
 * exceed ZQ_LLMINT8_MAX_OUTLIERS; only the first ones are decomposed).
 * Constraints: K % 16 == 0, K <= ZQ_MAX_H; out_kind ZQ_OUT_F32 or ZQ_OUT_BF16.
 * Errors: NULL, SHAPE, ALIGN, DTYPE, CUDA, DEVICE. */
#define ZQ_LLMINT8_MAX_OUTLIERS 8
int zq_llmint8_select(const float* amax, int64_t K, float threshold, const float* gamma,
                      const float* beta, int32_t* idx, int32_t* count, float* gamma_m,
                      float* beta_m, void* stream);
int zq_llmint8_outlier_act(const void* x, int x_dtype, int64_t T, int64_t K, const float* gamma,
                           const float* beta, float eps, const int32_t* idx, const int32_t* count,
                           void* xo, void* stream);
int zq_llmint8_outlier_weights(const float* W, int64_t N, int64_t K, const int32_t* idx,
                               const int32_t* count, void* wo, void* stream);
int zq_w8a8_linear_llmint8(const int8_t* xq, const float* s_tok, int64_t T, int64_t K,
                           const int8_t* Wq, const float* s_grp, int64_t N, int64_t group_rows,
                           const float* bias, int act, int out_kind, const void* xo, const void* wo,
                           void* y, void* stream);

/* ---- K-axis weight groups ------------------------------------------------
 * [ZQ] group-wise weight quantization and [TS36] §1.2.2 (group-wise weights;
 * the INT32 accumulation scaled by the weight and activation scales), with
 * the groups taken along the input axis: group (o, j) is output row o and
 * the group_cols (Gk) consecutive input columns j*Gk .. j*Gk+Gk-1, with its
 * own scale.  The scale then varies along the contraction, so the linear
 * scales every group's exact INT32 partial product before summing:
 *   y[t, o] = act(s_tok[t] * sum_j s_w[j, o] * acc_j[t, o] + bias[o]),
 *   acc_j[t, o] = sum over k in group j of xq[t, k] * Wq[o, k].
 * zq_quantize_weights_kgroups:
 *   W   : fp32 [N, K] device, row-major.
 *   Wq  : int8 [N, K] device (output): rint(w * (127/absmax)), ties to even,
 *         clamped to [-127, 127]; an all-zero group gets zero codes.
 *   s_w : fp32 [K/Gk, N] device (output), GROUP-MAJOR: s_w[j*N + o] is the
 *         scale absmax/127 of group (o, j).
 *   Constraints: K % 16 == 0, K % Gk == 0.  Errors: NULL, SHAPE, ALIGN, CUDA,
 *   DEVICE.
 * zq_w8a8_linear_kgroups:
 *   xq, s_tok : int8 [T, K] and fp32 [T] device (from zq_ln_quant /
 *         zq_act_quant); Wq, s_w as written above; bias fp32 [N] or NULL;
 *   act ZQ_ACT_NONE or ZQ_ACT_GELU; out_kind ZQ_OUT_F32 or ZQ_OUT_BF16;
 *   y : [T, N] device (output).  The group sums accumulate in fp32 in the
 *   order j = 0, 1, ...; the token scale multiplies the sum, then bias.
 *   Constraints: Gk % 32 == 0 (a tensor-core k-step of 32 INT8 values never
 *   straddles a group), Gk <= 256 (|acc_j| <= 2^22, see the kernel), K % Gk
 *   == 0, N % 16 == 0.  Alignment: xq, Wq, y, s_w and bias 16 bytes; s_tok 4.
 *   Errors: NULL, SHAPE, ALIGN, DTYPE, CUDA, DEVICE. */
int zq_quantize_weights_kgroups(const float* W, int64_t N, int64_t K, int64_t group_cols,
                                int8_t* Wq, float* s_w, void* stream);
int zq_w8a8_linear_kgroups(const int8_t* xq, const float* s_tok, int64_t T, int64_t K,
                           const int8_t* Wq, const float* s_w, int64_t N, int64_t group_cols,
                           const float* bias, int act, int out_kind, void* y, void* stream);

/* ---- diagnostics ----------------------------------------------------------
 * zq_device_status: synchronizes `stream`, then reads and clears the device
 * flag that bounded waits set on expiry.  Returns ZQ_OK, ZQ_ERR_TIMEOUT or
 * ZQ_ERR_CUDA.  Not callable during stream capture.
 * zq_status_string: static text for a status code (never NULL).
 * zq_last_cuda_error: text of the last CUDA error seen by this thread's
 * calls (static storage, "no error" when none).
 * zq_version: library version as 10000*major + 100*minor + patch.
 * zq_launch_count: number of kernels this library has launched in this
 * process (all devices, all threads); for accounting in benchmarks.
 * zq_watchdog_selftest: see below. */
int zq_device_status(void* stream);
/* zq_watchdog_selftest: enqueues one tiny kernel whose only thread waits on
 * a barrier that nothing signals.  Its bounded wait expires after the
 * library's wait limit (about 2 s), records a site code in the device flag
 * and returns, exactly as an expired wait inside the GEMM does; the next
 * zq_device_status() then reports ZQ_ERR_TIMEOUT (and clears the flag) and
 * the CUDA context stays usable.  It exists to test that failure path
 * without faulting or hanging the GPU.  Returns ZQ_OK, ZQ_ERR_CUDA or
 * ZQ_ERR_DEVICE. */
int zq_watchdog_selftest(void* stream);
const char* zq_status_string(int status);
const char* zq_last_cuda_error(void);
int zq_version(void);
uint64_t zq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* ZQ_H_ */
