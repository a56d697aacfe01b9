/*
 * sq.h -- C ABI of libsq, the SmoothQuant W8A8 int8 linear layer for B200 (sm_100a).
 *
 * The operations are those of the SmoothQuant page
 * ("w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)"),
 * restated as functions on caller-owned device buffers:
 *
 *   calibration    s_j  = max(mx_j,1e-8)^a / max(mw_j,1e-8)^(1-a), clamped at 1e-8
 *                  (calibrate_smoothquant; running max of SmoothQuantW8A8.calibrate)
 *   weight prep    W~ = W * s ; per-output-row symmetric int8 (freeze_quantization,
 *                  quantize_per_channel_symmetric)
 *   act quant      X~ = X / s ; per-token symmetric int8 (forward,
 *                  quantize_per_token_symmetric)
 *   int8 linear    acc = Xq Wq^T (int32) ; Y = bf16(acc * x_scale[m] * w_scale[n] + bias[n])
 *                  (forward: "INT8 x INT8 -> INT32 -> fp32" on real hardware)
 *   backward       straight-through gradients of the learnable-alpha layer's
 *                  quantised-mode forward: dX, dW, db, ds, d eta_alpha
 *                  (STEQuantize, SmoothQuantW8A8.alpha / forward)
 *
 * and two comparison points from other pages:
 *
 *   per-tensor     one scale per tensor (quantized_linear.py, quantize_tensor)
 *   weight-only    bf16 activations times int8 weights (torchao,
 *                  Int8WeightOnlyQuantizedLinearWeight)
 *
 * Conventions shared by every entry point
 *   - Layouts are row-major and dense: X[M][K], C[R][K], W[N][K] (nn.Linear
 *     [d_out][d_in]), Xq[M][K], Wq[N][K], Y[M][N]; s[K], x_scale[M], w_scale[N],
 *     bias[N].  bf16 values travel as their 16-bit patterns (sq_bf16).
 *   - Every pointer is a DEVICE pointer owned by the caller; the library keeps no
 *     reference after the call returns and allocates no device memory.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and runs asynchronously: a returned SQ_OK means "validated and launched".
 *     Output buffers must not alias inputs.
 *   - Integer codes are symmetric: -127..127 (-128 is never produced); rounding
 *     is to nearest, ties to even.
 *   - Requirements: K % 16 == 0 (TMA rows are 16-byte multiples), every pointer
 *     16-byte aligned, M, N, K >= 1 (R >= 0).  Violations return an error code
 *     and launch nothing.  Inputs must be finite; NaN/Inf give unspecified codes.
 *   - Errors: the return value is an sq_status; sq_last_error() gives a
 *     human-readable message for the calling thread's last failure.
 *     Device-side wait timeouts (never expected in correct use) are latched in a
 *     per-process device word read by sq_device_status().
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

typedef uint16_t sq_bf16; /* bf16 bit pattern */

typedef enum {
  SQ_OK = 0,
  SQ_ERR_NULL = 1,        /* a required pointer is NULL */
  SQ_ERR_SHAPE = 2,       /* inconsistent or out-of-range sizes */
  SQ_ERR_ALIGN = 3,       /* K % 16 != 0 or a pointer not 16-byte aligned */
  SQ_ERR_ARG = 4,         /* alpha outside [0, 1], or another bad scalar */
  SQ_ERR_UNSUPPORTED = 5, /* device is not sm_100 */
  SQ_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed */
  SQ_ERR_TIMEOUT = 7,     /* a device-side wait ran out (see sq_device_status) */
  SQ_ERR_WORKSPACE = 8    /* workspace NULL or smaller than required */
} sq_status;

/* Library version, e.g. 100 for 0.1.0. */
SQ_API int sq_version(void);

/* Message for the calling thread's most recent failing call ("" if none). */
SQ_API const char* sq_last_error(void);

/* Name of a status code. */
SQ_API const char* sq_status_string(sq_status st);

/* ------------------------------------------------------------ calibration
 * sq_calibrate -- smoothing factor s from activation and weight statistics.
 * Page: calibrate_smoothquant (formula for s_j, the 1e-8 clamps),
 * SmoothQuantW8A8.calibrate (running per-channel max of |X| over batches) and
 * freeze_quantization (s from the running max and the weight's per-input-
 * channel max).
 *
 *   C[R][K]    calibration activations (bf16); may be NULL when R == 0
 *   W[N][K]    layer weight (bf16)
 *   alpha      smoothing strength in [0, 1]
 *   s[K]       OUT: fp32 smoothing factor.  mx^a and mw^(1-a) are evaluated
 *              in float64 and the quotient is rounded once to fp32.
 *   mx_inout   NULL, or [K] fp32 running max-abs of activations: read, merged
 *              with this batch's column max, written back (start from zeros).
 *              With R == 0 it must be non-NULL and s comes from it alone:
 *              that call followed by sq_prepare_weight is the page's
 *              recompute_smooth_scale (new alpha after freezing).
 *   workspace  device scratch of at least sq_calibrate_workspace_bytes(K)
 *              bytes, 16-byte aligned; contents on entry are ignored.
 * Launches: a small kernel that clears the workspace, then one kernel
 * (column max-abs over C and W, streamed through shared memory by TMA; the
 * last block to finish each 256-column stripe computes s there and zeroes
 * the stripe's workspace words again).
 */
SQ_API size_t sq_calibrate_workspace_bytes(int64_t K);
SQ_API sq_status sq_calibrate(const sq_bf16* C, int64_t R, int64_t K,
                       const sq_bf16* W, int64_t N, float alpha,
                       float* s, float* mx_inout,
                       void* workspace, size_t workspace_bytes, void* stream);

/* sq_calibrate_noalloc -- sq_calibrate without a workspace argument.
 * The SmoothQuant page has no counterpart: this is a library convenience.
 * It is for callers that cannot hand the library scratch memory: code
 * embedded in a host engine that owns every device byte through its own
 * fixed pool and gives plugins no way to call cudaMalloc, or loops where an
 * allocation (which may block or synchronise the device) is not allowed.
 *   Arguments and results are those of sq_calibrate, minus the workspace.
 *   Limit: K <= 16384 (SQ_ERR_SHAPE with a message beyond that).
 *   Scratch: a fixed device array of about 128 KiB inside libsq, held by every GPU that
 *   loads the library until the process exits.  Nothing is allocated per call.
 *   The first call on each device looks up that array's device address (a
 *   one-time set-up, made with that device current); make that first call
 *   before any stream capture on the device.
 *   All calls on a device share the array: calls that may run at the same time
 *   on the GPU (different streams without ordering) race and give wrong s.
 *   Launches: one kernel and no memset.  The array is zero when the library
 *   loads and each call zeroes the words it used once it has read them, so
 *   one call's values never reach the next.  A call that timed out on the
 *   device (sq_device_status) may leave the array dirty; clearing the status
 *   with sq_device_status(&flags, 1) zeroes it again.
 */
SQ_API sq_status sq_calibrate_noalloc(const sq_bf16* C, int64_t R, int64_t K,
                                      const sq_bf16* W, int64_t N, float alpha,
                                      float* s, float* mx_inout, void* stream);

/* --------------------------------------------------------- weight prepare
 * sq_prepare_weight -- fold s into W and quantise per output channel.
 * Page: freeze_quantization (W_smooth = weight_fp * s) and
 * quantize_per_channel_symmetric(axis = 0).
 *
 *   W[N][K] bf16 in; s[K] fp32 in
 *   Wq[N][K]  OUT int8 codes  q = clamp(round_half_even(fl(W*s) / w_scale), +-127)
 *   w_scale[N] OUT fp32  fl( max(max_j |fl(W*s)|, 1e-8) / 127 )
 * Every step is the page's fp32 operation (correctly rounded), so the result is
 * bit-identical to an IEEE fp32 evaluation of the page's formulas.
 */
SQ_API sq_status sq_prepare_weight(const sq_bf16* W, int64_t N, int64_t K, const float* s,
                            int8_t* Wq, float* w_scale, void* stream);

/* ------------------------------------------------------- activation quant
 * sq_quantize_act -- dynamic per-token quantisation of X / s.
 * Page: forward (X_smooth = X / s) and quantize_per_token_symmetric.
 *
 *   X[M][K] bf16 in; s[K] fp32 in
 *   Xq[M][K]   OUT int8  q = clamp(round_half_even(fl(X/s) / x_scale), +-127)
 *   x_scale[M] OUT fp32  fl( max(max_j |fl(X/s)|, 1e-8) / 127 )
 * Divisions are correctly rounded fp32 divisions, as on the page.
 */
SQ_API sq_status sq_quantize_act(const sq_bf16* X, int64_t M, int64_t K, const float* s,
                          int8_t* Xq, float* x_scale, void* stream);

/* ------------------------------------------- per-tensor baseline quantiser
 * sq_quantize_per_tensor -- one scale for a whole tensor, the W8A8 variant the
 * SmoothQuant path is compared with.  Page: "quantized_linear.py --
 * QuantizedLinear + apply_w8a8", quantize_tensor (scale = max|x| / 127 on fp32
 * values, replaced by 1.0 when below 1e-8; codes round-half-even of the fp32
 * quotient x / scale, clamped to [-128, 127]) and QuantizedLinear.forward (the
 * product of the two dequantised tensors plus the bias).  With the weight and
 * the activations each quantised this way, sq_linear(Xq, x_scale, Wq,
 * w_scale, bias) computes that forward with an exact int8 product.
 *   A[rows][K]       bf16 tensor (weight or activations), K % 16 == 0
 *   Aq[rows][K]      OUT int8 codes (always within [-127, 127]: the maximum
 *                    maps to +-127)
 *   scale_rows[rows] OUT fp32: every entry holds the tensor's scale, the form
 *                    sq_linear takes for x_scale / w_scale
 *   workspace        at least sq_quantize_per_tensor_workspace_bytes() bytes,
 *                    16-byte aligned; contents on entry are ignored
 * Launches two kernels (block maxima of |A|, then the scale and the codes);
 * A is read twice from HBM.
 */
SQ_API size_t sq_quantize_per_tensor_workspace_bytes(void);
SQ_API sq_status sq_quantize_per_tensor(const sq_bf16* A, int64_t rows, int64_t K, int8_t* Aq,
                                        float* scale_rows, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* ------------------------------------------------ int8 weight-only linear
 * sq_linear_weight_only -- the decode comparison point beside W8A8: the
 * activations stay bf16 and only the weight is int8.  Page: torchao,
 * Int8WeightOnlyQuantizedLinearWeight._quantized_op:
 *     Y[m][n] = bf16( (sum_k X[m][k] * Wq[n][k]) * w_scale[n] + bias[n] ).
 *   X[M][K] bf16, Wq[N][K] int8 and w_scale[N] fp32 (per output channel, e.g.
 *   from sq_prepare_weight with s = 1), bias[N] bf16 or NULL -> Y[M][N] bf16.
 * The sum runs in fp32 on the CUDA cores (there is no int8 x bf16 tensor-core
 * product), in an order of its own, and is rounded once to bf16 after the
 * scale and bias: the result is within one bf16 ulp plus the fp32 summation
 * error of the exact value.  Built for few tokens (groups of 8 re-read Wq).
 * K <= 16384, a multiple of 16.
 */
SQ_API sq_status sq_linear_weight_only(const sq_bf16* X, int64_t M, const int8_t* Wq, const float* w_scale,
                                       const sq_bf16* bias, int64_t N, int64_t K, sq_bf16* Y, void* stream);

/* ---------------------------------- learnable-alpha straight-through backward
 * sq_ste_backward -- gradients of the quantised-mode forward of the
 * learnable-alpha layer.  Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e
 * alpha APRENDIVEL (V5)": SmoothQuantW8A8.alpha (alpha = sigmoid(eta_alpha)),
 * SmoothQuantW8A8.forward (s recomputed from the running activation max and
 * the detached weight max with the trainable alpha, X / s and weight * s
 * fake-quantised per token and per output channel, Y = X_q_deq W_q_deq^T + b)
 * and STEQuantize.backward (the gradient passes through round and clamp; the
 * scales receive none).  With G = dL/dY:
 *     dX[m][k] = (G Wdq)[m][k] / s[k]           Wdq = Wq * w_scale (per row n)
 *     dW[n][k] = (G^T Xdq)[n][k] * s[k]         Xdq = Xq * x_scale (per row m)
 *     db[n]    = sum_m G[m][n]
 *     d_eta    = alpha (1 - alpha) sum_k ds[k] raw[k] (ln mx[k] + ln mw[k]),
 * where ds[k] = sum_n dL/dW_smooth[n][k] W[n][k] - sum_m dL/dX_smooth[m][k]
 * X[m][k] / s[k]^2, raw[k] = mx[k]^alpha / mw[k]^(1-alpha) (mx, mw clamped at
 * 1e-8; channels with raw[k] < 1e-8 sit on the clamp of s and contribute
 * nothing) and mw[k] = max_n |W[n][k]|.
 *   G[M][N] bf16        dL/dY (an auxiliary loss on Y enters through it)
 *   X[M][K], W[N][K]    the layer's bf16 input and weight
 *   s[K]                the forward's smoothing factor (sq_calibrate with
 *                       mx_inout = mx, R = 0 and this alpha)
 *   mx[K]               the running activation max (calib_max_abs)
 *   alpha               the fp32 alpha of the forward, in [0, 1]
 *   Xq, x_scale, Wq, w_scale   the forward's codes and scales
 *                       (sq_quantize_act and sq_prepare_weight with s)
 *   dX[M][K], dW[N][K]  OUT fp32
 *   db[N]               OUT fp32, or NULL
 *   ds[K]               OUT fp32: dL/ds (the gradient reaching s), or NULL
 *   d_eta[1]            OUT fp32: dL/d eta_alpha
 *   workspace           sq_ste_backward_workspace_bytes(M, N, K) bytes,
 *                       16-byte aligned, contents ignored on entry
 * Requirements beyond the general ones: N % 8 == 0 (G is read by TMA rows).
 * The two products run on the tensor cores with the codes as exact bf16
 * operands and G times the scale split into two bf16 halves (2^-16 relative),
 * accumulating in fp32: each element of dX and dW is within
 * 2^-16 + 2^-23 + 2C * 2^-22 of the sum of its absolute products (C the
 * contraction length).  ds is formed from the quantisation errors W*s - Wdq
 * and X/s - Xdq, so it carries that relative error without cancellation.
 * Launches 6 kernels; reads G once.
 */
SQ_API size_t sq_ste_backward_workspace_bytes(int64_t M, int64_t N, int64_t K);
SQ_API sq_status sq_ste_backward(const sq_bf16* G, const sq_bf16* X, const sq_bf16* W, const float* s,
                                 const float* mx, float alpha, const int8_t* Xq, const float* x_scale,
                                 const int8_t* Wq, const float* w_scale, int64_t M, int64_t N, int64_t K,
                                 float* dX, float* dW, float* db, float* ds, float* d_eta, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------- int8 linear
 * sq_linear -- Y = bf16( (Xq Wq^T)[m][n] * x_scale[m] * w_scale[n] + bias[n] ).
 * Page: forward ("INT8 x INT8 -> INT32 -> fp32"; bias added after the product).
 *
 *   Xq[M][K], Wq[N][K] int8; x_scale[M], w_scale[N] fp32; bias[N] bf16 or NULL
 *   Y[M][N]   OUT bf16.  The int32 accumulation is exact (|acc| <= 127^2 K,
 *             K <= 133143); the epilogue runs in fp32 and rounds to bf16
 *             (nearest even), i.e. within one bf16 ulp of the exact value.
 *   workspace  optional device scratch (16-byte aligned; contents on entry
 *              ignored).  sq_workspace_bytes(M, N, K) gives the size that lets
 *              the GEMM split K over pairs of CTAs when the output has few
 *              128 x 256 tiles (at most half as many as SMs), exchanging
 *              partial sums through it (64 KB per CTA); 0 when no such split
 *              applies.  NULL or less than that size selects a path that needs
 *              none (same results, slower for such shapes).
 * Runs the tcgen05 (kind::i8) GEMM: TMA-fed shared-memory tiles, int32
 * accumulators in tensor memory, fused dequant + bias epilogue.  M <= 32 uses
 * a weight-streaming kernel instead (split-K over a thread-block cluster).
 */
SQ_API size_t sq_workspace_bytes(int64_t M, int64_t N, int64_t K);
SQ_API sq_status sq_linear(const int8_t* Xq, const float* x_scale, const int8_t* Wq,
                    const float* w_scale, const sq_bf16* bias,
                    int64_t M, int64_t N, int64_t K, sq_bf16* Y,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------ auxiliary loss (learnable alpha)
 * sq_rel_mse -- the relative-MSE auxiliary loss that trains alpha, and its
 * gradient folded into the gradient of the quantised output.  Page: module
 * docstring of "w8a8_smoothquant.py" (V5): ||Y_fp - Y_q||_F^2 / ||Y_fp||_F^2
 * added to the total loss so that its gradient reaches eta_alpha;
 * SmoothQuantW8A8.quantization_error (the unsquared ratio, norm floored at
 * 1e-12).
 *
 *   Y_fp[M][N], Y_q[M][N] bf16 (the unquantised and the W8A8 layer outputs)
 *   loss_out   one double (device): sum (Y_fp - Y_q)^2 / max(sum Y_fp^2, 1e-24),
 *              accumulated in float64
 *   G_in, G_out  [M][N] bf16 or both NULL; when given,
 *              G_out = bf16(G_in + lambda * 2 (Y_q - Y_fp) / max(sum Y_fp^2, 1e-24)),
 *              evaluated in float64 and rounded once (nearest, ties to even):
 *              the G of sq_ste_backward for a total loss L + lambda * aux.
 *              G_in == G_out is allowed (in place).  Y_fp carries no gradient
 *              (it does not depend on alpha).
 *   workspace  at least sq_rel_mse_workspace_bytes() bytes, 16-byte aligned.
 * Pointers 16-byte aligned (loss_out 8-byte); lambda finite.  Two kernels.
 */
SQ_API size_t sq_rel_mse_workspace_bytes(void);
SQ_API sq_status sq_rel_mse(const sq_bf16* Y_fp, const sq_bf16* Y_q, int64_t M, int64_t N, double lambda,
                     const sq_bf16* G_in, sq_bf16* G_out, double* loss_out,
                     void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------- fused forward
 * sq_forward -- the per-batch path: sq_quantize_act followed by sq_linear,
 * Y from bf16 X.  Page: forward of SmoothQuantW8A8 once frozen.
 *
 *   X[M][K] bf16, s[K], Wq[N][K], w_scale[N], bias[N] or NULL -> Y[M][N] bf16
 *   workspace  at least sq_forward_workspace_bytes(M, N, K) bytes (holds the
 *              intermediate Xq and x_scale, then sq_linear's workspace);
 *              contents on entry are ignored.
 * The codes and scales are identical to those of sq_quantize_act.  Up to 8
 * tokens the quantisation runs inside the weight-streaming kernel; otherwise
 * the row quantiser runs first and sq_linear's kernels follow.
 */
SQ_API size_t sq_forward_workspace_bytes(int64_t M, int64_t N, int64_t K);
SQ_API sq_status sq_forward(const sq_bf16* X, const float* s, const int8_t* Wq,
                     const float* w_scale, const sq_bf16* bias,
                     int64_t M, int64_t N, int64_t K, sq_bf16* Y,
                     void* workspace, size_t workspace_bytes, void* stream);

/* -------------------------------------- forward, quantisation in the GEMM
 * sq_forward_prologue -- the same Y as sq_forward, with the per-token
 * quantisation of X / s done inside the GEMM instead of by a separate pass
 * that writes Xq to global memory.  Page: forward of SmoothQuantW8A8 once
 * frozen (X / s, quantize_per_token_symmetric, the int8 product, the
 * dequantisation and bias).
 *
 *   X[M][K] bf16, s[K], Wq[N][K], w_scale[N], bias[N] or NULL -> Y[M][N] bf16
 *   workspace  at least sq_forward_prologue_workspace_bytes(M, K) bytes; it
 *              receives x_scale[M] (at offset 0) and RN(1/s_j)[K]; contents on
 *              entry are ignored.
 * Two kernels: a pre-pass that reads X once and writes only the per-token
 * scales (the scales of sq_quantize_act, bit for bit), then a CTA-pair GEMM
 * (tiles of 256 x 512) whose converter warps read X in bf16 and write the int8
 * codes straight into the tensor core's shared-memory operand.  The codes, and
 * so Y, are identical to those of sq_quantize_act followed by sq_linear.
 * Meant for many tokens (prefill); any M >= 1 is accepted.  K % 16 == 0,
 * 16 <= K <= 16384; pointers 16-byte aligned (bias may be NULL).
 */
SQ_API size_t sq_forward_prologue_workspace_bytes(int64_t M, int64_t K);
SQ_API sq_status sq_forward_prologue(const sq_bf16* X, const float* s, const int8_t* Wq,
                              const float* w_scale, const sq_bf16* bias,
                              int64_t M, int64_t N, int64_t K, sq_bf16* Y,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------- test hook
 * sq_gemm_s32 -- the same tcgen05 GEMM main loop with a raw int32 epilogue:
 * acc[M][N] = Xq Wq^T, exposing the accumulator for bit-exact checks.
 */
SQ_API sq_status sq_gemm_s32(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K,
                      int32_t* acc, void* stream);

/* ------------------------------------------------------ device status word
 * sq_device_status -- read (and with clear != 0, reset) the device-side status
 * flags of the current device: bit 0 = a bounded wait in a library kernel (a
 * GEMM pipeline wait, or a wait for streamed rows in the calibration and
 * quantisation kernels) timed out; the results of that call are undefined.
 * Synchronises the device.  Returns SQ_ERR_TIMEOUT if any bit is set.
 * Clearing a set status also re-zeroes the scratch of sq_calibrate_noalloc.
 * Both the read and the clear apply to the CURRENT device only: a timed-out
 * call on another device stays flagged (and its no-allocation scratch dirty)
 * until that device is made current and its status cleared.
 */
SQ_API sq_status sq_device_status(uint32_t* flags, int clear);

/* --------------------------------------------------------- fault injection
 * sq_debug_fail_after -- host-side fault injection for tests: after `n` more
 * successful launches, entry points return SQ_ERR_CUDA without touching the
 * GPU.  n < 0 disables injection (the default).
 */
SQ_API void sq_debug_fail_after(int n);

/* sq_debug_pipeline_stall -- device-side failure test: while enabled
 * (enable != 0), the GEMM kernels used by sq_linear / sq_forward / sq_gemm_s32
 * (any M), by sq_forward_prologue, by sq_ste_backward and by
 * sq_linear_weight_only, and the column-max kernel of sq_calibrate, never
 * load their first pipeline stage and every pipeline wait gives up after
 * timeout_ns (<= 0: the normal 2 s).  The kernel then sets bit 0 of
 * the device status word, drains its copies in flight, frees its tensor memory
 * and returns: the call's output is invalid, the CUDA context stays usable and
 * sq_device_status() reports SQ_ERR_TIMEOUT.  No GPU fault is involved.
 * enable == 0 restores normal operation. */
SQ_API void sq_debug_pipeline_stall(int enable, int64_t timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
