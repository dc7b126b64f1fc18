/*
 * sq_w8a8.h -- C ABI of the SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a).
 *
 * The method (SmoothQuant): a linear layer Y = X W is rewritten exactly as
 * Y = (X diag(s)^-1)(diag(s) W), with a per-input-channel migration factor
 *     s_j = max|X_j|^alpha / max|W_j|^(1 - alpha),
 * so that activation outliers move into the weights; the smoothed weights are
 * quantised per output channel and the smoothed activations per token to
 * symmetric INT8, and the product runs as an INT8 x INT8 -> int32 GEMM whose
 * epilogue multiplies back the two scales.
 *   Pages: "4.2 W8A8 量化与 SmoothQuant" (sec. 3 equivalence, sec. 4 factor and alpha,
 *   sec. 6 LayerNorm folding, sec. 7.1 calibration pipeline and granularity);
 *   "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section (W_j is row j of W;
 *   per-token / per-channel scales factor out of the GEMM);
 *   "SmoothQuant大模型平滑量化技术", Python demo (scale = max|.|/127, round, clip +-127).
 *
 * Conventions shared by every call
 *   - Every pointer except `stream` and the documented host-side outputs is a DEVICE
 *     pointer owned by the caller.  The library allocates no memory and keeps no
 *     state besides cached device properties and a device-side error word.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *     enqueues work on it and returns; nothing synchronises.
 *   - Matrices are row-major with a leading dimension `ld*` counted in elements.
 *     bf16 (SQ_BF16) and fp32 (SQ_F32) inputs need 16-byte aligned base pointers,
 *     rows that are a multiple of 16 bytes (cols * elt % 16 == 0) and ld * elt % 16 == 0.
 *   - Arithmetic: IEEE binary32, round to nearest even, one rounding per written
 *     operation (no contraction).  int8 codes are clamp(rne(v / scale), -127, 127);
 *     a scale of 0 (all-zero row or column) gives all-zero codes.
 *   - Errors: arguments are validated on the host before anything is enqueued and a
 *     bad argument returns its status with nothing launched.  A failed launch returns
 *     SQ_ERR_CUDA.  Faults inside a kernel surface at the caller's next
 *     synchronisation.  A kernel whose bounded internal wait runs out stops early and
 *     records a code readable with sq_device_error().
 *   - Sizes: a zero-sized problem returns SQ_OK and launches nothing, except that an
 *     empty calibration reduction (no rows) with accumulate = 0 zero-fills `out`; calls
 *     that need K > 0 (LayerNorm, GEMM) reject K == 0 as SQ_ERR_INVALID_ARG.
 */
#ifndef SQ_W8A8_H
#define SQ_W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, ld < cols, ...      */
  SQ_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement (K limits)    */
  SQ_ERR_ALIGNMENT = 3,   /* pointer / row / leading dimension not 16-byte aligned      */
  SQ_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed                      */
  SQ_ERR_WORKSPACE = 5    /* the GEMM workspace is missing or too small                  */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_BF16 = 1, SQ_I32 = 2 } sq_dtype;

/* Largest K the int32 accumulator holds: K * 127^2 <= 2^31 - 1 up to K = 133144;
 * rounded down to a multiple of 16. */
#define SQ_MAX_K 133136
/* Largest K of the LayerNorm / per-token quantiser (row kept on chip). */
#define SQ_MAX_K_ROW 65536

/* sq_calib_absmax -- calibration statistics, one pass over x.
 *   axis 0: out[j] = max_i |x[i, j]|, j < cols  (per input channel over calibration
 *           tokens: "4.2 W8A8…" sec. 7.1 step 2, "量化…PTQ" SmoothQuant section)
 *   axis 1: out[i] = max_j |x[i, j]|, i < rows  (per row; for weights W[K, N] row j is
 *           input channel j: "量化…PTQ" SmoothQuant section)
 *   x: [rows, cols] bf16 or fp32, leading dimension ld (elements).  out: fp32 [cols] or
 *   [rows].  accumulate = 0 overwrites out; 1 takes the running max with its contents
 *   (statistics over several calibration batches).  The result is exact (a max). */
sq_status sq_calib_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                          int axis, int accumulate, float* out, void* stream);

/* sq_calib_ln_absmax -- per-channel absmax of a LayerNorm output, without writing it:
 *   out[j] = max_i |LN(x_i)_j|, LN(x)_j = fma((x_j - mu) * rstd, gamma_j, beta_j),
 *   rstd = 1 / sqrt(var + eps) (biased variance, two passes, fixed reduction order of
 *   sq_ln_smooth_quant).  This is the statistic of the linear's input when a LayerNorm
 *   precedes it ("4.2 W8A8…" sec. 6 and 7.1).  x: [rows, K] bf16/fp32, ldx; gamma [K]
 *   fp32; beta [K] fp32 or NULL (= 0).  K % 16 == 0, K <= SQ_MAX_K_ROW.
 *   accumulate as for sq_calib_absmax. */
sq_status sq_calib_ln_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t K, int64_t ldx,
                             const float* gamma, const float* beta, float eps, int accumulate,
                             float* out, void* stream);

/* sq_smooth_factors -- s_j = ax_j^alpha / aw_j^(1 - alpha) ("4.2 W8A8…" sec. 4).
 *   ax, aw, s: fp32 [K].  0 <= alpha <= 1.  Evaluated in binary64 and rounded once to
 *   binary32: sqrt(ax/aw) at alpha = 0.5, ax at 1, 1/aw at 0, exp(alpha log ax -
 *   (1 - alpha) log aw) otherwise.  A channel with ax_j = 0 or aw_j = 0 gets s_j = 1. */
sq_status sq_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s,
                            void* stream);

/* sq_fold_quant_weights -- fold diag(s) into W and quantise per output channel
 * ("4.2 W8A8…" sec. 6 and 7.1):
 *   W'[j, k] = s_j * W[j, k]; sw[k] = max_j |W'[j, k]| / 127;
 *   Wq[k, j] = clamp(rne(W'[j, k] / sw[k]), -127, 127)
 *   gamma_f[j] = gamma[j] / s_j and beta_f[j] = beta[j] / s_j (LayerNorm folding),
 *   each written only when both its input and output pointers are non-NULL.
 *   W: [K, N] bf16/fp32 (row j = input channel), leading dimension ldw.
 *   Wq: int8 [N, K], K contiguous (the GEMM's K-major B operand), 16-byte aligned.
 *   sw: fp32 [N]; it also holds the column maxima while the call runs, so it must not
 *   alias an input.  K % 16 == 0, K <= SQ_MAX_K. */
sq_status sq_fold_quant_weights(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw,
                                const float* s, const float* gamma, const float* beta,
                                int8_t* Wq, float* sw, float* gamma_f, float* beta_f,
                                void* stream);

/* sq_fold_kernel_launches -- how many kernels sq_fold_quant_weights (and
 *   sq_fold_quant_weights_fp8) launches for these arguments: 1 for the one-pass routes,
 *   3 for the streaming two-pass route (column maxima, codes, scales), 0 when K or N is 0.
 *   Host only: no CUDA call, no validation beyond that (the fold itself validates).
 *   The pages have no counterpart; it reports this library's routing, for launch
 *   accounting by callers that count kernels. */
int sq_fold_kernel_launches(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw);

/* sq_fold_next_smoothing -- the next linear's smoothing folded offline into this linear
 * ("量化：只压权重，与训练后量化（PTQ）", SmoothQuant section: diag(s)^-1 can be folded offline into
 * the preceding LayerNorm or linear layer, at no runtime cost; "4.2 W8A8…" sec. 6: the input of
 * a linear comes from a LayerNorm or from the previous GEMM).  When this linear's output is the
 * next linear's input (with no LayerNorm between), dividing this linear's per-output-channel
 * weight scale by the next linear's factors makes its GEMM emit the smoothed input directly:
 *   sw_out[n] = sw[n] / s_next[n]  (binary32, correctly rounded), so that
 *   y'[m, n] = ((float)acc[m, n] * sx[m]) * sw_out[n]  is  y[m, n] / s_next[n]  up to rounding.
 *   The next linear then folds s_next into its own weights as usual (sq_fold_quant_weights)
 *   and quantises y' with unit factors (sq_ln_smooth_quant, plain mode, s = 1).
 *   sw, s_next, sw_out: fp32 [N] device arrays (sw_out may alias sw).  Works for INT8 and FP8
 *   scales alike. */
sq_status sq_fold_next_smoothing(const float* sw, const float* s_next, int64_t N, float* sw_out, void* stream);

/* sq_ln_smooth_quant -- fused LayerNorm -> X diag(s)^-1 -> per-token INT8
 * ("4.2 W8A8…" sec. 6 and 7.1; "量化…PTQ" per-token activations):
 *   LayerNorm mode (gamma_f != NULL, s == NULL): y = LN(x) with the folded gamma' = gamma/s,
 *     beta' = beta/s (beta_f may be NULL = 0); statistics as in sq_calib_ln_absmax.
 *   plain mode (gamma_f == NULL, s != NULL): y_j = x_j / s_j (input from a previous GEMM).
 *   sx[m] = max_j |y[m, j]| / 127;  xq[m, j] = clamp(rne(y[m, j] / sx[m]), -127, 127).
 *   x: [M, K] bf16/fp32, ldx.  xq: int8 [M, K] dense, 16-byte aligned.  sx: fp32 [M].
 *   K % 16 == 0, K <= SQ_MAX_K_ROW.  Exactly one of gamma_f and s is non-NULL. */
sq_status sq_ln_smooth_quant(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx,
                             const float* gamma_f, const float* beta_f, const float* s, float eps,
                             int8_t* xq, float* sx, void* stream);

/* sq_ln_smooth_quant_per_tensor -- the same y as sq_ln_smooth_quant, quantised with ONE scale
 * for the whole activation tensor (the coarser per-tensor granularity of "4.2 W8A8…" sec. 7.1
 * and of "量化…PTQ": static per-tensor at the coarse end, dynamic per-token at the fine end):
 *   static_scale = 0 (dynamic): scale = max_{m,j} |y[m, j]| / 127, written to *scale;
 *   static_scale = 1 (static, calibrated): *scale is read (positive, finite);
 *   xq[m, j] = clamp(rne(y[m, j] / scale), -127, 127) -- values beyond a static scale saturate;
 *   sx[m] = scale for every row, so sq_w8a8_gemm applies it unchanged.
 *   scale: one fp32 in device memory.  Other arguments as for sq_ln_smooth_quant.  The
 *   dynamic form makes two passes over x (statistics, then codes) and uses sx as scratch
 *   in between. */
sq_status sq_ln_smooth_quant_per_tensor(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                        const float* gamma_f, const float* beta_f, const float* s, float eps,
                                        int static_scale, float* scale, int8_t* xq, float* sx, void* stream);

/* sq_w8a8_gemm -- INT8 x INT8 -> int32 GEMM on the tcgen05 tensor cores with the dequant
 * epilogue ("4.2 W8A8…" intro: the GEMM runs on INT8 tensor cores; "量化…PTQ": per-token
 * and per-channel scales are multiplied back after the GEMM):
 *   acc[m, n] = sum_j xq[m, j] * wq[n, j]   (exact int32)
 *   ydt = SQ_BF16: y[m, n] = bf16_rne(((float)acc[m, n] * sx[m]) * sw[n])
 *   ydt = SQ_F32:  y[m, n] = ((float)acc[m, n] * sx[m]) * sw[n]
 *   ydt = SQ_I32:  y[m, n] = acc[m, n]            (sx, sw may then be NULL)
 *   xq: int8 [M, K] dense; wq: int8 [N, K] dense; both 16-byte aligned; K % 16 == 0,
 *   K <= SQ_MAX_K.  y: [M, N] with leading dimension ldy >= N, aligned to its element
 *   size (16-byte aligned rows take the vectorised store path).  M == 0 or N == 0 is a
 *   no-op; K == 0 is invalid.
 *   workspace: device scratch of at least sq_w8a8_gemm_workspace_size(M, N, K) bytes
 *   (may be NULL when that size is 0), 256-byte aligned.  Zero-fill it once before its first
 *   use (cudaMemset, torch.zeros): it holds sums of the split work that must start at zero,
 *   and every call leaves all of it zero-filled again, so one
 *   workspace serves any number of calls and shapes (and the FP8 GEMM) without clearing.  (A
 *   call whose kernel stopped on a bounded wait -- sq_device_error() != 0 -- may leave it
 *   dirty: zero it again.)  Calls that share a workspace must be ordered on one stream.
 *   For M > 128 with many output tiles the workspace is optional: it lets the last, short
 *   wave of tiles be split along K over all SMs (summed by a second kernel); with a smaller
 *   or NULL workspace those tiles run whole, with the same result. */
sq_status sq_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                       int64_t M, int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy,
                       void* workspace, size_t ws_bytes, void* stream);

/* sq_w8a8_gemm_rowmax -- sq_w8a8_gemm whose epilogue also emits the per-row max of the output,
 * for a linear whose output is the next linear's input ("4.2 W8A8 量化与 SmoothQuant", sec. 6:
 * the input of a linear comes from a LayerNorm or from the previous GEMM's output, and the
 * smoothing folds into that previous layer; "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section).
 * With the next linear's factors folded into sw (sq_fold_next_smoothing), y is already the next
 * linear's smoothed input, and
 *   rowmax[m] = max_n |y[m, n]|  over the values as stored (bf16-rounded for SQ_BF16),
 * which is exactly the statistic the next per-token quantiser would compute by reading y;
 * sq_quant_codes then finishes the quantisation in one read of y.
 *   Arguments as for sq_w8a8_gemm except: ydt is SQ_BF16 or SQ_F32; rowmax: fp32 [M] device
 *   array, 4-byte aligned, overwritten (the call zero-fills it before the GEMM runs). */
sq_status sq_w8a8_gemm_rowmax(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                              int64_t M, int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy,
                              float* rowmax, void* workspace, size_t ws_bytes, void* stream);

/* sq_quant_codes -- the codes pass of the per-token quantiser for rows whose max is known
 * (from sq_w8a8_gemm_rowmax): sx[m] = rowmax[m] / 127 (binary32, correctly rounded);
 * xq[m, j] = clamp(rne(x[m, j] / sx[m]), -127, 127) (a zero max gives zero codes).  With rowmax
 * the row maxima of x this equals sq_ln_smooth_quant(x, plain mode, s = 1) bit for bit, with
 * one read of x ("SmoothQuant大模型平滑量化技术", Python demo: max/127, round, clip).
 *   x: [M, K] bf16/fp32, ldx (16-byte aligned rows); rowmax: fp32 [M]; xq: int8 [M, K] dense,
 *   16-byte aligned; sx: fp32 [M].  K % 16 == 0 (no upper limit: rows are not held on chip). */
sq_status sq_quant_codes(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* rowmax,
                         int8_t* xq, float* sx, void* stream);

/* Workspace bytes sq_w8a8_gemm needs for this shape on the current device (0 when the
 * launch it picks does not split K).  Returns (size_t)-1 for invalid sizes. */
size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/* Size of the scratch array behind sq_w8a8_gemm_noalloc (16 MiB). */
#define SQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/* sq_w8a8_gemm_noalloc -- sq_w8a8_gemm for callers that cannot allocate device memory.
 *   The pages have no counterpart: this is a library convenience.  Some callers must not
 *   call cudaMalloc: a plug-in inside a host program that owns all device memory through
 *   its own pool (an allocation would fail or break that program's accounting), or a
 *   latency-critical loop where cudaMalloc may synchronise the device.  This variant takes
 *   no workspace: when the launch splits K, its int32 partial sums go to a scratch array of
 *   SQ_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that loads the
 *   library holds until the process exits.  The caller still passes all inputs and
 *   outputs, with the same meaning, layout and checks as sq_w8a8_gemm.
 *   - The arguments are checked first, in the order sq_w8a8_gemm checks them; then a shape
 *     whose required workspace exceeds the scratch returns SQ_ERR_WORKSPACE with nothing
 *     launched.  The required workspace is sq_w8a8_gemm_workspace_size's, except for large
 *     CTA-pair shapes, whose optional split tail (see sq_w8a8_gemm) this entry point does
 *     not use: they run with no scratch at all.
 *   - The first call on a device looks up the scratch array's device address (set-up, once
 *     per device, with that device current); make that first call before any stream
 *     capture.  A failed look-up returns SQ_ERR_CUDA.
 *   - Every call on a device shares the one array, which keeps the last call's contents.
 *     The set-up zero-fills it once (the split-work sums must start at zero, see
 *     sq_w8a8_gemm); every call leaves it zero-filled again.  Calls that overlap on the GPU
 *     (different streams, no ordering) race on it. */
sq_status sq_w8a8_gemm_noalloc(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                               int64_t M, int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy,
                               void* stream);

/* sq_alpha_search -- migration strength by grid search on calibration data ("4.2 W8A8…"
 * sec. 5.2: alpha is chosen once, offline, by a grid search over calibration samples;
 * "量化…PTQ", AWQ paragraph: the data-only objective || Q(W diag(s)) (diag(s)^-1 X) - W X ||).
 * For each alphas[i] the W8A8 layer of this library runs on the calibration batch x:
 *   ax = absmax of the layer input (LN(x; gamma, beta) when gamma is given, else x; as
 *   sq_calib_ln_absmax / sq_calib_absmax), aw = weight row absmax, s = sq_smooth_factors(alpha),
 *   the fold (gamma' = gamma / s), the per-token quantiser and the GEMM with the binary32
 *   epilogue Y_hat = ((float)acc * sx) * sw;
 *   err[i] = ||Y_hat - Y||_F^2 / ||Y||_F^2 with Y = X_in W accumulated in binary32 (k in
 *   increasing order) from binary32 X_in (the LayerNorm output) and W.
 *   x: [M, K] bf16/fp32 (ldx); gamma, beta: the layer's LayerNorm (both NULL: no LayerNorm;
 *   beta may be NULL); W: [K, N] bf16/fp32 (ldw), row j = input channel j.  Constraints as
 *   for the steps above (K % 16 == 0, 16-byte aligned rows).
 *   alphas: HOST array of n_alpha values in [0, 1], 1 <= n_alpha <= 256.
 *   err: DEVICE array of n_alpha doubles (8-byte aligned), written asynchronously.
 *   workspace: device scratch of sq_alpha_search_workspace_size(M, K, N) bytes, 256-byte
 *   aligned, owned by the caller; calls sharing it must be ordered on one stream.
 *   Errors: a step's own status (nothing is rolled back; err is then undefined). */
sq_status sq_alpha_search(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx,
                          const float* gamma, const float* beta, float eps,
                          const void* W, sq_dtype wdt, int64_t N, int64_t ldw,
                          const float* alphas, int n_alpha, double* err,
                          void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes of sq_alpha_search for these sizes ((size_t)-1 for invalid sizes). */
size_t sq_alpha_search_workspace_size(int64_t M, int64_t K, int64_t N);

/* ------------------------------------------------------------------------------------------
 * FP8 variant.  "量化：只压权重，与训练后量化（PTQ）" (decode roofline: W8A8 in FP8 runs on tensor
 * cores with twice the BF16 peak) and "4.2 W8A8 量化与 SmoothQuant" (closing questions: FP8 as
 * the 8-bit format) name FP8 W8A8 without fixing the encoding.  The library reads it as E4M3
 * of the OCP 8-bit floating point specification (OFP8): sign, 4 exponent bits (bias 7),
 * 3 mantissa bits, no infinities, 0x7F / 0xFF = NaN, largest finite 448.  The scheme is the
 * INT8 one with 448 in place of 127: scale = max|.| / 448 (binary32, correctly rounded) and
 * code = E4M3(RN(v / scale)), round to nearest even, saturating at +-448; a zero scale gives
 * +0 codes.  Codes are stored as uint8_t bit patterns.
 * ------------------------------------------------------------------------------------------ */

/* sq_fold_quant_weights_fp8 -- sq_fold_quant_weights with E4M3 weights:
 *   sw[k] = max_j |W'[j, k]| / 448;  Wq[k, j] = E4M3(RN(W'[j, k] / sw[k])).
 *   Every argument has the meaning, layout, ownership and checks of sq_fold_quant_weights
 *   (Wq: uint8 [N, K], K contiguous, 16-byte aligned). */
sq_status sq_fold_quant_weights_fp8(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw,
                                    const float* s, const float* gamma, const float* beta,
                                    uint8_t* Wq, float* sw, float* gamma_f, float* beta_f, void* stream);

/* sq_ln_smooth_quant_fp8 -- sq_ln_smooth_quant with per-token E4M3 codes:
 *   sx[m] = max_j |y[m, j]| / 448;  xq[m, j] = E4M3(RN(y[m, j] / sx[m])).
 *   y, the two modes and every argument as for sq_ln_smooth_quant (xq: uint8 [M, K]). */
sq_status sq_ln_smooth_quant_fp8(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                 const float* gamma_f, const float* beta_f, const float* s, float eps,
                                 uint8_t* xq, float* sx, void* stream);

/* sq_w8a8_gemm_fp8 -- E4M3 x E4M3 GEMM on the tcgen05 tensor cores (kind::f8f6f4) with the
 * same dequant epilogue:
 *   acc[m, n] = sum_j dec(xq[m, j]) dec(wq[n, j])   accumulated in binary32 by the tensor
 *              cores (every product is exact; the order and rounding of the sum are the
 *              hardware's, so acc is within the binary32 summation error bound of the exact
 *              sum, not bit-identical to it)
 *   ydt = SQ_BF16: y[m, n] = bf16_rne((acc[m, n] * sx[m]) * sw[n]);  SQ_F32: the same in fp32.
 *   SQ_I32 is invalid.  Operands, leading dimension, alignment, K limit and workspace as for
 *   sq_w8a8_gemm; the workspace size is sq_w8a8_gemm_workspace_size(M, N, K) (fp32
 *   partials, summed in split order). */
sq_status sq_w8a8_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                           int64_t M, int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy,
                           void* workspace, size_t ws_bytes, void* stream);

/* Reads (and with clear != 0 resets) the device-side error word of the current device:
 * 0 when no kernel gave up on a bounded wait.  Synchronises `stream`.  Bits: 1, 2, 4 -- a GEMM
 * wait (producer, tensor-core issue, epilogue); 8 -- a weight-fold copy; 16 -- an activation-row
 * copy.  A kernel whose wait runs out stops at once: it lets the copies it has already issued
 * land (each within 100 ms), takes no further work and leaves; its outputs are then undefined. */
sq_status sq_device_error(unsigned int* code, int clear, void* stream);

/* sq_selfcheck_shared_divisor -- checks, on the device, the division every quantiser and the
 * weight fold use for code = rne(v / scale) ("SmoothQuant大模型平滑量化技术", Python demo: the code
 * is the rounded quotient, so the quotient must be the correctly rounded one).  The kernels
 * divide all elements of a row (column) by one shared scale through one correctly rounded
 * reciprocal and Markstein's correction step; this call evaluates that routine, in its scalar
 * and its packed-pair form, on every pair (a[j], b[i]) and compares the bits with IEEE
 * round-to-nearest division:
 *   counts[0] += pairs where the scalar form differs, counts[1] += where the packed form
 *   differs, counts[2] += pairs checked (zero divisors are skipped: a zero scale means
 *   "all codes 0" and has no quotient).
 *   a: fp32 [na] dividends, na even, 2 <= na <= 4096; b: fp32 [nb] divisors; q: NULL or fp32
 *   [nb, na], the scalar form's quotients (q[i * na + j] = a[j] / b[i]); counts: 3 device
 *   uint64, 8-byte aligned, accumulated into (zero them first).  All device pointers. */
sq_status sq_selfcheck_shared_divisor(const float* a, int64_t na, const float* b, int64_t nb, float* q,
                                      unsigned long long* counts, void* stream);

/* sq_set_wait_limit -- the limit of every bounded wait in this library's kernels on the
 * current device (default 10 s; the setting outlasts the call, for this process only).  A
 * diagnostic: 0 makes every wait run out at once, so that a test can drive each kernel's
 * give-up path (error bit, drain, early exit) without a GPU fault.  Synchronises `stream`.
 * The pages have no counterpart. */
sq_status sq_set_wait_limit(unsigned long long ns, void* stream);

/* Human-readable name of a status. */
const char* sq_status_string(sq_status status);

/* ABI version of this header (major * 100 + minor). */
int sq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQ_W8A8_H */
