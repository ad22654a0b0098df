/*
 * fp8amax.h — C ABI of the B200 (sm_100a) FP8-AMAX scaled linear layer.
 *
 * The method (review page "Training and inference of large language models
 * using 8-bit floating point", Perez, Zhang et al., section "Proposed method"):
 * for every weight, activation and gradient tensor take the per-tensor maximum
 * absolute value (amax); derive an exponent bias from log2 of the ratio of the
 * FP8 format's largest value to that amax, less a configurable margin
 * (compute_bias); multiply the tensor by 2^bias before casting it to FP8
 * (E4M3 for weights and activations, E5M2 for gradients); run the matmul on
 * the FP8 operands and multiply its output by 2^-(biasA + biasB).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument except `stream` is a DEVICE pointer into memory the
 *     caller owns (cudaMalloc / a framework allocator).  The library allocates
 *     nothing and keeps no per-call state; scalars (amax, bias) stay on the
 *     device, so a whole forward + backward step runs without a host sync.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call only enqueues work on it and returns; outputs are
 *     valid once the stream reaches that point.
 *   - Tensors are dense and row-major.  Data pointers must be 16-byte aligned
 *     (FP8_ERR_MISALIGNED otherwise).
 *   - Argument errors are reported synchronously through the return value and
 *     nothing is launched.  A failed launch returns FP8_ERR_CUDA.  Errors that
 *     happen while a kernel runs surface at the caller's next stream sync, as
 *     for any CUDA call.  No entry point aborts, traps or prints.
 *   - Calls are thread-safe; calls on different streams may overlap.
 *   - FP8 tensors are arrays of uint8_t codes in the OCP E4M3 / E5M2 encodings.
 */
#ifndef FP8AMAX_H_
#define FP8AMAX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8_OK = 0,
    FP8_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative or overflowing size, bad enum  */
    FP8_ERR_UNSUPPORTED = 2,      /* a shape this library does not handle (see each call) */
    FP8_ERR_MISALIGNED = 3,       /* a data pointer that is not 16-byte aligned           */
    FP8_ERR_CUDA = 4,             /* a CUDA runtime / driver call or launch failed        */
    FP8_ERR_TIMEOUT = 5,          /* a kernel's bounded wait ran out (see fp8_device_error) */
    FP8_ERR_NO_DEVICE = 6         /* no usable sm_100 device is current                   */
} fp8_status_t;

typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_format_t;     /* FP8_E4 / FP8_E5 of the page */
typedef enum { FP8_DTYPE_BF16 = 0, FP8_DTYPE_FP32 = 1 } fp8_dtype_t;
typedef enum { FP8_PASS_FWD = 0, FP8_PASS_DGRAD = 1, FP8_PASS_WGRAD = 2 } fp8_pass_t;

/*
 * Step 1 — per-tensor amax ("Proposed method": maximum absolute value of the
 * whole tensor).
 *   x        [n] elements of type dt (BF16 or FP32), device, 16-byte aligned.
 *   amax     one float, device: receives max_i |x_i| (an exact fp32 value).
 *            Any NaN in x gives a NaN; otherwise an inf gives +inf; n == 0
 *            gives 0.  The call initialises *amax itself (stream-ordered).
 * One 128-bit-load reduction kernel plus a 4-byte memset.
 */
fp8_status_t fp8_amax(const void *x, fp8_dtype_t dt, size_t n, float *amax, void *stream);

/*
 * Step 2 — compute_bias ("Proposed method": log2 of the format maximum over the
 * tensor amax, with a configurable margin).
 *   amax     one float, device (as written by fp8_amax).
 *   bias     one int32, device: receives floor(log2(fmt_max / amax)) - margin,
 *            fmt_max = 448 (E4M3) or 57344 (E5M2), computed exactly from the
 *            bits of amax.  amax == 0, inf or NaN gives 0 whatever the margin.
 *   margin   any int32; larger margins leave more headroom below fmt_max.
 */
fp8_status_t fp8_compute_bias(const float *amax, fp8_format_t fmt, int32_t margin,
                              int32_t *bias, void *stream);

/*
 * Step 3 — scale, then cast ("Proposed method": the input is scaled before the
 * conversion to FP8).
 *   out[i] = RNE_satfinite_fmt(x[i] * 2^bias): round to nearest, ties to even,
 *   FP8 subnormals kept, finite overflow (and +-inf) saturates to +-fmt_max,
 *   NaN stays NaN, the sign of zero is kept.  The power-of-two scale is exact.
 *   x        [n] elements of type dt, device, 16-byte aligned.
 *   bias     one int32, device (as written by fp8_compute_bias, or any value).
 *   out      [n] uint8 FP8 codes, device, 16-byte aligned, may not alias x.
 */
fp8_status_t fp8_cast_scaled(const void *x, fp8_dtype_t dt, size_t n, const int32_t *bias,
                             fp8_format_t fmt, uint8_t *out, void *stream);

/*
 * Steps 1-3 in one call: amax, then bias, then the scaled cast, all on the
 * device (two kernels and a 4-byte memset).  Same arguments and results as
 * calling fp8_amax, fp8_compute_bias and fp8_cast_scaled in turn; amax and bias
 * are written for the caller to keep or log (the page's per-tensor scale
 * statistics).
 */
fp8_status_t fp8_quantize(const void *x, fp8_dtype_t dt, size_t n, fp8_format_t fmt,
                          int32_t margin, float *amax, int32_t *bias, uint8_t *out,
                          void *stream);

/*
 * Step 4 — the FP8 matmuls with the unscale ("Proposed method": matmul on the
 * scaled FP8 operands, output multiplied back after it).  fp32 accumulation on
 * the tensor cores (tcgen05, kind::f8f6f4); the epilogue multiplies by
 * 2^-(bias_a + bias_b) and rounds once (RNE) to the output type.
 *
 * Shapes: T tokens, a linear layer [in -> out].  All row-major:
 *   X [T, in], W [out, in], dY [T, out], Y [T, out], dX [T, in], dW [out, in].
 * Requirements: T >= 0; in and out positive multiples of 16 (FP8_ERR_UNSUPPORTED
 * otherwise); every pointer 16-byte aligned; formats E4M3 or E5M2 (any mix).
 * Outputs are dense and may not alias the inputs.  T == 0 leaves Y / dX empty
 * and writes dW = 0.
 */

/* Y = (X8 . W8^T) * 2^-(bias_x + bias_w) */
fp8_status_t fp8_linear_fwd(const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                            const uint8_t *w8, fp8_format_t fw, const int32_t *bias_w,
                            int64_t T, int64_t in, int64_t out,
                            void *y, fp8_dtype_t y_dtype, void *stream);

/* dX = (dY8 . W8) * 2^-(bias_dy + bias_w)   (W8 read in place, not transposed) */
fp8_status_t fp8_linear_bwd_dgrad(const uint8_t *dy8, fp8_format_t fdy, const int32_t *bias_dy,
                                  const uint8_t *w8, fp8_format_t fw, const int32_t *bias_w,
                                  int64_t T, int64_t in, int64_t out,
                                  void *dx, fp8_dtype_t dx_dtype, void *stream);

/* dW = (dY8^T . X8) * 2^-(bias_dy + bias_x)   (dY8 and X8 read in place) */
fp8_status_t fp8_linear_bwd_wgrad(const uint8_t *dy8, fp8_format_t fdy, const int32_t *bias_dy,
                                  const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                                  int64_t T, int64_t in, int64_t out,
                                  void *dw, fp8_dtype_t dw_dtype, void *stream);

/*
 * fwd and dgrad with the amax of their output fused into the GEMM epilogue
 * (the output of one linear is the input of the next, whose FP8-AMAX cast
 * needs that amax).  Same results in y / dx as fp8_linear_fwd /
 * fp8_linear_bwd_dgrad; in addition *y_amax / *dx_amax (one float, device,
 * 4-byte aligned) receives max |value| over the output exactly as stored
 * (after its rounding to BF16/FP32), with fp8_amax's NaN/inf rules, so it is
 * bit-identical to calling fp8_amax on the output, without reading it back.
 * T == 0 writes 0.
 */
fp8_status_t fp8_linear_fwd_amax(const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                                 const uint8_t *w8, fp8_format_t fw, const int32_t *bias_w,
                                 int64_t T, int64_t in, int64_t out,
                                 void *y, fp8_dtype_t y_dtype, float *y_amax, void *stream);

fp8_status_t fp8_linear_bwd_dgrad_amax(const uint8_t *dy8, fp8_format_t fdy,
                                       const int32_t *bias_dy, const uint8_t *w8, fp8_format_t fw,
                                       const int32_t *bias_w, int64_t T, int64_t in, int64_t out,
                                       void *dx, fp8_dtype_t dx_dtype, float *dx_amax,
                                       void *stream);

/*
 * fp8_linear_fwd with a split-K workspace.  For few tokens (T <= 128, e.g.
 * decode-sized inference calls) the GEMM streams the weights and one tile per
 * 128 x 256 block of Y leaves SMs idle; for more tokens, outputs with too few
 * 256 x 256 tiles to fill half the GPU.  With a caller-provided workspace a
 * long K dimension is split across more CTAs, each writing an fp32 partial to
 * the workspace; a second kernel on the same stream adds the partials in a
 * fixed order (deterministic) before the unscale and the single rounding.  Results equal fp8_linear_fwd's
 * within the GEMM tolerance (the fp32 summation order differs); shapes that do
 * not split run exactly as fp8_linear_fwd.
 *   fp8_linear_fwd_workspace_size(T, in, out) returns the bytes needed (0
 *   when the problem is not split; then `workspace` may be NULL).  Needs a
 *   current sm_100 device; returns 0 for invalid shapes.
 *   workspace  device memory of at least that many bytes, 256-byte aligned,
 *              owned by the caller; its contents on entry do not matter.
 *              Two calls that share a workspace must not overlap on the GPU.
 * FP8_ERR_INVALID_ARGUMENT when the workspace is too small.
 */
size_t fp8_linear_fwd_workspace_size(int64_t T, int64_t in, int64_t out);

fp8_status_t fp8_linear_fwd_ws(const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                               const uint8_t *w8, fp8_format_t fw, const int32_t *bias_w,
                               int64_t T, int64_t in, int64_t out, void *y, fp8_dtype_t y_dtype,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * fp8_linear_bwd_wgrad with a split-K workspace, for weight gradients whose
 * output [out, in] has too few 256 x 256 tiles to fill the GPU while K = T is
 * long (small layers over many tokens: a 768 x 768 dW over 8192 tokens is 9
 * tiles).  K is split across more CTA pairs, each writing an fp32 partial;
 * a second kernel adds them in a fixed order (deterministic) and runs the
 * epilogue.  Results equal fp8_linear_bwd_wgrad's within the GEMM
 * tolerance; problems that do not split run exactly as fp8_linear_bwd_wgrad.
 * fp8_linear_bwd_wgrad_workspace_size returns the bytes needed (0: no split).
 * Workspace rules as for fp8_linear_fwd_ws.
 */
size_t fp8_linear_bwd_wgrad_workspace_size(int64_t T, int64_t in, int64_t out);

fp8_status_t fp8_linear_bwd_wgrad_ws(const uint8_t *dy8, fp8_format_t fdy, const int32_t *bias_dy,
                                     const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                                     int64_t T, int64_t in, int64_t out, void *dw,
                                     fp8_dtype_t dw_dtype, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * The launch plan of one GEMM pass on the current device, for performance
 * work and for tests that must know which kernel shape ran.  The paper has no
 * counterpart.  Nothing is launched and no data pointer is involved.
 *   pass            FP8_PASS_FWD (Y = X.W^T, M = T, N = out, K = in),
 *                   FP8_PASS_DGRAD (dX = dY.W, M = T, N = in, K = out) or
 *                   FP8_PASS_WGRAD (dW = dY^T.X, M = out, N = in, K = T).
 *   with_workspace  nonzero: the plan of fp8_linear_fwd_ws / _bwd_wgrad_ws
 *                   given the workspace their size query asks for (ignored
 *                   for DGRAD, which has no such entry point).
 *   plan            out: output tile rows and columns, CTAs that compute one
 *                   tile (1, or 2 for a CTA pair) and the number of ranges
 *                   K is split into (1: not split).
 * Returns FP8_ERR_INVALID_ARGUMENT for a null plan, a negative size or an
 * unknown pass, FP8_ERR_NO_DEVICE without an sm_100 device.
 */
typedef struct {
    int32_t tile_m, tile_n, ctas_per_tile, k_splits;
} fp8_gemm_plan_t;

fp8_status_t fp8_linear_plan(fp8_pass_t pass, int64_t T, int64_t in, int64_t out,
                             int with_workspace, fp8_gemm_plan_t *plan);

/*
 * fp8_linear_fwd_ws for callers that cannot allocate device memory when they
 * run a forward (an allocator that must not be entered there, a fixed memory
 * pool, a serving loop that forbids allocation, a C program with no device
 * allocator).  The paper has no counterpart: this is a packaging of the same
 * forward.  Same arguments and results as fp8_linear_fwd_ws without the
 * workspace: the split-K scratch is a 16 MiB array inside the library that
 * every GPU which loads the library holds until the process exits.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Nothing is allocated, by this call or below it.
 *   - A problem with T <= 64 whose split-K scratch would exceed 16 MiB (very
 *     wide outputs) returns FP8_ERR_UNSUPPORTED; for T > 64 a split whose
 *     partials would not fit is not made and the forward runs unsplit;
 *     problems that do not split use no scratch at all.
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (different streams, no ordering between
 *     them) race on it and must be serialised by the caller.
 */
fp8_status_t fp8_linear_fwd_noalloc(const uint8_t *x8, fp8_format_t fx, const int32_t *bias_x,
                                    const uint8_t *w8, fp8_format_t fw, const int32_t *bias_w,
                                    int64_t T, int64_t in, int64_t out,
                                    void *y, fp8_dtype_t y_dtype, void *stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *fp8_status_string(fp8_status_t status);

/*
 * Every spin-wait inside the library's kernels is bounded in time.  A wait
 * that runs out makes the kernel record a code in a device-side error word,
 * drain its own asynchronous copies and tensor-core work, free its tensor
 * memory and return, leaving the CUDA context usable.  This call synchronises
 * the current device, reads that word (FP8_OK or FP8_ERR_TIMEOUT), and clears
 * it when `clear` is non-zero.  `where` (may be NULL) receives the code of the
 * wait that gave up.
 */
fp8_status_t fp8_device_error(int clear, int32_t *where);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a
 * barrier nothing will ever complete, with a limit of `timeout_ns`
 * (1e6 .. 5e9), and returns what fp8_device_error then reports (FP8_ERR_TIMEOUT
 * when the machinery works).  Clears the error word before returning.
 */
fp8_status_t fp8_selftest_bounded_wait(uint64_t timeout_ns);

/* Version of this ABI: 1. */
int fp8_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8AMAX_H_ */
