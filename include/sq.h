/*
 * sq.h -- C ABI of libsq, the SmoothQuant W8A8 INT8 linear layer for NVIDIA
 * B200 (sm_100a).
 *
 * The layer computes Y[M, N] = X[M, K] W[N, K]^T with both operands in int8:
 *   offline   A_j   = max over calibration tokens of |X_cal[t, j]|
 *             B_j   = max over output channels of |W[n, j]|
 *             s_j   = A_j^alpha / B_j^(1 - alpha)
 *             W'    = W diag(s), quantised per output channel (row n) to int8
 *   online    X^    = X diag(s)^-1, quantised per token (row m) to int8
 *             acc   = Xq Wq^T in int32, Y = (acc * sx[m]) * sw[n]
 * and, around it: RMSNorm with gamma / s folded in and fused with the
 * per-token quantiser (sq_fold_gamma, sq_rmsnorm_quant); the gated SiLU
 * activation of the down projection fused with its quantiser
 * (sq_silu_mul_quant); GPTQ rounding of the weight in place of the plain one
 * (sq_gptq_*).
 *
 * Sources (page title, section):
 *   "Understanding W8A8 INT8 LLM Quantization": "Why Naive Weight Quantization
 *     Doesn't Work, and How GPTQ Fixes It" (per-channel scale max|w|/127 and
 *     round(w/scale)); "Why Activation Quantization Is Hard, and How
 *     SmoothQuant Fixes It" (one dynamic scale per token); "Where the outlier
 *     actually comes from" and "How the smoothing factor is computed"
 *     (calibration absmax per channel, the factor s, dividing the activation
 *     and multiplying the matching weight input channel by s).
 *   "quant_llm_int8": "The architecture: every piece explained" and "End-to-end
 *     flow" (int8 matmul accumulating in int32, dequantised by the outer
 *     product of per-row activation scales and per-column weight scales).
 *   "How does SmoothQuant int8 LLM calibration work...": "The Technical
 *     Workflow for Int8 Quantization Deployment" (absmax per channel over
 *     calibration samples; alpha between 0 and 1).
 *   The sources of the fused and offline extras are cited at each of them.
 *
 * Numerics (every entry point; GPTQ and the gated activation's e^x state
 * their own sequences of fused multiply-adds): fp32 IEEE arithmetic,
 * round-to-nearest-even,
 * no fused multiply-add in any step whose result is rounded; codes are
 * clamp(round_half_even(v / scale), -127, 127) (-128 is never produced); a
 * zero absolute maximum gives scale 0 and all-zero codes; s_j is evaluated in
 * fp64 and rounded once to fp32, and is 1 where A_j or B_j is 0.  Inputs must
 * be finite.  Results are bit-identical to the plain CPU definition, except
 * that s_j may differ in its last bit where the fp64 quotient lies within a
 * few fp64 ulps of an fp32 rounding midpoint (libm and CUDA pow differ by up
 * to 2 fp64 ulps).
 *
 * Conventions (every entry point):
 *   - Every pointer is a DEVICE pointer owned by the caller; the library never
 *     allocates or frees caller memory.  Buffers must not alias unless stated.
 *   - Every pointer must be 16-byte aligned.
 *   - Matrices are row-major; X is [rows, K] (K contiguous), W is [N, K]
 *     (output channels x input channels, K contiguous), Y is [M, N].
 *   - K and N must be multiples of 16; M, T >= 1.
 *   - All work is enqueued on `stream` (0 = legacy default stream) and is
 *     asynchronous; results are valid once the stream has been synchronised.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and return SQ_ERR_INVALID_ARG (or SQ_ERR_UNSUPPORTED for sizes beyond a
 *     stated limit); a failed launch returns SQ_ERR_CUDA.  No C++ exception
 *     crosses this interface.
 *   - Kernels that wait on on-chip barriers give up after about two seconds,
 *     record an error word on the device and return; sq_device_status()
 *     reports it as SQ_ERR_TIMEOUT.  No kernel traps.
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sq_stream_t; /* identical to cudaStream_t */

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,
    SQ_ERR_UNSUPPORTED = 2,
    SQ_ERR_CUDA = 3,
    SQ_ERR_TIMEOUT = 4
} sq_status;

typedef enum {
    SQ_F32 = 0, /* IEEE binary32 */
    SQ_BF16 = 1 /* bfloat16, 16-bit pattern */
} sq_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
SQ_API const char *sq_status_string(sq_status st);

/* Library version as 10000*major + 100*minor + patch. */
SQ_API int sq_version(void);

/*
 * Calibration statistics ("How the smoothing factor is computed": A_j is the
 * largest activation magnitude seen in channel j over calibration samples).
 *   x    [T, K] of dtype dt, row stride ldx elements (ldx >= K, and ldx times
 *        the element size a multiple of 16 bytes).
 *   ax   [K] fp32, ACCUMULATED: ax[j] = max(ax[j], max_t |x[t, j]|).  The
 *        caller zero-fills ax before the first batch of a calibration run and
 *        may then call this once per calibration batch.
 * Errors: SQ_ERR_INVALID_ARG for NULL/misaligned pointers, T < 1, K < 16,
 * K % 16 != 0, bad ldx or dt.
 */
SQ_API sq_status sq_calib_absmax(const void *x, sq_dtype dt, int64_t T, int64_t K, int64_t ldx,
                          float *ax, sq_stream_t stream);

/*
 * Smoothing factors ("How the smoothing factor is computed"):
 *   B_j = max_n |w[n, j]|,  s_j = A_j^alpha / B_j^(1-alpha) (fp64, rounded
 *   once to fp32; s_j = 1 where A_j == 0 or B_j == 0).
 *   ax   [K] fp32 calibration absmax (from sq_calib_absmax).
 *   w    [N, K] of dtype dt (the unsmoothed weight).
 *   alpha in [0, 1] (migration strength), finite.
 *   s    [K] fp32 output.
 *   aw   [K] fp32 output with B_j, or NULL.  s and aw must not alias ax.
 * Errors: as above, plus alpha outside [0, 1].
 */
SQ_API sq_status sq_smooth_factors(const float *ax, const void *w, sq_dtype dt, int64_t N, int64_t K,
                            float alpha, float *s, float *aw, sq_stream_t stream);

/*
 * Smoothed per-output-channel weight quantisation ("Where the outlier actually
 * comes from": multiply the matching weight input channel by s; "Why Naive
 * Weight Quantization Doesn't Work": scale = max|w'|/127, q = round(w'/scale)):
 *   w'[n, k] = w[n, k] * s[k];  sw[n] = max_k |w'[n, k]| / 127;
 *   wq[n, k] = clamp(round(w'[n, k] / sw[n]), -127, 127).
 *   w [N, K] dtype dt; s [K] fp32; wq [N, K] int8 out; sw [N] fp32 out.
 * K is at most 65536 (bf16) or 32768 (fp32); larger K is SQ_ERR_UNSUPPORTED.
 */
SQ_API sq_status sq_smooth_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K,
                                 const float *s, int8_t *wq, float *sw, sq_stream_t stream);

/*
 * Dynamic per-token activation quantisation ("Why Activation Quantization Is
 * Hard": one scale per token over all channels, computed at run time), of the
 * smoothed activation:
 *   x^[m, k] = x[m, k] / s[k];  sx[m] = max_k |x^[m, k]| / 127;
 *   xq[m, k] = clamp(round(x^[m, k] / sx[m]), -127, 127).
 *   x [M, K] dtype dt; s [K] fp32; xq [M, K] int8 out; sx [M] fp32 out.
 * K limits as for sq_smooth_quant_weight.
 */
SQ_API sq_status sq_quant_act(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                       int8_t *xq, float *sx, sq_stream_t stream);

/*
 * RMSNorm's gamma with the smoothing factors folded in ("Understanding W8A8
 * INT8 LLM Quantization", section "Where the outlier actually comes from":
 * SmoothQuant divides the norm's gamma by s, so the norm already produces the
 * smoothed activation):  g[j] = gamma[j] / s[j] (one IEEE fp32 division).
 *   gamma [K], s [K], g [K] fp32 device arrays, 16-byte aligned; K a multiple
 *   of 16.  Offline, once per linear.
 */
SQ_API sq_status sq_fold_gamma(const float *gamma, const float *s, int64_t K, float *g,
                               sq_stream_t stream);

/*
 * RMSNorm with the folded gamma, then per-token int8 quantisation, in one
 * pass over the hidden states (same page and section; the per-token scale as
 * in sq_quant_act):
 *   ms[m]   = sum_k h[m, k]^2 / K + eps       (squares exact in fp64, fp64 sum)
 *   rinv[m] = RN_fp32(1 / sqrt(ms[m]))        (IEEE fp64; 0 when ms[m] is 0)
 *   a[m, k] = (h[m, k] * rinv[m]) * g[k]      (two fp32 multiplies)
 *   sx[m]   = max_k |a[m, k]| / 127;  xq[m, k] = clamp(round(a[m, k] / sx[m]), -127, 127)
 *   h [M, K] dtype dt; g [K] fp32 (from sq_fold_gamma); eps >= 0 finite;
 *   xq [M, K] int8 out; sx [M] fp32 out; rinv [M] fp32 out (may be NULL).
 * The order of the fp64 sum is unspecified: when the fp64 value of
 * 1/sqrt(ms) lies at an fp32 rounding midpoint, rinv may round either way.
 * K limits as for sq_smooth_quant_weight.
 */
SQ_API sq_status sq_rmsnorm_quant(const void *h, sq_dtype dt, int64_t M, int64_t K, const float *g,
                                  float eps, int8_t *xq, float *sx, float *rinv, sq_stream_t stream);

/*
 * The gated feed-forward activation of the down projection, quantised in the
 * same pass that computes it, so that it never travels through HBM in bf16
 * ("Understanding W8A8 INT8 LLM Quantization", section "Inter-Token Latency
 * (ITL)": the per-token quantisation is memory-bound work; "How does
 * SmoothQuant int8 LLM calibration work...", section "Hardware Acceleration
 * and Inference Optimization Strategies": fuse the feed-forward network with
 * its neighbours).  The pages do not define the activation; this is the
 * gated SiLU of the Llama layers:
 *   E(x)    = e^x by a fixed fp32 sequence: 0 for x < -87, +inf for x > 88,
 *             else Cody-Waite reduction with RN(log2 e), RN(ln 2) and
 *             RN(ln 2 - RN(ln 2)), then the degree-7 Taylor series by
 *             Horner's rule with fused multiply-adds and coefficients
 *             RN(1/k!), times 2^n (within 1 ulp of e^x);
 *   h[m, j] = RN(RN(g / RN(1 + E(-g))) * u), g = gu[m, j], u = gu[m, I + j],
 *             rounded to dt (bf16 by round-half-to-even): the value an
 *             unfused feed-forward step would store;
 *   then exactly sq_quant_act on h: sx[m] = max_j |h / s_j| / 127, codes.
 *   gu [M, 2I] dtype dt (each row: the I gate values, then the I up values);
 *   s [I] fp32; xq [M, I] int8 out; sx [M] fp32 out; h [M, I] dtype dt out
 *   (may be NULL: then h is not stored).
 * I a multiple of 16, at most 32768 (bf16) or 16384 (fp32).  Inputs must be
 * finite, and so must h (|SiLU(gate) * up| within dt's range).
 */
SQ_API sq_status sq_silu_mul_quant(const void *gu, sq_dtype dt, int64_t M, int64_t I, const float *s,
                                   int8_t *xq, float *sx, void *h, sq_stream_t stream);

/*
 * GPTQ weight rounding, offline, in place of sq_smooth_quant_weight's plain
 * rounding ("Understanding W8A8 INT8 LLM Quantization", section "How GPTQ
 * improves on naive quantization": quantise a channel's weights one at a
 * time and push each rounding error onto the channel's not yet quantised
 * weights, weighted by the Hessian from the calibration activations).  Three
 * calls, each a fixed sequence of IEEE fp64 operations in a fixed order (so
 * the results do not depend on the thread layout):
 *
 * sq_gptq_hessian: H[i][j] = sum over tokens t (ascending) of
 *   xh[t][i] * xh[t][j], one fp64 FMA a term, with xh = RN_f32(x / s) (the
 *   smoothed activation, as in sq_quant_act).  x [T, K] dtype dt (calibration
 *   tokens); s [K]; H [K, K] fp64 out (overwritten; symmetric).
 *
 * sq_gptq_factor: damps H in place, H[i][i] += d with d =
 *   RN(RN(sum_i H[i][i] / K) * damp_frac) (the sum in index order; d = 1 when
 *   the sum is 0), then writes U [K, K] fp64, the upper Cholesky factor of
 *   H^-1 (zero below the diagonal), through U = J L^-1 J: J reverses the
 *   index order and L is the lower Cholesky factor of J H J, computed column
 *   by column; L^-1 by forward
 *   substitution, row by row, the same way.  Every dot product there is 32
 *   interleaved partial sums (partial l over the terms l, l + 32, ... from
 *   the first, ascending, one FMA a term) combined by the xor butterfly over
 *   offsets 16, 8, 4, 2, 1.  workspace: device scratch of at least
 *   sq_gptq_workspace_size(K) bytes (2 K * K fp64).  A non-positive pivot
 *   leaves U NaN and sets the device error word (sq_device_status returns
 *   SQ_ERR_INVALID_ARG).  Takes K + 3 kernel launches.
 *
 * sq_gptq_quant_weight: per output channel n, w = RN_f32(W[n] * s) widened to
 *   fp64 and sw[n] = RN_f32(max |w| / 127) (sq_smooth_quant_weight's scale);
 *   then for k = 0 .. K-1 in order: q = clamp(rint(w[k] / sw[n]), -127, 127)
 *   (fp64, half to even), e = fma(-q, sw[n], w[k]) / U[k][k], and
 *   w[j] = fma(-e, U[k][j], w[j]) for every j > k.  w [N, K] dtype dt;
 *   s [K]; U from sq_gptq_factor; wq [N, K] int8 out; sw [N] fp32 out.
 *
 * K a multiple of 16, at most 16384.
 */
SQ_API size_t sq_gptq_workspace_size(int64_t K);
SQ_API sq_status sq_gptq_hessian(const void *x, sq_dtype dt, int64_t T, int64_t K, const float *s,
                                 double *H, sq_stream_t stream);
SQ_API sq_status sq_gptq_factor(double *H, int64_t K, float damp_frac, double *U, void *workspace,
                                size_t ws_bytes, sq_stream_t stream);
SQ_API sq_status sq_gptq_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s,
                                      const double *U, int8_t *wq, float *sw, sq_stream_t stream);

/*
 * W8A8 GEMM with the dequantising epilogue ("quant_llm_int8": int32
 * accumulation, outer product of row and column scales):
 *   acc[m, n] = sum_k xq[m, k] * wq[n, k]   (exact int32; K * 127^2 < 2^31,
 *                                            so K <= 133144)
 *   y[m, n]   = ((float)acc[m, n] * sx[m]) * sw[n], stored as out_dt
 *               (SQ_BF16: round-half-to-even of the fp32 value).
 *   xq [M, K] int8, sx [M] fp32, wq [N, K] int8, sw [N] fp32, y [M, N].
 * Runs on the 5th-generation tensor cores (tcgen05, int8 x int8 -> int32 in
 * tensor memory); y must not alias any input.
 */
SQ_API sq_status sq_w8a8_gemm(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                       int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                       sq_stream_t stream);

/*
 * sq_w8a8_gemm with a workspace, which lets the GEMM use every SM whatever the
 * shape ("quant_llm_int8", "The architecture: every piece explained": the
 * same int32 accumulation and outer-product dequantisation):
 *   - up to 128 tokens, the weight is streamed by at most one CTA per SM,
 *     each taking an equal share of the 128-channel x 128-byte weight
 *     blocks; where summing shared blocks would cost more than it saves
 *     (typically from 64 tokens) the CTAs take whole 128-channel blocks
 *     instead (up to 32 tokens on layers whose output channels split into
 *     slabs of 128-256 per SM, every CTA takes whole channels and the
 *     workspace is not touched);
 *   - more tokens: the same tiles as sq_w8a8_gemm; with SQ_GEMM_SK=1 in the
 *     environment the tiles that do not fill whole rounds of the CTA pairs
 *     are split along K over all pairs (off by default: slower on B200).
 *   A tile shared by several CTAs is summed through int32 partials in the
 *   workspace (exact: the result is the same bits as sq_w8a8_gemm's).
 *   workspace: device scratch of at least sq_w8a8_gemm_workspace_size(M, N,
 *   K) bytes, 16-byte aligned, owned by the caller, any contents; calls that
 *   run concurrently need separate workspaces.  A small kernel clears the
 *   workspace's tile counters before a GEMM that uses them.  Errors as
 *   sq_w8a8_gemm, plus SQ_ERR_INVALID_ARG for a missing or too small
 *   workspace.
 */
SQ_API sq_status sq_w8a8_gemm_ws(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                                 int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                                 void *workspace, size_t ws_bytes, sq_stream_t stream);

/* Bytes of workspace sq_w8a8_gemm_ws needs (0 for invalid sizes): for
 * M <= 128, 4 * ceil(N / 128) bytes of tile counters (rounded up to 256) and
 * min(ceil(N / 128) * ceil(K / 128), 160) * 2 * T * 512 bytes of partial sums,
 * T = 32, 64 or 128 the token count rounded up to one of those; for more
 * tokens, 1280 bytes of counters and 40 MiB of partial sums. */
SQ_API size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * The raw int32 accumulators acc[m, n] = sum_k xq[m, k] * wq[n, k] of the same
 * tensor-core kernels (no scales), for verification.  acc is [M, N] int32.
 */
SQ_API sq_status sq_w8a8_gemm_s32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                           int32_t *acc, sq_stream_t stream);

/*
 * The online linear layer: sq_quant_act followed by sq_w8a8_gemm, i.e. the
 * per-layer work that "Understanding W8A8 INT8 LLM Quantization", section
 * "Inter-Token Latency (ITL)", charges to every generated token: find each
 * token's range and scale, cast to int8, multiply in int8, dequantise.
 *   x [M, K] dtype in_dt; s [K]; wq [N, K]; sw [N]; y [M, N] dtype out_dt.
 *   workspace: device scratch, 16-byte aligned, owned by the caller and not
 *   read by the caller afterwards (may be NULL when
 *   sq_linear_workspace_size(M, N, K) is 0); calls that run concurrently
 *   need separate workspaces.  It must hold at least the int8 codes and
 *   scales, M * K + 4 * M bytes (each rounded up to 256); with
 *   sq_linear_workspace_size(M, N, K) bytes it also holds the GEMM's own
 *   workspace, and the GEMM runs as sq_w8a8_gemm_ws (every SM busy whatever
 *   the shape) instead of as sq_w8a8_gemm.
 * Two kernels run back to back (the second launch overlaps the first);
 * the workspace holds the int8 activations and their scales in between, and
 * the GEMM's tile counters and partial sums (the quantiser clears the
 * counters on every call, so the workspace may hold anything beforehand).
 * For M <= 128 the GEMM streams the weight over every SM; its launch and
 * set-up overlap the quantiser.
 * With the environment variable SQ_LINEAR_FUSED=1, up to 32 tokens are
 * instead quantised inside an older cluster split-K GEMM kernel (no
 * workspace; slower on B200).
 */
SQ_API sq_status sq_linear(const void *x, sq_dtype in_dt, const float *s, const int8_t *wq,
                    const float *sw, int64_t M, int64_t N, int64_t K, void *y, sq_dtype out_dt,
                    void *workspace, size_t ws_bytes, sq_stream_t stream);

/* Bytes of workspace sq_linear needs for these sizes to run at its best (0
 * when it needs none): M * K bytes of codes and 4 * M of scales (each
 * rounded up to 256), then sq_w8a8_gemm_workspace_size(M, N, K). */
SQ_API size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * sq_linear without any allocation, for callers that cannot allocate device
 * memory: for example a plugin inside a host framework that owns every device
 * allocation and hands the library only its input and output buffers, or a
 * latency-critical serving loop in which a cudaMalloc (which can synchronise
 * the whole device) is not allowed.  The pages have no counterpart to this
 * entry point; it is a packaging of sq_linear.
 *
 * Same arguments, arithmetic and results as sq_linear, but the workspace is a
 * fixed scratch array that lives in the library itself (a file-scope device
 * array of SQ_LINEAR_NOALLOC_SCRATCH_BYTES bytes, held by every GPU that loads
 * the library until the process exits).  The call makes no cudaMalloc or
 * cudaFree and calls no allocating library routine.
 *   - Sizes whose int8 codes and scales (M * K + 4 * M bytes, each rounded
 *     up to 256) exceed SQ_LINEAR_NOALLOC_SCRATCH_BYTES are rejected with
 *     SQ_ERR_UNSUPPORTED before anything is enqueued.  When the GEMM's own
 *     workspace does not fit next to them, the GEMM runs without one (as
 *     sq_w8a8_gemm).
 *   - The first call on a device (with that device current) looks up the
 *     device address of the scratch array once and keeps it for the process;
 *     make that first call before any stream capture on the device.  The
 *     kept address is not valid after cudaDeviceReset on that device: do not
 *     call this entry point on a device after resetting it.
 *   - All calls on a device share the one scratch array, which keeps the
 *     previous call's contents (nothing in it needs to start at zero).  Calls
 *     that can overlap on the GPU (different streams without ordering between
 *     them) race on it: order them, or use sq_linear with separate workspaces.
 */
#define SQ_LINEAR_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
SQ_API sq_status sq_linear_noalloc(const void *x, sq_dtype in_dt, const float *s,
                                   const int8_t *wq, const float *sw, int64_t M, int64_t N,
                                   int64_t K, void *y, sq_dtype out_dt, sq_stream_t stream);

/*
 * Device error word: synchronises `stream`, then reads and clears the error
 * word the kernels set when a bounded on-chip wait gives up, or when
 * sq_gptq_factor meets a non-positive pivot.  Returns SQ_OK, SQ_ERR_TIMEOUT
 * (a wait gave up), SQ_ERR_INVALID_ARG (code 0xA00: the GPTQ Hessian was not
 * positive definite), with the kernel's location code in *code when code is
 * not NULL, or SQ_ERR_CUDA if the synchronisation itself failed.
 */
SQ_API sq_status sq_device_status(sq_stream_t stream, uint32_t *code);

/*
 * Self-test of the failure detection: enqueues one tiny kernel whose single
 * waiting thread waits on an on-chip barrier that nothing ever arrives on,
 * with a limit of limit_us microseconds (1 .. 2000000).  The wait gives up,
 * records the location code 0x900 in the device error word and the kernel
 * returns, so the context stays usable; sq_device_status then reports
 * SQ_ERR_TIMEOUT with that code.  The pages have no counterpart: this checks
 * the library's own bounded waits.
 */
SQ_API sq_status sq_selftest_wait_timeout(uint32_t limit_us, sq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
