/*
 * sq.h -- C ABI of libsq, the B200 (sm_100a) SmoothQuant W8A8 linear layer.
 *
 * The layer has four parts, each one or two calls below:
 *   (1) per-input-channel calibration statistic max|X_j|       sq_calib_absmax
 *   (2) smoothing factors, offline weight transform + INT8     sq_smooth_scales, sq_quant_weight
 *   (3) runtime smoothing x/s + INT8 activation quantisation   sq_smooth_quant_act, sq_rmsnorm_quant
 *   (4) INT8 x INT8 -> INT32 GEMM with a dequant epilogue       sq_linear_w8a8 (+ fused variants)
 *
 * Sources (the pages this layer is built from):
 *   kwkr.cn blog on SmoothQuant W8A8 ("kwkr"), sections 1.2, 2.1-2.3, 3.1-3.3, 5.2
 *   tbr8.org article on activation outliers ("tbr8"), PyTorch toy example
 *   pwwt.cn "SmoothQuant技术解析：LLM模型INT8无损量化实践" ("pwwt"), 3.1
 *   aiunderstanding.org "SmoothQuant 和激活量化" ("aiu"), technical insight
 *   blog.yoooo.fun "010. SmoothQuant Integration" ("adr-010"), context and key design points
 *
 * Conventions for every call:
 *   - Layouts are row-major.  X is [M, K] (tokens x input channels), W is [N, K]
 *     (output x input channels, the nn.Linear layout), Y = X W^T is [M, N].
 *     "Channel j" is the K index.
 *   - Every pointer is DEVICE memory owned by the caller, unless a parameter
 *     says "host".  The library allocates no device memory; calls that need
 *     scratch take a caller-provided workspace.
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *     NULL is the legacy default stream) on the current CUDA device.  On a
 *     created stream the kernels are launched with programmatic dependent
 *     launch (no gap for launch processing between consecutive kernels); on
 *     the default streams (legacy or per-thread) they are launched plainly.
 *   - Arguments are validated before any launch: null pointers, sizes, 16-byte
 *     alignment where vector or TMA access needs it, dtype support.  A bad
 *     argument returns an error status and launches nothing.  No call aborts,
 *     prints, or throws across the ABI.
 *   - Kernels that wait on on-chip barriers give up after a bounded time and
 *     record SQ_ERR_TIMEOUT in a device-side error word instead of hanging;
 *     sq_sync_status() synchronises a stream and reports (and clears) it.
 *   - Quantised codes are symmetric INT8 in [-127, 127] (zero point 0; -128 is
 *     never produced), rounded half to even.  Scales are fp32.
 *   - Canonical fp32 order (bit-exact contract with the CPU oracle):
 *       recip(v)      = v > 0 ? fl(1/v) : 0
 *       act code      = q(fl(fl(x * recip(s_j)) * recip(a)))
 *       weight code   = q(fl(fl(w * s_j) * recip(w_scale_n)))
 *       absmax scale  = fl(max |value| / 127)
 *       dequant       = fmaf((float)acc, fl(a_m * w_scale_n), bias_n)
 *                       (fl((float)acc * fl(a_m * w_scale_n)) without bias),
 *                       then one rounding to the output dtype.
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size/dtype/mode, alpha outside [0,1] */
    SQ_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement (shape limits) */
    SQ_ERR_MISALIGNED = 3,    /* pointer or leading dimension not 16-byte aligned */
    SQ_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (see sq_last_cuda_error) */
    SQ_ERR_TIMEOUT = 5,       /* a kernel's bounded barrier wait expired */
    SQ_ERR_WORKSPACE = 6      /* workspace missing or smaller than required */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_F16 = 1, SQ_BF16 = 2 } sq_dtype;

typedef enum {
    SQ_ACT_STATIC = 0,        /* one per-tensor scale a (adr-010 context step 3) */
    SQ_ACT_PER_TOKEN = 1      /* one scale per row of X, computed at run time */
} sq_act_mode;

typedef void *sq_stream;      /* cudaStream_t */

/* Human-readable name of a status.  Never NULL. */
const char *sq_status_string(sq_status st);

/* Last CUDA error code (cudaError_t as int) seen by this thread's calls, 0 if none. */
int sq_last_cuda_error(void);

/* Upper bound, in nanoseconds, on any single on-chip barrier wait inside this
 * library's kernels (default 2e9 = 2 s; 0 restores the default).  A wait that
 * runs out records SQ_ERR_TIMEOUT and the kernel returns without hanging. */
void sq_set_wait_timeout_ns(unsigned long long ns);

/* Test hooks (off by default), bit flags of `what`:
 *   1: failure detection.  In every GEMM launched afterwards, the producer
 *      warp of CTA 0 withholds its first pipeline stage (no arrival, no
 *      load), so the MMA warp's bounded wait on that stage runs out: the
 *      kernel records SQ_ERR_TIMEOUT, drains what it had in flight and
 *      returns, and the CUDA context stays usable.  Nothing faults, traps or
 *      hangs.
 *   2: small-M GEMMs run without the cluster split (on the stream-K or
 *      one-tile-per-CTA schedules), so that tests reach those paths.
 *   4: sq_linear_w8a8_noalloc checks its requests against a capacity of
 *      64 KiB of partial sums instead of its whole array, so that tests reach
 *      its rejection of oversize requests.
 * what = 0 turns them off. */
void sq_debug_inject(int what);

/* Synchronises `stream`, then returns SQ_ERR_TIMEOUT if any kernel of this
 * library recorded a barrier timeout on the current device since the last
 * check (and clears the record), SQ_ERR_CUDA if the stream reported an error,
 * else SQ_OK. */
sq_status sq_sync_status(sq_stream stream);

/* -------------------------------------------------------------------------
 * (1) Calibration statistic.  kwkr 3.1: per layer, per channel max of the
 * activations (and of the weights); adr-010 key design point 1: the running
 * per-channel max-abs is the only state calibration keeps (O(K) memory).
 *
 *   absmax[j] = max(absmax[j], max_{r < rows} |x[r * ld + j]|),  j < cols
 *
 * x: [rows, ld] of `dt` (fp32/fp16/bf16), ld >= cols (elements).  absmax:
 * fp32 [cols], read and written (a running max: the caller zeroes it once and
 * calls once per calibration batch).  The same call gives max|W_j| when x is
 * the weight [N, K] (a column max over output rows).  Exact (a max of exactly
 * widened values), so the result does not depend on launch order.  NaN inputs
 * are not supported.  rows == 0 is a no-op.
 * ------------------------------------------------------------------------- */
sq_status sq_calib_absmax(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                          float *absmax, sq_stream stream);

/* -------------------------------------------------------------------------
 * (1b) Robust calibration statistics.  kwkr 3.1: instead of the per-channel
 * max, a high quantile of |X_j| (the page names 99.9 %) or the mean of the
 * maxima of several calibration samples, so that one abnormal token does not
 * set the channel's smoothing factor.  Either result stands in for act_max
 * in sq_smooth_scales unchanged.
 * ------------------------------------------------------------------------- */

/* Nearest-rank p-quantile of |x| per column over all `rows` calibration
 * tokens (the batches laid end to end, or strided with ld):
 *
 *   out[j] = the k-th smallest of |x[t * ld + j]|, t < rows,  k = ceil(p * rows)
 *            (the product in fp64; 1 <= k <= rows)
 *
 * The result is one of the data values, widened exactly to fp32 (p = 1 gives
 * the max).  Found by a radix select on the magnitude bit patterns: 2 passes
 * over x for fp16/bf16, 4 for fp32.  x: [rows, ld] of `dt`, 16-byte aligned,
 * cols * sizeof(dt) and ld * sizeof(dt) multiples of 16 (else
 * SQ_ERR_MISALIGNED).  1 <= rows < 2^32; 0 < p <= 1.  out: fp32 [cols].
 * workspace: sq_calib_quantile_workspace_size(cols) bytes, 16-byte aligned
 * (per-column histograms of 256 bins, prefixes and ranks); no
 * initialisation needed.  NaN inputs are not supported. */
size_t sq_calib_quantile_workspace_size(int64_t cols);
sq_status sq_calib_quantile(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld, double p,
                            float *out, void *workspace, size_t workspace_bytes, sq_stream stream);

/* Mean of per-sample maxima, one calibration batch (sample) per call:
 *
 *   batch max      m_j = max_r |x[r * ld + j]|                (exact, into batch_max)
 *   running sum    sum_max[j] += (double) m_j;  batch_max[j] = 0
 *
 * then sq_calib_mean_of_max gives out[j] = fl32(sum_max[j] / n_batches) (fp64
 * division).  The fp64 sum is taken in call order, one add per batch.
 * batch_max: fp32 [cols], zero before the first call (every call leaves it
 * zero).  sum_max: fp64 [cols], zeroed by the caller before the first batch.
 * rows >= 1. */
sq_status sq_calib_batchmax_accumulate(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                       float *batch_max, double *sum_max, sq_stream stream);
sq_status sq_calib_mean_of_max(const double *sum_max, int64_t cols, int64_t n_batches, float *out,
                               sq_stream stream);

/* -------------------------------------------------------------------------
 * (2a) Smoothing factors.  kwkr 2.2, aiu, adr-010 context step 1:
 *
 *   s_j = max(act_max_j, 1e-5)^alpha / max(w_max_j, 1e-5)^(1 - alpha)
 *
 * evaluated in fp64 and rounded once to fp32 (the clamp at 1e-5 follows tbr8's
 * example).  If a_static != NULL it also receives the closed-form per-tensor
 * activation scale of adr-010 key design point 1:
 *
 *   a_static[0] = fl(max_j fl(act_max_j * recip(s_j)) / 127)
 *
 * act_max, w_max, s: fp32 [K].  a_static: fp32 [1] or NULL.  0 <= alpha <= 1.
 * ------------------------------------------------------------------------- */
sq_status sq_smooth_scales(const float *act_max, const float *w_max, int64_t K, float alpha,
                           float *s, float *a_static, sq_stream stream);

/* -------------------------------------------------------------------------
 * (2b) Offline weight transform and per-output-row INT8 quantisation.
 * kwkr 3.2-3.3 (W' = W diag(s) stored as INT8, one scale per output channel),
 * adr-010 context steps 2-3 (weights per row):
 *
 *   W'[n,j]    = fl(W[n,j] * s_j)
 *   w_scale[n] = fl(max_j |W'[n,j]| / 127)
 *   wq[n,j]    = q(fl(W'[n,j] * recip(w_scale[n])))
 *
 * w: [N, K] of `dt`, contiguous.  s: fp32 [K].  wq: int8 [N, K] (K-major: the
 * GEMM's B operand as is).  w_scale: fp32 [N].  An all-zero row gets scale 0
 * and codes 0.  w and wq 16-byte aligned; K*sizeof(dt) and K multiples of 16
 * bytes are not required (ragged K is handled).
 * ------------------------------------------------------------------------- */
sq_status sq_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s,
                          int8_t *wq, float *w_scale, sq_stream stream);

/* The same transform for a gate/up pair that share one s (both read the same
 * normalised input), written in the interleaved row order that
 * sq_linear_w8a8_gateup_silu consumes: output rows are blocks of 64, block b
 * holding gate rows 32b..32b+31 then up rows 32b..32b+31.
 * w_gate, w_up: [N_h, K] of `dt`.  wq_gu: int8 [2*N_h, K].  w_scale_gu: fp32
 * [2*N_h], same order.  N_h must be a multiple of 32. */
sq_status sq_quant_weight_gateup(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h,
                                 int64_t K, const float *s, int8_t *wq_gu, float *w_scale_gu,
                                 sq_stream stream);

/* Cross-layer folding ("010. SmoothQuant Integration", Alternative C; kwkr
 * 3.2): when the smoothed layer's input is (or depends linearly on) a
 * previous linear's output, 1/s of the smoothed layer moves into that
 * previous layer's output rows, and the runtime x/s step disappears.  These
 * calls transform the PREVIOUS layer's weight with the fold applied first:
 *
 *   W'[n,j] = fl(fl(W[n,j] * recip(s_next_n)) * s_j)     (then per-row INT8 as in sq_quant_weight)
 *
 * s: this layer's own smoothing factors [K]; s_next: the smoothing factors of
 * the next layer's input channels, one per output row n [N].
 * sq_quant_weight_gateup_fold folds only the up rows (h = silu(g) * u is
 * linear in u, so h / s_next = silu(g) * (u / s_next)); s_next is [N_h],
 * indexed by channel; the gate rows are those of sq_quant_weight_gateup.  A
 * gate/up GEMM on folded weights is then called with s2 = NULL (its requant
 * multiplies by recip(a2) only). */
sq_status sq_quant_weight_fold(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s,
                               const float *s_next, int8_t *wq, float *w_scale, sq_stream stream);
sq_status sq_quant_weight_gateup_fold(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h,
                                      int64_t K, const float *s, const float *s_next, int8_t *wq_gu,
                                      float *w_scale_gu, sq_stream stream);

/* -------------------------------------------------------------------------
 * (3a) Runtime smoothing + INT8 activation quantisation.  The 1/s scaling
 * happens strictly before quantisation (kwkr 3.2 and 5.2):
 *
 *   x'[m,j] = fl(x[m,j] * recip(s_j))
 *   static:    a = a_scale[0] (read);                       xq = q(fl(x' * recip(a)))
 *   per-token: a_scale[m] = fl(max_j |x'[m,j]| / 127) (written); xq = q(fl(x' * recip(a_scale[m])))
 *
 * x: [M, K] of `dt`, contiguous, 16-byte aligned.  s: fp32 [K].  a_scale: fp32
 * [1] (static, input) or [M] (per-token, output).  xq: int8 [M, K] (K-major:
 * the GEMM's A operand as is), 16-byte aligned.
 * ------------------------------------------------------------------------- */
sq_status sq_smooth_quant_act(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                              sq_act_mode mode, float *a_scale, int8_t *xq, sq_stream stream);

/* (3b) RMSNorm with 1/s folded into its gain, fused with the static INT8
 * quantisation (kwkr 2.3 and 3.2: absorb the per-channel scaling into the
 * preceding norm's gamma so smoothing costs nothing at run time; aiu):
 *
 *   r_m  = fl(1 / fl(sqrt(fl(mean + eps))))
 *   mean = fl32(sum_j x_mj^2 / d), the sum of (exact) squares taken in fp64
 *   g'_j = fl(gamma_j * recip(s_j))
 *   xq   = q(fl(fl(fl(x * r_m) * g'_j) * recip(a_scale[0])))
 *
 * x: [M, d] of `dt`.  gamma, s: fp32 [d].  a_scale: fp32 [1] (static).
 * xq: int8 [M, d].  rstd: fp32 [M] receives r_m, or NULL.  The fp64 sum is a
 * tree sum; its order only matters when the fp64 mean sits within ~1e-15 of
 * an fp32 rounding boundary. */
sq_status sq_rmsnorm_quant(const void *x, sq_dtype dt, int64_t M, int64_t d, const float *gamma,
                           const float *s, float eps, const float *a_scale, int8_t *xq,
                           float *rstd, sq_stream stream);

/* (3c) Calibration statistic of an RMSNorm output, for the linear that reads
 * it (kwkr 3.1: statistics are taken per layer on the layer's own input; the
 * gate/up projections of a decoder MLP read the normalised activations):
 *
 *   absmax[j] = max(absmax[j], max_m |fl(fl(x_mj * r_m) * gamma_j)|),  r_m as in sq_rmsnorm_quant
 *
 * x: [M, d] of `dt`, 16-byte aligned.  gamma: fp32 [d].  absmax: fp32 [d],
 * a running max (the caller zeroes it once).  The per-thread column maxima
 * stay in registers for d * sizeof(dt) <= 64 KiB; wider rows take a slow
 * per-element path. */
sq_status sq_rmsnorm_absmax(const void *x, sq_dtype dt, int64_t M, int64_t d, const float *gamma,
                            float eps, float *absmax, sq_stream stream);

/* -------------------------------------------------------------------------
 * (4) W8A8 GEMM with the dequant epilogue (pwwt 3.1: INT8 matmul with the
 * scale multiplications merged into it; adr-010 key design points 4-5 name
 * the real INT8 kernel as the follow-up of its fake-quant layer):
 *
 *   acc[m,n] = sum_k xq[m,k] * wq[n,k]           (exact int32; K < 133144)
 *   y[m,n]   = RN_out(fmaf((float)acc, fl(a_m * w_scale[n]), bias[n]))
 *
 * a_m = a_scale[0] (static) or a_scale[m] (per-token).  xq: int8 [M, K],
 * wq: int8 [N, K], both K-major and 16-byte aligned, K a multiple of 16.
 * w_scale: fp32 [N].  bias: [N] of out_dt, or NULL.  y: [M, N] of out_dt
 * (fp32/fp16/bf16), 16-byte aligned, N a multiple of 16.  M >= 1.
 * Runs on the 5th-generation tensor cores (tcgen05 kind::i8, TMA-fed shared
 * memory tiles, TMEM int32 accumulators; CTA pairs with cta_group::2 for
 * M > 128).  Small M (<= 128) takes a weight-streaming path (weights fill the
 * 128-row MMA, tokens are its N).  When one 128-row weight tile per SM would
 * leave more than half of the SMs idle, a cluster of 2 or 4 CTAs shares each
 * tile's K range and combines the int32 partial sums in distributed shared
 * memory; no workspace is needed.  For 64 < M <= 128 with more than 74
 * weight tiles, CTA pairs (cta_group::2) take the weights as their 256-row
 * operand and half the token tile each, writing the output transposed.  The
 * stream-K schedule (iterations shared
 * evenly among the SMs, partial sums through global memory) is the fallback
 * when the cluster split is off (sq_debug_inject(2)); it needs
 * `workspace` of sq_linear_workspace_size(M, N, K) bytes (16-byte aligned;
 * the size depends on the current device's SM count and the test hooks, and
 * is 0 when no workspace is used): one BM x BN int32 partial-sum slot per CTA
 * plus one int32 arrival counter per weight tile.  The counters must be zero
 * before the first use of a workspace (e.g. cudaMemsetAsync once) and are
 * left zero by every call; the slots need no initialisation.  Without a
 * workspace (NULL or too small) that path runs one tile per CTA.  Results are
 * bit-identical on every schedule (exact int32 sums).  Calls sharing one
 * workspace must not overlap on the GPU.
 * ------------------------------------------------------------------------- */
size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K);

sq_status sq_linear_w8a8(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                         const float *a_scale, sq_act_mode mode, const float *w_scale,
                         const void *bias, sq_dtype out_dt, void *y, void *workspace,
                         size_t workspace_bytes, sq_stream stream);

/* sq_linear_w8a8 for callers that cannot allocate device memory (the pages
 * have no counterpart to this call).  Some callers cannot call cudaMalloc at
 * all: a plugin running inside a host engine that owns every device buffer
 * and hands it only inputs and outputs, or a latency-critical serving loop
 * that must not pay cudaMalloc's implicit device-wide synchronisation.  This
 * call takes no workspace and runs the same schedules as sq_linear_w8a8, so
 * its results are bit-identical to that call's.  M > 128, and the small-M
 * schedules that keep their partial sums on chip (the cluster split, one tile
 * per CTA, the swapped CTA pairs), use no scratch at all and accept any shape
 * sq_linear_w8a8
 * accepts.  Only the small-M stream-K schedule (the fallback when the cluster
 * split is off, sq_debug_inject(2)) shares weight tiles between CTAs through
 * scratch memory; here that scratch is a fixed array inside the library:
 * 8 MiB of int32 partial-sum slots (sq_linear_w8a8_noalloc_max_elems() int32
 * values) plus 64 KiB of per-tile arrival counters, held by every GPU that
 * loads the library until the process exits.  The schedule needs one slot of
 * 128 x (16 or 32) int32 per CTA, at most 2.4 MB with the 148 SMs of a B200;
 * a request whose slots or counters would not fit (a device with many more
 * SMs) returns SQ_ERR_UNSUPPORTED without launching anything.  The call
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on each device that needs the array looks up its device
 *     address (with that device current) and caches it; make that first call
 *     before any stream capture.
 *   - Each call that shares tiles zeroes the arrival counters it uses (a
 *     stream-ordered memset) before its kernel, since the array keeps the
 *     previous call's contents (a call that timed out leaves its counters
 *     raised); a partial-sum slot is always written before it is read.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (different streams, no ordering between them) race and corrupt each
 *     other's results.  Serialise them on one stream or order them with events.
 * Arguments, layouts and results are those of sq_linear_w8a8. */
sq_status sq_linear_w8a8_noalloc(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                                 const float *a_scale, sq_act_mode mode, const float *w_scale,
                                 const void *bias, sq_dtype out_dt, void *y, sq_stream stream);

/* Capacity of the fixed partial-sum array of sq_linear_w8a8_noalloc, in int32 values (2^21). */
size_t sq_linear_w8a8_noalloc_max_elems(void);

/* fp16 storage of the scales ("010. SmoothQuant Integration", consequences:
 * storage).  sq_scales_to_f16 rounds fp32 scales to fp16 (nearest even;
 * uint16 bit patterns), sq_scales_from_f16 widens them back exactly.
 * sq_linear_w8a8_f16scales is sq_linear_w8a8 with a_scale and w_scale stored
 * as fp16: the epilogue widens them exactly, so its result equals
 * sq_linear_w8a8 given the widened fp32 scales, bit for bit.  w_scale_f16
 * 16-byte aligned. */
sq_status sq_scales_to_f16(const float *in, int64_t n, uint16_t *out, sq_stream stream);
sq_status sq_scales_from_f16(const uint16_t *in, int64_t n, float *out, sq_stream stream);
sq_status sq_linear_w8a8_f16scales(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                                   const uint16_t *a_scale_f16, sq_act_mode mode,
                                   const uint16_t *w_scale_f16, const void *bias, sq_dtype out_dt, void *y,
                                   void *workspace, size_t workspace_bytes, sq_stream stream);

/* Raw int32 accumulators acc[m,n] = sum_k xq[m,k] * wq[n,k] from the same
 * tensor-core mainloop (for exact INT32 checks).  acc: int32 [M, N]. */
sq_status sq_gemm_s32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                      int32_t *acc, sq_stream stream);

/* Gate/up GEMM with the SiLU*mul epilogue of a decoder MLP block.  wq_gu and
 * w_scale_gu are in the interleaved order of sq_quant_weight_gateup.  With
 * g, u the fp32 dequant values (no bias) of the gate and up rows of output
 * channel c:
 *
 *   h[m,c] = RN_bf16(fl(silu(g) * u)),  silu(g) = g / (1 + exp(-g))
 *
 * h: bf16 [M, N_h] or NULL.  If hq != NULL the epilogue also smooths and
 * quantises h for the next linear with a static scale:
 *   hq[m,c] = q(fl(fl(h[m,c] * recip(s2_c)) * recip(a2[0])))
 * using the bf16-rounded h (so it equals sq_smooth_quant_act on h).
 * s2: fp32 [N_h] or NULL, a2: fp32 [1] (required with hq).  s2 == NULL is
 * the folded form (weights from sq_quant_weight_gateup_fold, h already
 * divided by s2): hq[m,c] = q(fl(h[m,c] * recip(a2[0]))).  N_h a multiple
 * of 128.
 * silu(g) is computed in fp32 with CUDA's fast exponential and division
 * intrinsics (errors of a few fp32 ulp, far below bf16's 8 bits); h matches
 * a correctly rounded SiLU within 2 bf16 ulp (or 1e-30 absolute). */
sq_status sq_linear_w8a8_gateup_silu(const int8_t *xq, const int8_t *wq_gu, int64_t M,
                                     int64_t N_h, int64_t K, const float *a_scale,
                                     sq_act_mode mode, const float *w_scale_gu, void *h,
                                     const float *s2, const float *a2, int8_t *hq,
                                     sq_stream stream);

/* -------------------------------------------------------------------------
 * FP8 (E4M3) variant.  aiunderstanding.org, "SmoothQuant 和激活量化" (on the
 * method's future): the same smoothing carries over to FP8 formats on the
 * Hopper / Blackwell tensor cores.  The calls mirror the INT8 ones with the
 * same fp32 operation order; only the code format changes:
 *
 *   E4M3 code     = e4m3(v): round to nearest even, magnitudes beyond the
 *                   largest finite value 448 saturate to +-448 (never NaN)
 *   absmax scale  = fl(max |value| / 448)
 *   act code      = e4m3(fl(fl(x * recip(s_j)) * recip(a)))
 *   weight code   = e4m3(fl(fl(w * s_j) * recip(w_scale_n)))
 *   acc[m,n]      = sum_k dec(xq8[m,k]) * dec(wq8[n,k])  in fp32 on the
 *                   tensor cores (tcgen05 kind::f8f6f4; every product is
 *                   exact, the sum is rounded in an unspecified order)
 *   y[m,n]        = RN_out(fmaf(acc, fl(a_m * w_scale_n), bias_n))
 *
 * Codes are uint8 bit patterns (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits).  Layouts, alignment and ownership are those of the INT8
 * calls; the FP8 GEMM runs on the CTA-pair kernel for every M.
 * ------------------------------------------------------------------------- */

/* sq_smooth_scales with the static activation scale for E4M3 codes:
 * a_static[0] = fl(max_j fl(act_max_j * recip(s_j)) / 448).  s is the same. */
sq_status sq_smooth_scales_fp8(const float *act_max, const float *w_max, int64_t K, float alpha,
                               float *s, float *a_static, sq_stream stream);

/* W' = fl(W * s_j); w_scale[n] = fl(max_j |W'[n,j]| / 448); wq8 = e4m3 codes
 * of fl(W' * recip(w_scale[n])).  wq8: uint8 [N, K]. */
sq_status sq_quant_weight_fp8(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s,
                              uint8_t *wq8, float *w_scale, sq_stream stream);

/* x' = fl(x * recip(s_j)); static: a = a_scale[0] (read); per-token:
 * a_scale[m] = fl(max_j |x'[m,j]| / 448) (written); xq8 = e4m3 codes of
 * fl(x' * recip(a)).  xq8: uint8 [M, K]. */
sq_status sq_smooth_quant_act_fp8(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                                  sq_act_mode mode, float *a_scale, uint8_t *xq8, sq_stream stream);

/* y[m,n] = RN_out(fmaf(acc, fl(a_m * w_scale[n]), bias[n])) with the fp32
 * tensor-core sum acc of the E4M3 products (see above).  Shapes and
 * alignment as sq_linear_w8a8 (K a multiple of 16, N a multiple of 16);
 * no workspace. */
sq_status sq_linear_fp8(const uint8_t *xq8, const uint8_t *wq8, int64_t M, int64_t N, int64_t K,
                        const float *a_scale, sq_act_mode mode, const float *w_scale,
                        const void *bias, sq_dtype out_dt, void *y, sq_stream stream);

/* The calibration statistic of h for the next linear, taken in the same
 * epilogue instead of writing h (kwkr 3.1: statistics per layer on the
 * layer's own input; h is the down projection's input):
 *
 *   h_absmax[c] = max(h_absmax[c], max_m |h[m,c]|),  h as in sq_linear_w8a8_gateup_silu
 *
 * (the bf16-rounded h, so the result equals sq_calib_absmax on the h that
 * sq_linear_w8a8_gateup_silu writes).  h_absmax: fp32 [N_h], a running max
 * the caller zeroes once.  Nothing else is written.  N_h a multiple of 128. */
sq_status sq_linear_w8a8_gateup_silu_absmax(const int8_t *xq, const int8_t *wq_gu, int64_t M, int64_t N_h,
                                            int64_t K, const float *a_scale, sq_act_mode mode,
                                            const float *w_scale_gu, float *h_absmax, sq_stream stream);

/* -------------------------------------------------------------------------
 * Per-layer alpha search (adr-010 key design point 2: pick, per layer, the
 * alpha of a small grid with the least output reconstruction error, using the
 * same quantisation math as the final layer).
 * ------------------------------------------------------------------------- */

/* Unquantised reference product of fp16 inputs on the tensor cores
 * (tcgen05 kind::f16, fp32 accumulation): y = RN_f16(sum_k x[m,k] w[n,k]).
 * x: fp16 [M, K], w: fp16 [N, K], y: fp16 [M, N]; K a multiple of 8, N a
 * multiple of 16, all 16-byte aligned. */
sq_status sq_gemm_f16_ref(const void *x, const void *w, int64_t M, int64_t N, int64_t K,
                          void *y, sq_stream stream);

/* Sum of squared differences of two fp16 tensors, added in fp64 to
 * *sse (device fp64 [1]; the caller zeroes it).  n elements, 16-byte aligned. */
sq_status sq_sse_f16(const void *y, const void *y_ref, int64_t n, double *sse, sq_stream stream);

/* Bytes of device workspace sq_alpha_search needs. */
size_t sq_alpha_search_workspace_size(int64_t M_held, int64_t N, int64_t K, int n_alpha);

/* For each alpha in alphas[0..n_alpha) (host array, ascending): s -> static
 * scale -> weight quant -> quant of the held batch -> INT8 GEMM -> fp16 y ->
 * mse = mean((y - y_ref)^2), with y_ref = sq_gemm_f16_ref(x_held, w).  The
 * chosen alpha is the first whose mse is not beaten by more than 1e-6
 * relative by a later one (ties go to the smaller alpha).
 * x_held: fp16 [M_held, K]; w: fp16 [N, K]; act_max, w_max: fp32 [K].
 * best_alpha: HOST float; mse: HOST double [n_alpha] or NULL.  Synchronises
 * `stream` (the choice is made on the host).  n_alpha in [1, 16]. */
sq_status sq_alpha_search(const void *x_held, const void *w, int64_t M_held, int64_t N, int64_t K,
                          const float *act_max, const float *w_max, const float *alphas,
                          int n_alpha, void *workspace, size_t workspace_bytes,
                          float *best_alpha, double *mse, sq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
