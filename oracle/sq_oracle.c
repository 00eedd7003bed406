/*
 * sq_oracle.c -- plain CPU oracle for the SmoothQuant W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm use it.  It shares no code, header or table
 * with the CUDA library: every step is written out here, one scalar
 * operation at a time, in the order fixed below, so that a reader can check
 * it against the pages by eye.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (no FMA contraction: every fp32 product and sum is rounded on its own;
 * the one fused multiply-add of the dequant epilogue is an explicit fmaf()).
 *
 * Sources (the five pages on SmoothQuant this layer is built from):
 *   [KWKR]   kwkr.cn blog, "SmoothQuant W8A8 ... single node 530B" (Chinese
 *            engineering notes), sections 1.2, 2.1-2.3, 3.1-3.3, 5.2.
 *   [TBR8]   tbr8.org "activation outliers: why SmoothQuant ..." article,
 *            PyTorch toy example (clamp of the statistic at 1e-5).
 *   [PWWT]   pwwt.cn "SmoothQuant技术解析：LLM模型INT8无损量化实践", 3.1
 *            (INT8 matmul with merged scale multiply).
 *   [AIU]    aiunderstanding.org "SmoothQuant 和激活量化", technical insight.
 *   [ADR10]  blog.yoooo.fun "010. SmoothQuant Integration", Context and
 *            key design points 1-6.
 *
 * Canonical fp32 order (the GPU follows the same order by specification):
 *   recip(v)      = v > 0 ? fl(1/v) : 0
 *   quant(v)      = clamp(round_half_even(v), -127, 127)
 *   act code      = quant(fl(fl(x * recip(s_j)) * recip(a)))
 *   weight code   = quant(fl(fl(w * s_j) * recip(w_scale_n)))
 *   per-row scale = fl(max_j |value_j| / 127)
 *   dequant       = fmaf((float)acc, fl(a_m * w_scale_n), bias_n)
 *                   (fl((float)acc * fl(a_m * w_scale_n)) without bias)
 *
 * Parity status of every function is listed in oracle/__init__.py's header.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2 };
enum { OR_STATIC = 0, OR_PER_TOKEN = 1 };

/* ---------------------------------------------------------------------- */
/* Number formats, written from the IEEE 754 binary16 / bfloat16 layouts.  */
/* ---------------------------------------------------------------------- */

float oracle_f16_to_f32(uint16_t h)
{
    /* binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits */
    unsigned sign = (h >> 15) & 1u, e = (h >> 10) & 31u, m = h & 1023u;
    float mag;
    if (e == 0)        mag = ldexpf((float)m, -24);               /* zero / subnormal */
    else if (e == 31)  mag = m ? NAN : INFINITY;
    else               mag = ldexpf((float)(m | 1024u), (int)e - 25);
    return sign ? -mag : mag;
}

float oracle_bf16_to_f32(uint16_t b)
{
    /* bfloat16 is the top half of a binary32 */
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_f16(float f)
{
    /* round to nearest, ties to even */
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u) return sign | 0x7e00u;                 /* NaN */
    if (ax >= 0x477ff000u) return sign | 0x7c00u;                /* >= 65520 -> inf */
    if (ax < 0x38800000u) {                                       /* < 2^-14: subnormal */
        float k = nearbyintf(fabsf(f) * 16777216.0f);             /* units of 2^-24, exact scaling */
        return sign | (uint16_t)k;                                /* k == 1024 is 2^-14 */
    }
    uint32_t e = (ax >> 23) - 127u + 15u;
    uint32_t m = ax & 0x7fffffu;
    uint32_t h = (e << 10) | (m >> 13);
    uint32_t rem = m & 0x1fffu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;  /* carry may bump the exponent */
    return sign | (uint16_t)h;
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    if ((x & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((x >> 16) | 0x40u);   /* quiet NaN */
    x += 0x7fffu + ((x >> 16) & 1u);                               /* ties to even */
    return (uint16_t)(x >> 16);
}

static float ld(const void *p, int dt, int64_t i)
{
    if (dt == OR_F32)  return ((const float *)p)[i];
    if (dt == OR_F16)  return oracle_f16_to_f32(((const uint16_t *)p)[i]);
    return oracle_bf16_to_f32(((const uint16_t *)p)[i]);
}

static void st(void *p, int dt, int64_t i, float v)
{
    if (dt == OR_F32)       ((float *)p)[i] = v;
    else if (dt == OR_F16)  ((uint16_t *)p)[i] = oracle_f32_to_f16(v);
    else                    ((uint16_t *)p)[i] = oracle_f32_to_bf16(v);
}

/* ---------------------------------------------------------------------- */
/* Symmetric INT8 quantisation: x_q = round(x / s), zero point 0           */
/* [KWKR] 1.2 and 3.3; [ADR10] context step 3 and key design point 6.     */
/* ---------------------------------------------------------------------- */

float oracle_recip(float v) { return v > 0.0f ? 1.0f / v : 0.0f; }

int8_t oracle_quant(float v)
{
    float r = nearbyintf(v);            /* default rounding mode: ties to even */
    if (r > 127.0f)  r = 127.0f;        /* symmetric range, -128 never used */
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* Per-tensor (or per-row) scale from an absolute maximum: max / 127. */
float oracle_scale_from_absmax(float m) { return m / 127.0f; }

/* ---------------------------------------------------------------------- */
/* a1/a2: calibration statistic max|X_j| over tokens (running max)         */
/* [KWKR] 3.1 (per-layer, per-channel max of activations and weights);     */
/* [ADR10] key design point 1 (add_batch keeps the per-channel max-abs).   */
/* ---------------------------------------------------------------------- */

void oracle_calib_absmax(const void *x, int dt, int64_t rows, int64_t cols, int64_t ld_,
                         float *absmax)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j) {
            float a = fabsf(ld(x, dt, r * ld_ + j));
            if (a > absmax[j]) absmax[j] = a;
        }
}

/* ---------------------------------------------------------------------- */
/* a3: smoothing factor s_j = max|X_j|^alpha / max|W_j|^(1-alpha)           */
/* [KWKR] 2.2; [AIU] technical insight; [ADR10] context step 1.            */
/* Both statistics are clamped to >= 1e-5 first ([TBR8] clamps at 1e-5).  */
/* Computed in fp64 and rounded once to fp32.                              */
/* ---------------------------------------------------------------------- */

void oracle_smooth_scales(const float *act_max, const float *w_max, int64_t K, float alpha,
                          float *s)
{
    double al = (double)alpha;
    for (int64_t j = 0; j < K; ++j) {
        double a = fmax((double)act_max[j], 1e-5);
        double w = fmax((double)w_max[j], 1e-5);
        s[j] = (float)(pow(a, al) / pow(w, 1.0 - al));
    }
}

/* Closed-form per-tensor activation scale max_j(act_max_j / s_j) / 127:    */
/* [ADR10] key design point 1.                                             */
float oracle_static_scale(const float *act_max, const float *s, int64_t K)
{
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        float v = act_max[j] * oracle_recip(s[j]);
        if (v > m) m = v;
    }
    return oracle_scale_from_absmax(m);
}

/* ---------------------------------------------------------------------- */
/* a4: offline weight transform W' = diag(s) W (column j times s_j in the   */
/* [N,K] out x in layout), then per-output-row symmetric INT8.             */
/* [KWKR] 3.2 and 3.3 (per output channel weight scale); [ADR10] context   */
/* steps 2-3 (weights per row).                                            */
/* ---------------------------------------------------------------------- */

void oracle_quant_weight(const void *w, int dt, int64_t N, int64_t K, const float *s,
                         int8_t *wq, float *w_scale)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float m = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            float wp = ld(w, dt, n * K + j) * s[j];
            if (fabsf(wp) > m) m = fabsf(wp);
        }
        float sc = oracle_scale_from_absmax(m);
        float inv = oracle_recip(sc);
        w_scale[n] = sc;
        for (int64_t j = 0; j < K; ++j) {
            float wp = ld(w, dt, n * K + j) * s[j];
            wq[n * K + j] = oracle_quant(wp * inv);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* a5/a5': runtime smoothing X' = X diag(s)^-1 followed by INT8 quant.      */
/* Smoothing strictly before quantisation: [KWKR] 3.2 and 5.2.             */
/* static: a_scale[0] is given ([ADR10] per-tensor activation scale).      */
/* per-token: a_scale[m] = max_j |x'_mj| / 127 is written.                 */
/* ---------------------------------------------------------------------- */

void oracle_smooth_quant_act(const void *x, int dt, int64_t M, int64_t K, const float *s,
                             int mode, float *a_scale, int8_t *xq)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float inv_a;
        if (mode == OR_STATIC) {
            inv_a = oracle_recip(a_scale[0]);
        } else {
            float mx = 0.0f;
            for (int64_t j = 0; j < K; ++j) {
                float xs = ld(x, dt, m * K + j) * oracle_recip(s[j]);
                if (fabsf(xs) > mx) mx = fabsf(xs);
            }
            a_scale[m] = oracle_scale_from_absmax(mx);
            inv_a = oracle_recip(a_scale[m]);
        }
        for (int64_t j = 0; j < K; ++j) {
            float xs = ld(x, dt, m * K + j) * oracle_recip(s[j]);
            xq[m * K + j] = oracle_quant(xs * inv_a);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* a6: INT8 x INT8 -> INT32 product (exact integer arithmetic), then the   */
/* dequant with the two scales merged ([PWWT] 3.1, merged scale multiply). */
/* acc[m,n] = sum_k xq[m,k] * wq[n,k]                                       */
/* ---------------------------------------------------------------------- */

void oracle_gemm_s32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                     int32_t *acc)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k)
                a += (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];
            acc[m * N + n] = a;
        }
}

/* y[m,n] = (float)acc * fl(a_m * w_scale_n) (+ bias_n as one fused multiply-add), */
/* rounded once to the output type.  bias has the output type.                     */
void oracle_dequant(const int32_t *acc, int64_t M, int64_t N, const float *a_scale, int mode,
                    const float *w_scale, const void *bias, int out_dt, void *y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float am = (mode == OR_STATIC) ? a_scale[0] : a_scale[m];
        for (int64_t n = 0; n < N; ++n) {
            float c = am * w_scale[n];
            float af = (float)acc[m * N + n];
            float v = bias ? fmaf(af, c, ld(bias, out_dt, n)) : af * c;
            st(y, out_dt, m * N + n, v);
        }
    }
}

/* Same epilogue, fp32 values kept (used by the gate/up SiLU*mul step). */
void oracle_dequant_f32(const int32_t *acc, int64_t M, int64_t N, const float *a_scale, int mode,
                        const float *w_scale, float *y)
{
    for (int64_t m = 0; m < M; ++m) {
        float am = (mode == OR_STATIC) ? a_scale[0] : a_scale[m];
        for (int64_t n = 0; n < N; ++n) {
            float c = am * w_scale[n];
            y[m * N + n] = (float)acc[m * N + n] * c;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* a8: RMSNorm with 1/s folded into its gain, then INT8 quant.              */
/* Folding 1/s into the norm's per-channel gain: [KWKR] 2.3 and 3.2;       */
/* [AIU] technical insight (scaling absorbed into a fused op).             */
/*   r_m = 1 / sqrt(mean_j x_mj^2 + eps)   (sum of squares in fp64)        */
/*   g'_j = fl(gamma_j * recip(s_j))                                        */
/*   code = quant(fl(fl(fl(x * r_m) * g'_j) * recip(a)))                    */
/* r_given (nullable) replaces r_m so that codes can be compared given the  */
/* other side's r_m; r_out (nullable) receives r_m.                        */
/* ---------------------------------------------------------------------- */

void oracle_rmsnorm_quant(const void *x, int dt, int64_t M, int64_t d, const float *gamma,
                          const float *s, float eps, const float *a_scale, const float *r_given,
                          int8_t *xq, float *r_out)
{
    float inv_a = oracle_recip(a_scale[0]);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t j = 0; j < d; ++j) {
            double v = (double)ld(x, dt, m * d + j);
            ss += v * v;
        }
        float mean = (float)(ss / (double)d);
        float r = 1.0f / sqrtf(mean + eps);
        if (r_given) r = r_given[m];
        if (r_out) r_out[m] = r;
        for (int64_t j = 0; j < d; ++j) {
            float gp = gamma[j] * oracle_recip(s[j]);
            float y = (ld(x, dt, m * d + j) * r) * gp;
            xq[m * d + j] = oracle_quant(y * inv_a);
        }
    }
}

/* Calibration statistic of the RMSNorm output (the activation that enters the  */
/* gate/up linear): absmax_j = max(absmax_j, max_m |fl(fl(x_mj * r_m) * gamma_j)|), */
/* r_m as in oracle_rmsnorm_quant ([KWKR] 3.1 statistic taken on the layer's     */
/* actual input).                                                                */
void oracle_rmsnorm_absmax(const void *x, int dt, int64_t M, int64_t d, const float *gamma, float eps,
                           float *absmax)
{
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t j = 0; j < d; ++j) {
            double v = (double)ld(x, dt, m * d + j);
            ss += v * v;
        }
        float mean = (float)(ss / (double)d);
        float r = 1.0f / sqrtf(mean + eps);
        for (int64_t j = 0; j < d; ++j) {
            float y = (ld(x, dt, m * d + j) * r) * gamma[j];
            if (fabsf(y) > absmax[j]) absmax[j] = fabsf(y);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* a9: SiLU(gate) * up on the fp32 dequantised gate/up outputs, rounded to  */
/* bf16.  silu(g) = g / (1 + exp(-g)), evaluated in fp64, rounded to fp32, */
/* then to bf16.                                                           */
/* ---------------------------------------------------------------------- */

void oracle_silu_mul_bf16(const float *g, const float *u, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; ++i) {
        double gd = (double)g[i];
        double hv = gd / (1.0 + exp(-gd)) * (double)u[i];
        h[i] = oracle_f32_to_bf16((float)hv);
    }
}

/* ---------------------------------------------------------------------- */
/* a7: output reconstruction error used by the per-layer alpha search       */
/* ([ADR10] key design point 2): mean((y - y_ref)^2) over fp16 outputs, in  */
/* fp64.                                                                    */
/* ---------------------------------------------------------------------- */

double oracle_mse_f16(const uint16_t *y, const uint16_t *y_ref, int64_t n)
{
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double d = (double)oracle_f16_to_f32(y[i]) - (double)oracle_f16_to_f32(y_ref[i]);
        acc += d * d;
    }
    return n > 0 ? acc / (double)n : 0.0;
}

/* Unquantised reference product y_ref = RN16(sum_k x w) of fp16 inputs,     */
/* accumulated in fp64 (the exact sum up to fp64 rounding), rounded to fp16.  */
void oracle_gemm_f16_ref(const uint16_t *x, const uint16_t *w, int64_t M, int64_t N, int64_t K,
                         uint16_t *y)
{
    /* both operands are widened once (exactly) to fp64, then summed in fp64 */
    double *xd = (double *)malloc((size_t)(M * K) * sizeof(double));
    double *wd = (double *)malloc((size_t)(N * K) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M * K; ++i) xd[i] = (double)oracle_f16_to_f32(x[i]);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N * K; ++i) wd[i] = (double)oracle_f16_to_f32(w[i]);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double a = 0.0;
            for (int64_t k = 0; k < K; ++k)
                a += xd[m * K + k] * wd[n * K + k];
            y[m * N + n] = oracle_f32_to_f16((float)a);
        }
    free(xd);
    free(wd);
}

/* Array forms of the number-format conversions (used to widen / round whole
 * tensors in the pipelines and tests). */
void oracle_to_f32_array(const void *src, int dt, int64_t n, float *dst)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = ld(src, dt, i);
}

void oracle_from_f32_array(const float *src, int64_t n, int dt, void *dst)
{
    for (int64_t i = 0; i < n; ++i) st(dst, dt, i, src[i]);
}
