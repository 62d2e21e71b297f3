/*
 * COAT oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of what the COAT
 * FP8-optimizer-state AdamW step and COAT's two activation quantizers
 * compute.  It exists to check the CUDA library; only the test suite,
 * the package entry's smoke() check and bench.py's CPU-baseline leg may
 * load it.  It shares no code, header, table or constant generator with
 * the CUDA library, and it includes nothing from it.
 *
 * Sources (pages, by title and section):
 *   [COAT]  "COAT: 压缩优化器状态和激活以实现内存高效的 FP8 训练"
 *           (blog.daoxuan.cc/posts/57954) -- sections
 *           "为什么二阶动量对量化比一阶动量更敏感" (AdamW, why v is sensitive),
 *           "二阶动量的动态范围反而更小" (dynamic ranges),
 *           "扩展函数：把窄分布拉宽" (the expansion function f and k),
 *           "混合粒度：线性层和非线性层分开处理" (1xG groups, Group Scaling),
 *           "结果和边界" (k must follow the target format's range).
 *   [ATLAS] "LLM Atlas / systems / numerics" (llm-atlas.k1412.top) --
 *           section 03 "FP8" (E4M3 max 448, min subnormal 2^-9; E5M2 max
 *           57344, min subnormal 2^-16) and section 08 "Adam -> AdamW"
 *           (m_t, v_t, update -eta*m_hat/(sqrt(v_hat)+eps), decay (1-eta*lambda)).
 *   [FPX]   "FP8/FP4 formats" blog (53ai.com/news/qianyanjishu/2200.html),
 *           section "FP格式" -- ExMy construction and the subnormal rule
 *           (exponent field 0: implicit bit 0, exponent 1-bias).
 *   [QA]    "AI 低精度格式（bfloat16/FP8/TF32）" (codechuan.com) -- BF16->FP32
 *           is a 16-bit zero pad; FP32 master weights.
 *
 * Arithmetic conventions (compile with -O2 -ffp-contract=off, no fast-math):
 *   - element arithmetic is IEEE binary32 (+ - * / sqrt), one rounding per
 *     operation, in the order written; the pages fix FP32 master weights
 *     and FP32 updates [QA], [ATLAS 02].
 *   - transcendentals (log, pow) are evaluated in binary64 and rounded once
 *     to binary32 where a binary32 result is stored.
 *   - FP8 encoding is round-to-nearest-even with saturation to +-max
 *     ("satfinite"); NaN encodes as 0x7F.
 *
 * Parity status: every exported function is pinned by tests under
 * tests/test_oracle_*.py (format tables, library special cases, closed
 * forms, invariants).  The size of the error reduction that the expansion
 * function brings (a ratio quoted on real OLMo states) is only checked in
 * direction: that magnitude is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_E4M3 0
#define ORC_E5M2 1

#define ORC_OK 0
#define ORC_BAD_ARG 1

/* ------------------------------------------------------------------ */
/* Bit-level number formats                                            */
/* ------------------------------------------------------------------ */

/* Value of an ExMy field pair with the given bias.  [FPX] "FP格式": a
 * normal number is (1 + m/2^M) * 2^(e - bias); at the minimum exponent
 * field (e == 0) the implicit leading bit becomes 0 and the exponent is
 * pinned to 1 - bias, which gives the subnormals and zero. */
double orc_exmy_value(int ebits, int mbits, int bias, uint32_t e, uint32_t m)
{
    (void)ebits;
    double frac = (double)m / (double)(1u << mbits);
    if (e == 0)
        return frac * ldexp(1.0, 1 - bias);
    return (1.0 + frac) * ldexp(1.0, (int)e - bias);
}

/* Decode one FP8 byte.  E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa
 * bits; S.1111.111 is NaN and there is no infinity, so the largest finite
 * value is 1.75 * 2^8 = 448 [ATLAS 03], [FPX].  E5M2: 1 sign, 5 exponent
 * (bias 15), 2 mantissa bits, IEEE-like: exponent field 31 holds inf
 * (mantissa 0) and NaN [QA "E4M3/E5M2"]; largest finite 1.75 * 2^15 = 57344. */
double orc_fp8_decode(uint8_t code, int fmt)
{
    int neg = (code >> 7) & 1;
    double v;
    if (fmt == ORC_E4M3) {
        uint32_t e = (code >> 3) & 15u, m = code & 7u;
        if (e == 15u && m == 7u)
            return NAN;
        v = orc_exmy_value(4, 3, 7, e, m);
    } else {
        uint32_t e = (code >> 2) & 31u, m = code & 3u;
        if (e == 31u)
            return m == 0u ? (neg ? -INFINITY : INFINITY) : NAN;
        v = orc_exmy_value(5, 2, 15, e, m);
    }
    return neg ? -v : v;
}

/* Largest finite positive code of each format. */
static int orc_top_code(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }

double orc_fp8_max(int fmt) { return orc_fp8_decode((uint8_t)orc_top_code(fmt), fmt); }

double orc_fp8_min_subnormal(int fmt) { return orc_fp8_decode(0x01, fmt); }

/* Dynamic range R of a format: largest finite over smallest positive
 * value.  [COAT "二阶动量的动态范围反而更小"]: for E4M3, 448 / 2^-9. */
double orc_fp8_range(int fmt) { return orc_fp8_max(fmt) / orc_fp8_min_subnormal(fmt); }

static double orc_pos_table[2][128];
static int orc_pos_table_ready = 0;

static void orc_init_tables(void)
{
    if (orc_pos_table_ready)
        return;
    for (int f = 0; f < 2; ++f)
        for (int c = 0; c < 128; ++c)
            orc_pos_table[f][c] = orc_fp8_decode((uint8_t)c, f);
    orc_pos_table_ready = 1;
}

/* Encode a binary32 value: the nearest finite FP8 value, ties to the code
 * with an even last bit, magnitudes at or beyond the largest finite value
 * saturate to it, NaN gives 0x7F.  The sign bit is copied from y (so -0.0
 * gives 0x80).  Nearest-value search over the positive codes, in binary64
 * where all the differences below are exact. */
uint8_t orc_fp8_encode(float y, int fmt)
{
    orc_init_tables();
    if (isnan(y))
        return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    int top = orc_top_code(fmt);
    const double *tab = orc_pos_table[fmt];
    if (a >= tab[top])
        return (uint8_t)(sign | top);
    /* binary search: largest code lo with tab[lo] <= a (tab is increasing) */
    int lo = 0, hi = top;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (tab[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    /* now tab[lo] <= a < tab[lo + 1] */
    double dlo = a - tab[lo];
    double dhi = tab[lo + 1] - a;
    int c;
    if (dlo < dhi)
        c = lo;
    else if (dhi < dlo)
        c = lo + 1;
    else
        c = (lo & 1) ? lo + 1 : lo;
    return (uint8_t)(sign | c);
}

/* BF16 -> binary32: the 16 BF16 bits become the high half, the low half is
 * zero [QA "BF16 与 FP32 互转"]. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> BF16, round to nearest, ties to even; NaN -> 0x7FC0 (quiet,
 * sign dropped).  Nearest of the two BF16 neighbours, compared in binary64. */
uint16_t orc_f32_to_bf16(float f)
{
    if (isnan(f))
        return 0x7FC0;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lo_bits = u & 0xFFFF0000u;
    if (lo_bits == u)
        return (uint16_t)(u >> 16);
    /* neighbour one BF16 step further from zero (same sign) */
    uint32_t hi_bits = lo_bits + 0x00010000u;
    float lo_f, hi_f;
    memcpy(&lo_f, &lo_bits, sizeof lo_f);
    memcpy(&hi_f, &hi_bits, sizeof hi_f);
    double a = fabs((double)f);
    double dlo = a - fabs((double)lo_f);
    /* past the largest finite BF16 the upper neighbour is infinity, which
     * IEEE rounding places at 2^128 */
    double dhi = (isinf(hi_f) ? ldexp(1.0, 128) : fabs((double)hi_f)) - a;
    uint32_t r;
    if (dlo < dhi)
        r = lo_bits;
    else if (dhi < dlo)
        r = hi_bits;
    else
        r = ((lo_bits >> 16) & 1u) ? hi_bits : lo_bits;
    return (uint16_t)(r >> 16);
}

/* ------------------------------------------------------------------ */
/* COAT optimizer-state compression                                    */
/* ------------------------------------------------------------------ */

/* The range that k aims to fill.  [COAT "扩展函数"]: k is chosen so the
 * expanded group spans E4M3's range; k_range = 1 takes the storage
 * format's own range instead ([COAT "结果和边界"]: for another format, k
 * follows that format's range). */
static double orc_target_range(int store_fmt, int k_range)
{
    return k_range == 1 ? orc_fp8_range(store_fmt) : orc_fp8_range(ORC_E4M3);
}

/* Inverse expansion of one stored element.  [COAT "扩展函数"]: the stored
 * value is sign(x)|x|^k after scaling; dequantization takes the 1/k power.
 * Scale convention: x = sign(d) * |d|^(1/k) * s, d the decoded FP8 value. */
float orc_state_dequant_one(uint8_t code, float k, float s, int fmt)
{
    if (s == 0.0f)
        return 0.0f;
    double d = orc_fp8_decode(code, fmt);
    if (d == 0.0)
        return 0.0f;
    float p = (float)pow(fabs(d), 1.0 / (double)k);
    float x = p * s;
    return d < 0.0 ? -x : x;
}

/* Quantize one group of FP32 state values (len >= 1).
 * [COAT "扩展函数"] with the sign function of that section:
 *   M  = max |x|, mn = min nonzero |x|, R_X = M / mn;
 *   k  = log(R_target) / log(R_X)  (per group, per step; clamped to k_max
 *        when k_max > 0; k = 1 when R_X == 1);
 *   y  = fmt_max * (|x| / M)^k : the expanded group rescaled so that its
 *        maximum lands on the format's maximum;
 *   code = sign(x) . RNE_satfinite(y); x == 0 gives code 0x00;
 *   s  = M * fmt_max^(-1/k), the scale with which x = |d|^(1/k) * s.
 * An all-zero group stores k = 1, s = 0 and zero codes.  NaN elements are
 * skipped by the range and encode as 0x7F. */
static void orc_quant_group(const float *x, int64_t len, int fmt, int k_range,
                            float k_max, int force_k1, uint8_t *code,
                            float *k_out, float *s_out)
{
    float M = 0.0f, mn = INFINITY;
    for (int64_t i = 0; i < len; ++i) {
        float a = fabsf(x[i]);
        if (isnan(a))
            continue;
        if (a > M)
            M = a;
        if (a > 0.0f && a < mn)
            mn = a;
    }
    if (M == 0.0f) {
        for (int64_t i = 0; i < len; ++i)
            code[i] = isnan(x[i]) ? 0x7F : 0x00;
        *k_out = 1.0f;
        *s_out = 0.0f;
        return;
    }
    double kd;
    if (force_k1 || M == mn) {
        kd = 1.0;
    } else {
        kd = log(orc_target_range(fmt, k_range)) / log((double)M / (double)mn);
        if (k_max > 0.0f && kd > (double)k_max)
            kd = (double)k_max;
    }
    float kf = (float)kd;
    double fmax = orc_fp8_max(fmt);
    float s = (float)((double)M * pow(fmax, -1.0 / (double)kf));
    for (int64_t i = 0; i < len; ++i) {
        float xi = x[i];
        if (isnan(xi)) {
            code[i] = 0x7F;
        } else if (xi == 0.0f) {
            code[i] = 0x00;
        } else {
            float y = (float)(fmax * pow((double)fabsf(xi) / (double)M, (double)kf));
            uint8_t c = orc_fp8_encode(y, fmt);
            code[i] = (uint8_t)(xi < 0.0f ? (c | 0x80) : c);
        }
    }
    *k_out = kf;
    *s_out = s;
}

int orc_quantize_state(const float *x, int64_t n, int64_t G, int fmt, int k_range,
                       float k_max, int force_k1, uint8_t *code, float *k, float *s)
{
    if (n < 0 || G < 1 || (fmt != ORC_E4M3 && fmt != ORC_E5M2))
        return ORC_BAD_ARG;
    for (int64_t g0 = 0, gi = 0; g0 < n; g0 += G, ++gi) {
        int64_t len = n - g0 < G ? n - g0 : G;
        orc_quant_group(x + g0, len, fmt, k_range, k_max, force_k1, code + g0, k + gi, s + gi);
    }
    return ORC_OK;
}

/* Dequantize n stored elements with per-group (k, s).  k == NULL means
 * k = 1 for every group (plain scaled FP8, as for activations). */
int orc_dequant(const uint8_t *q, const float *k, const float *s, int64_t n, int64_t G,
                int fmt, float *out)
{
    if (n < 0 || G < 1 || (fmt != ORC_E4M3 && fmt != ORC_E5M2))
        return ORC_BAD_ARG;
    for (int64_t i = 0; i < n; ++i) {
        int64_t gi = i / G;
        if (k) {
            out[i] = orc_state_dequant_one(q[i], k[gi], s[gi], fmt);
        } else {
            float d = (float)orc_fp8_decode(q[i], fmt);
            out[i] = d * s[gi];
        }
    }
    return ORC_OK;
}

typedef struct {
    float beta1, beta2, lr, eps, weight_decay;
    int64_t step;
    int64_t group_size;
    int32_t m_fmt, v_fmt, k_range;
    float k_max;
    int32_t force_k1;
} orc_adamw_cfg;

/* One COAT AdamW step over a flat parameter buffer of n elements.
 *
 * Per element ([ATLAS 08], [COAT "为什么二阶动量..."]: AdamW with decoupled
 * weight decay on FP32 master weights and BF16 gradients):
 *   g   = float(bf16 grad)
 *   m   = dequant(m code), v = dequant(v code)          (inverse expansion)
 *   m_t = beta1*m + (1-beta1)*g
 *   v_t = beta2*v + (1-beta2)*(g*g)
 *   m^  = m_t / (1 - beta1^t),  v^ = v_t / (1 - beta2^t)
 *   theta_t = theta*(1 - lr*lambda) - lr * m^ / (sqrt(v^) + eps)
 * then per 1xG group the new m_t and v_t are re-quantized (orc_quant_group):
 * the stored states are m_t and v_t themselves, not the bias-corrected ones.
 * The scalar factors 1-beta, 1-beta^t and 1-lr*lambda are rounded to
 * binary32 once (1-beta^t from a binary64 power).
 * m_t_out / v_t_out, when non-NULL, receive the FP32 moments before
 * re-quantization (for error reports). */
int orc_adamw_fp8_step(float *theta, const uint16_t *grad, uint8_t *m_code, float *m_k,
                       float *m_s, uint8_t *v_code, float *v_k, float *v_s, int64_t n,
                       const orc_adamw_cfg *cfg, float *m_t_out, float *v_t_out)
{
    if (!cfg || n < 0 || cfg->group_size < 1 || cfg->step < 1)
        return ORC_BAD_ARG;
    if (cfg->m_fmt != ORC_E4M3 && cfg->m_fmt != ORC_E5M2)
        return ORC_BAD_ARG;
    if (cfg->v_fmt != ORC_E4M3 && cfg->v_fmt != ORC_E5M2)
        return ORC_BAD_ARG;
    const float b1 = cfg->beta1, b2 = cfg->beta2;
    const float c1 = 1.0f - b1;
    const float c2 = 1.0f - b2;
    const float bc1 = (float)(1.0 - pow((double)b1, (double)cfg->step));
    const float bc2 = (float)(1.0 - pow((double)b2, (double)cfg->step));
    const float decay = 1.0f - cfg->lr * cfg->weight_decay;
    const float lr = cfg->lr, eps = cfg->eps;
    const int64_t G = cfg->group_size;

    float *mt = (float *)malloc(sizeof(float) * (size_t)G);
    float *vt = (float *)malloc(sizeof(float) * (size_t)G);
    if (!mt || !vt) {
        free(mt);
        free(vt);
        return ORC_BAD_ARG;
    }
    for (int64_t g0 = 0, gi = 0; g0 < n; g0 += G, ++gi) {
        int64_t len = n - g0 < G ? n - g0 : G;
        for (int64_t j = 0; j < len; ++j) {
            int64_t i = g0 + j;
            float g = orc_bf16_to_f32(grad[i]);
            float m = orc_state_dequant_one(m_code[i], m_k[gi], m_s[gi], cfg->m_fmt);
            float v = orc_state_dequant_one(v_code[i], v_k[gi], v_s[gi], cfg->v_fmt);
            float m_new = b1 * m + c1 * g;
            float v_new = b2 * v + c2 * (g * g);
            float m_hat = m_new / bc1;
            float v_hat = v_new / bc2;
            float u = m_hat / (sqrtf(v_hat) + eps);
            theta[i] = theta[i] * decay - lr * u;
            mt[j] = m_new;
            vt[j] = v_new;
            if (m_t_out)
                m_t_out[i] = m_new;
            if (v_t_out)
                v_t_out[i] = v_new;
        }
        orc_quant_group(mt, len, cfg->m_fmt, cfg->k_range, cfg->k_max, cfg->force_k1,
                        m_code + g0, m_k + gi, m_s + gi);
        orc_quant_group(vt, len, cfg->v_fmt, cfg->k_range, cfg->k_max, cfg->force_k1,
                        v_code + g0, v_k + gi, v_s + gi);
    }
    free(mt);
    free(vt);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* COAT activation quantizers                                          */
/* ------------------------------------------------------------------ */

/* Scale and its reciprocal for a group or tensor maximum: s = amax/fmt_max,
 * inv = fmt_max/amax (binary32 divisions), so the maximum lands on the
 * format's maximum.  A zero (or vanishingly small, <= 2^-100) maximum uses
 * s = inv = 1, which keeps every quotient finite. */
static void orc_act_scale(float amax, int fmt, float *s, float *inv)
{
    const float fmax = (float)orc_fp8_max(fmt);
    if (!(amax > 0x1p-100f)) {
        *s = 1.0f;
        *inv = 1.0f;
    } else {
        *s = amax / fmax;
        *inv = fmax / amax;
    }
}

/* 1xG group quantization of a row-major BF16 matrix [rows, cols] with
 * row stride ld (elements).  [COAT "混合粒度"]: nonlinear-layer inputs are
 * quantized in 1xG groups along the channel (column) axis.  Codes go to
 * q[rows, cols] (row stride cols), scales to scale[rows, cols/G]. */
int orc_group_quant_1xG(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int64_t G,
                        int fmt, uint8_t *q, float *scale)
{
    if (rows < 0 || cols < 0 || G < 1 || cols % G != 0 || ld < cols)
        return ORC_BAD_ARG;
    if (fmt != ORC_E4M3 && fmt != ORC_E5M2)
        return ORC_BAD_ARG;
    const int64_t ng = cols / G;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t gi = 0; gi < ng; ++gi) {
            const uint16_t *xg = x + r * ld + gi * G;
            float amax = 0.0f;
            for (int64_t j = 0; j < G; ++j) {
                float a = fabsf(orc_bf16_to_f32(xg[j]));
                if (a > amax)
                    amax = a;
            }
            float s, inv;
            orc_act_scale(amax, fmt, &s, &inv);
            scale[r * ng + gi] = s;
            for (int64_t j = 0; j < G; ++j)
                q[r * cols + gi * G + j] = orc_fp8_encode(orc_bf16_to_f32(xg[j]) * inv, fmt);
        }
    }
    return ORC_OK;
}

/* Group Scaling per-tensor quantization of n BF16 values.
 * [COAT "混合粒度"]: step (i) takes the max of each 1xG run into a small
 * intermediate (group_amax[ceil(n/G)]); step (ii) takes the max of that
 * intermediate; step (iii) casts the whole tensor with the single scale.
 * If amax_precomputed != 0, group_amax is taken as given (the producer
 * filled it) and step (i) is skipped. */
int orc_group_scaling_pertensor(const uint16_t *x, int64_t n, int64_t G, int fmt,
                                float *group_amax, int amax_precomputed, uint8_t *q,
                                float *scale)
{
    if (n < 0 || G < 1 || (fmt != ORC_E4M3 && fmt != ORC_E5M2))
        return ORC_BAD_ARG;
    const int64_t ng = (n + G - 1) / G;
    if (!amax_precomputed) {
        for (int64_t gi = 0; gi < ng; ++gi) {
            float amax = 0.0f;
            for (int64_t i = gi * G; i < n && i < (gi + 1) * G; ++i) {
                float a = fabsf(orc_bf16_to_f32(x[i]));
                if (a > amax)
                    amax = a;
            }
            group_amax[gi] = amax;
        }
    }
    float amax = 0.0f;
    for (int64_t gi = 0; gi < ng; ++gi)
        if (group_amax[gi] > amax)
            amax = group_amax[gi];
    float s, inv;
    orc_act_scale(amax, fmt, &s, &inv);
    *scale = s;
    for (int64_t i = 0; i < n; ++i)
        q[i] = orc_fp8_encode(orc_bf16_to_f32(x[i]) * inv, fmt);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Array helpers for the tests (plain loops over the scalar functions) */
/* ------------------------------------------------------------------ */

void orc_fp8_encode_array(const float *y, int64_t n, int fmt, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_fp8_encode(y[i], fmt);
}

void orc_f32_to_bf16_array(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_f32_to_bf16(x[i]);
}
