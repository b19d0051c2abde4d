/*
 * oracle.c -- plain, slow, single-threaded CPU oracle for the per-rank
 * mixed-precision optimizer step over an owned flat shard.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file.  Only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the
 * CUDA library: every number it uses is derived here from the definitions.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -std=c99 -shared -fPIC
 * (no contraction: every FP32 product and sum below is rounded on its own).
 *
 * Sources (pages, by title and section):
 *  [NEOX-DD]  "GPT-NeoX: how it opened the door to democratised 100B-scale
 *             training" (ainews.cool), section "技术深度解析" (technical
 *             deep-dive): under ZeRO stage 1 the optimizer state is split
 *             across data-parallel ranks and each device updates only the
 *             shard it owns.
 *  [OPT-CS]   "OPT: Open Pre-trained Transformer Language Models"
 *             (ai-papers.xuzou.cn summary), section "计算设置" (compute
 *             setup): Adam state kept in FP32 and sharded, weights in FP16,
 *             dynamic loss scaling used against underflow.
 *  [OPT-BN]   same page, section "瓶颈" (bottlenecks): mixed-precision Adam
 *             costs about 16 bytes per parameter; loss divergence went with
 *             the loss scale collapsing toward zero.
 *  [OPT-MA]   same page, section "方法适配" (method adaptation): a gradient
 *             pre-divide factor against over/underflow of the cross-rank
 *             gradient sum; gradient clipping changed from 1.0 to 0.3; the
 *             dynamic loss scaler reset / restart from a healthy checkpoint.
 *  [ADAMW]    The pages never write Adam's update out.  The update is the
 *             textbook AdamW of Loshchilov & Hutter ("Decoupled Weight Decay
 *             Regularization", ICLR 2019) with Kingma & Ba's bias correction,
 *             in the form p <- p(1 - lr*wd) - (lr/bc1) * m / (sqrt(v)/sqrt(bc2) + eps).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - overflow = any non-finite unscaled gradient element, or a non-finite norm;
 *  - on overflow the step is skipped: no state changes, the applied-step count
 *    t does not advance, the scale drops by scale_factor (floored at min_scale)
 *    and the growth counter resets; with a hysteresis h > 1 the scale drops
 *    only once h overflows happened since the last growth (Megatron-style);
 *  - the SGD fallback is plain SGD without momentum, with the same decoupled
 *    weight decay as AdamW;
 *  - after scale_window consecutive applied steps the scale grows by
 *    scale_factor (unless the grown scale would not be finite) and the
 *    counter resets;
 *  - pre-divide: each buffer is multiplied by fl32(1/predivide) before the FP32
 *    sum over buffers; the sum is then multiplied by fl32(1/(post*S)) with
 *    post = K/predivide (computed in double, then rounded once);
 *  - the reported norm is the pre-clip L2 norm of the unscaled gradient;
 *  - clip coefficient c = clip/(norm + 1e-6) in double, used only when < 1;
 *  - the 16-bit cast is IEEE round-to-nearest-even, overflowing to +-inf.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 and bfloat16 <-> binary32, written from the format      */
/* definitions (sign | exponent | fraction), round-to-nearest-even.          */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0 = subnormal (fraction * 2^-24), exponent 31 = inf / NaN. */
float orc_f16_decode(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    float mag;
    if (exp == 0)
        mag = ldexpf((float)frac, -24);
    else if (exp == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexpf((float)(1024 + frac), exp - 25);
    return sign ? -mag : mag;
}

/* Round-to-nearest-even: keep `q` (the value's integer multiple of the target
 * ulp), look at the discarded remainder `rem` out of `half*2`. */
static uint32_t rne(uint32_t q, uint32_t rem, uint32_t half)
{
    if (rem > half || (rem == half && (q & 1u)))
        return q + 1u;
    return q;
}

uint16_t orc_f16_encode(float f)
{
    uint32_t x = f32_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u)                        /* NaN stays NaN (quiet) */
        return (uint16_t)(sign | 0x7e00u | ((ax >> 13) & 0x3ffu));
    if (ax == 0x7f800000u)                       /* +-inf */
        return (uint16_t)(sign | 0x7c00u);
    int e = (int)(ax >> 23) - 127;               /* unbiased exponent */
    uint32_t sig = (ax & 0x7fffffu) | 0x800000u; /* 24-bit significand */
    if (e >= 16)                                 /* >= 2^16: beyond the range */
        return (uint16_t)(sign | 0x7c00u);
    if (e >= -14) {
        /* normal: value = sig * 2^(e-23); keep 11 bits -> drop 13 */
        uint32_t q = rne(sig >> 13, sig & 0x1fffu, 0x1000u);
        /* q in [1024, 2048]; 2048 carries into the exponent (and to inf
         * when e == 15, which is the correct encoding 0x7c00). */
        uint32_t code = ((uint32_t)(e + 15) << 10) + (q - 1024u);
        return (uint16_t)(sign | code);
    }
    if (ax < 0x00800000u) {                      /* binary32 zero / subnormal */
        return sign;                             /* < 2^-126, far below 2^-25 */
    }
    /* subnormal result: units of 2^-24; value/2^-24 = sig * 2^(e+1) */
    int s = -(e + 1);                            /* right shift, >= 14 */
    if (s > 24)                                  /* value < 2^-25: rounds to 0 */
        return sign;
    uint32_t q = rne(sig >> s, sig & ((1u << s) - 1u), 1u << (s - 1));
    return (uint16_t)(sign | q);                 /* q == 1024 is the min normal */
}

/* bfloat16: the upper 16 bits of a binary32. */
float orc_bf16_decode(uint16_t h) { return bits_f32((uint32_t)h << 16); }

uint16_t orc_bf16_encode(float f)
{
    uint32_t x = f32_bits(f);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u)                        /* NaN stays NaN (quiet) */
        return (uint16_t)((x >> 16) | 0x0040u);
    /* finite or inf: drop 16 bits with RNE; a carry out of the largest
     * finite value gives 0x7f80 = inf, as IEEE rounding requires. */
    return (uint16_t)rne(x >> 16, x & 0xffffu, 0x8000u);
}

void orc_f16_encode_array(const float* in, uint16_t* out, uint64_t n)
{ for (uint64_t i = 0; i < n; i++) out[i] = orc_f16_encode(in[i]); }
void orc_bf16_encode_array(const float* in, uint16_t* out, uint64_t n)
{ for (uint64_t i = 0; i < n; i++) out[i] = orc_bf16_encode(in[i]); }
void orc_f16_decode_array(const uint16_t* in, float* out, uint64_t n)
{ for (uint64_t i = 0; i < n; i++) out[i] = orc_f16_decode(in[i]); }
void orc_bf16_decode_array(const uint16_t* in, float* out, uint64_t n)
{ for (uint64_t i = 0; i < n; i++) out[i] = orc_bf16_decode(in[i]); }

static float dec16(uint16_t h, int bf16) { return bf16 ? orc_bf16_decode(h) : orc_f16_decode(h); }
static uint16_t enc16(float f, int bf16) { return bf16 ? orc_bf16_encode(f) : orc_f16_encode(f); }

/* ------------------------------------------------------------------------ */
/* Step definitions                                                          */
/* ------------------------------------------------------------------------ */

typedef struct {
    float beta1, beta2, eps;
    float clip_norm;      /* <= 0: clipping off                       [OPT-MA] */
    float predivide;      /* gradient pre-divide factor               [OPT-MA] */
    float scale_factor;   /* loss-scale growth / backoff factor       [OPT-CS] */
    float min_scale;      /* floor of the loss scale                  [OPT-BN] */
    int32_t scale_window; /* applied steps between scale growths               */
    int32_t hysteresis;   /* overflows since the last growth before a back-off
                             (<= 1: back off at every overflow)                */
    int32_t optimizer;    /* 0: AdamW; 1: SGD, the fallback tried   [OPT-MA] */
} orc_hparams;

typedef struct {
    float scale;          /* S: the loss scale the current grads carry */
    int32_t good;         /* consecutive applied steps since the last change */
    int64_t t;            /* applied (non-skipped) Adam steps */
    int32_t hyst;         /* overflows still tolerated before a back-off */
    int32_t pad_;
} orc_scaler;

typedef struct {
    uint64_t offset, numel;
    float weight_decay;
} orc_segment;

typedef struct {
    int32_t overflow;
    int32_t pad_;
    double sumsq;         /* sum of squared unscaled grads (double)        */
    double norm;          /* pre-clip L2 norm; +inf when overflowed        */
    float coef;           /* clip coefficient actually applied             */
    float scale_used;     /* S the grads of this step carried              */
    float scale_next;     /* S the caller multiplies the next loss by      */
    float step_size;      /* fl32(lr / bc1)                                */
    float bc2_sqrt;       /* fl32(sqrt(bc2))                               */
    int32_t pad2_;
    int64_t t;            /* applied steps after this call                 */
} orc_step_info;

/* Factors of the ingest (pre-divide and unscale).                  [OPT-MA]
 * inv_pre = fl32(1/predivide); inv_us = fl32(1/(post*S)), post = K/predivide,
 * both formed in double and rounded once. */
void orc_ingest_factors(int32_t K, float predivide, float scale,
                        float* inv_pre, float* inv_us)
{
    double post = (double)K / (double)predivide;
    *inv_pre = (float)(1.0 / (double)predivide);
    *inv_us = (float)(1.0 / (post * (double)scale));
}

/* Unscaled gradient of one element: a = sum over buffers, in buffer order,
 * of fl32(g_k * inv_pre); then fl32(a * inv_us).                 [OPT-MA][OPT-CS] */
static float unscaled_grad(const uint16_t* const* g, int32_t K, int gbf16,
                           uint64_t j, float inv_pre, float inv_us)
{
    float a = 0.0f;
    for (int32_t k = 0; k < K; k++) {
        float term = dec16(g[k][j], gbf16) * inv_pre;
        a = a + term;
    }
    return a * inv_us;
}

/* The unscaled gradients of elements [0, n) into out[] (for inspection). */
void orc_unscaled_grads(const uint16_t* const* g, int32_t K, int32_t gbf16, uint64_t n,
                        float inv_pre, float inv_us, float* out)
{
    for (uint64_t j = 0; j < n; j++)
        out[j] = unscaled_grad(g, K, gbf16, j, inv_pre, inv_us);
}

/* Pass over the gradients of elements [0, n): count the non-finite unscaled
 * gradients and sum their squares in double, in index order.   [OPT-CS][OPT-MA] */
void orc_grad_stats(const uint16_t* const* g, int32_t K, int32_t gbf16, uint64_t n,
                    float inv_pre, float inv_us,
                    int64_t* nonfinite, double* sumsq)
{
    int64_t bad = 0;
    double s = 0.0;
    for (uint64_t j = 0; j < n; j++) {
        float x = unscaled_grad(g, K, gbf16, j, inv_pre, inv_us);
        if (!isfinite(x))
            bad++;
        double xd = (double)x;
        s += xd * xd;
    }
    *nonfinite = bad;
    *sumsq = s;
}

/* Dynamic loss scaler.                                  [OPT-CS][OPT-BN][OPT-MA]
 * overflow: step skipped, counter reset; the hysteresis count drops by one
 *           (not below 0) and, once it is 0, S <- max(S / factor, min_scale).
 *           With hysteresis <= 1 that is every overflow.
 * applied:  counter + 1; at scale_window: S <- S * factor unless that is not
 *           finite (then S stays), counter reset, hysteresis count refilled. */
int32_t orc_hysteresis(const orc_hparams* hp) { return hp->hysteresis > 1 ? hp->hysteresis : 1; }

void orc_scaler_update(const orc_hparams* hp, orc_scaler* sc, int32_t overflow)
{
    if (overflow) {
        sc->good = 0;
        if (sc->hyst > 0)
            sc->hyst -= 1;
        if (sc->hyst == 0) {
            float s = sc->scale / hp->scale_factor;
            sc->scale = s > hp->min_scale ? s : hp->min_scale;
        }
        return;
    }
    sc->good += 1;
    if (sc->good >= hp->scale_window) {
        float s = sc->scale * hp->scale_factor;
        if (isfinite(s))            /* a scale never grows to infinity */
            sc->scale = s;
        sc->good = 0;
        sc->hyst = orc_hysteresis(hp);
    }
}

/* Global-norm clip coefficient: clip/(norm + 1e-6) when that is below one,
 * else 1 (also 1 when clipping is off).                               [OPT-MA] */
float orc_clip_coef(float clip, double norm)
{
    if (!(clip > 0.0f))
        return 1.0f;
    double c = (double)clip / (norm + 1e-6);
    if (c >= 1.0)
        return 1.0f;
    return (float)c;
}

/* Weight decay of global element index `idx` from a sorted segment table. */
static float segment_wd(const orc_segment* segs, int32_t nsegs, uint64_t idx)
{
    int32_t lo = 0, hi = nsegs - 1;
    while (lo < hi) {                 /* last segment whose offset <= idx */
        int32_t mid = (lo + hi + 1) / 2;
        if (segs[mid].offset <= idx) lo = mid; else hi = mid - 1;
    }
    return segs[lo].weight_decay;
}

/* AdamW update of n elements.                                   [ADAMW][OPT-CS]
 * Element j has global index index[j] (or first + j when index is NULL), its
 * K gradients at g[k][j], and FP32 state master[j], m[j], v[j], 16-bit copy
 * w[j].  Each line is one FP32 operation, rounded on its own. */
void orc_adam_apply(uint64_t n, const uint64_t* index, uint64_t first,
                    const uint16_t* const* g, int32_t K, int32_t gbf16,
                    const orc_segment* segs, int32_t nsegs,
                    float* master, float* m, float* v, uint16_t* w, int32_t wbf16,
                    const orc_hparams* hp, float lr, const orc_step_info* info)
{
    float inv_pre, inv_us;
    orc_ingest_factors(K, hp->predivide, info->scale_used, &inv_pre, &inv_us);
    const float c = info->coef;
    const float b1 = hp->beta1, b2 = hp->beta2, eps = hp->eps;
    const float omb1 = 1.0f - b1, omb2 = 1.0f - b2;
    const float step_size = info->step_size, bcs = info->bc2_sqrt;
    for (uint64_t j = 0; j < n; j++) {
        uint64_t idx = index ? index[j] : first + j;
        float wd = segment_wd(segs, nsegs, idx);
        float gj = unscaled_grad(g, K, gbf16, j, inv_pre, inv_us);
        float gh = gj * c;                         /* clipped grad      */
        float mj = b1 * m[j];                      /* first moment      */
        mj = mj + omb1 * gh;
        float vj = b2 * v[j];                      /* second moment     */
        float gg = omb2 * gh;
        vj = vj + gg * gh;
        float den = sqrtf(vj) / bcs;               /* sqrt(v/bc2) + eps */
        den = den + eps;
        float p = master[j];
        float lrwd = lr * wd;                      /* decoupled decay   */
        float keep = 1.0f - lrwd;
        p = p * keep;
        float upd = mj / den;                      /* Adam direction    */
        p = p - step_size * upd;
        m[j] = mj;
        v[j] = vj;
        master[j] = p;
        w[j] = enc16(p, wbf16);                    /* working copy      */
    }
}

/* Plain SGD (no momentum) with the same decoupled weight decay, the
 * alternative optimizer the OPT run tried:                           [OPT-MA]
 * p <- p(1 - lr*wd) - lr * (g*c); the moments are left untouched. */
void orc_sgd_apply(uint64_t n, const uint64_t* index, uint64_t first,
                   const uint16_t* const* g, int32_t K, int32_t gbf16,
                   const orc_segment* segs, int32_t nsegs,
                   float* master, uint16_t* w, int32_t wbf16,
                   const orc_hparams* hp, float lr, const orc_step_info* info)
{
    float inv_pre, inv_us;
    orc_ingest_factors(K, hp->predivide, info->scale_used, &inv_pre, &inv_us);
    const float c = info->coef;
    for (uint64_t j = 0; j < n; j++) {
        uint64_t idx = index ? index[j] : first + j;
        float wd = segment_wd(segs, nsegs, idx);
        float gj = unscaled_grad(g, K, gbf16, j, inv_pre, inv_us);
        float g_clipped = gj * c;
        float q = master[j];
        float lr_wd = lr * wd;
        float retain = 1.0f - lr_wd;     /* decoupled decay */
        q = q * retain;
        float delta = lr * g_clipped;    /* gradient step   */
        q = q - delta;
        master[j] = q;
        w[j] = enc16(q, wbf16);
    }
}

/* The per-step scalar decisions, given the pass-1 results: overflow, norm,
 * scaler, clip coefficient, applied-step count and bias corrections.
 * Returns the info the update needs; updates the scaler state in place. */
void orc_step_decide(const orc_hparams* hp, orc_scaler* sc, float lr,
                     int64_t nonfinite, double sumsq, orc_step_info* info)
{
    memset(info, 0, sizeof(*info));
    info->scale_used = sc->scale;
    int32_t overflow = nonfinite != 0;
    double norm = sqrt(sumsq);
    if (!overflow && !isfinite(norm))
        overflow = 1;
    info->sumsq = sumsq;
    orc_scaler_update(hp, sc, overflow);
    info->scale_next = sc->scale;
    info->overflow = overflow;
    if (overflow) {
        info->norm = INFINITY;
        info->coef = 0.0f;
        info->t = sc->t;
        return;
    }
    info->norm = norm;
    sc->t += 1;
    info->t = sc->t;
    info->coef = orc_clip_coef(hp->clip_norm, norm);
    double bc1 = 1.0 - pow((double)hp->beta1, (double)sc->t);
    double bc2 = 1.0 - pow((double)hp->beta2, (double)sc->t);
    info->step_size = (float)((double)lr / bc1);
    info->bc2_sqrt = (float)sqrt(bc2);
}

/* One full step over a whole shard of n elements held in host memory:
 * pass 1 (ingest, overflow flag, norm), the scalar decisions, then pass 2
 * (AdamW + cast) unless the step overflowed.  Returns info->overflow. */
int32_t orc_step(uint64_t n, const uint16_t* const* g, int32_t K, int32_t gbf16,
                 const orc_segment* segs, int32_t nsegs,
                 float* master, float* m, float* v, uint16_t* w, int32_t wbf16,
                 const orc_hparams* hp, orc_scaler* sc, float lr, orc_step_info* info)
{
    float inv_pre, inv_us;
    orc_ingest_factors(K, hp->predivide, sc->scale, &inv_pre, &inv_us);
    int64_t bad;
    double sumsq;
    orc_grad_stats(g, K, gbf16, n, inv_pre, inv_us, &bad, &sumsq);
    orc_step_decide(hp, sc, lr, bad, sumsq, info);
    if (!info->overflow) {
        if (hp->optimizer == 1)
            orc_sgd_apply(n, NULL, 0, g, K, gbf16, segs, nsegs, master, w, wbf16, hp, lr, info);
        else
            orc_adam_apply(n, NULL, 0, g, K, gbf16, segs, nsegs,
                           master, m, v, w, wbf16, hp, lr, info);
    }
    return info->overflow;
}

/* ------------------------------------------------------------------------ */
/* float64 brute force: the same equations with every intermediate in       */
/* double and double state.  For tiny shards; it bounds the FP32 oracle's   */
/* own rounding.                                                            */
/* ------------------------------------------------------------------------ */
int32_t orc64_step(uint64_t n, const uint16_t* const* g, int32_t K, int32_t gbf16,
                   const orc_segment* segs, int32_t nsegs,
                   double* master, double* m, double* v,
                   const orc_hparams* hp, orc_scaler* sc, float lr, double* norm_out)
{
    double S = (double)sc->scale;
    double post = (double)K / (double)hp->predivide;
    double sumsq = 0.0;
    int32_t overflow = 0;
    for (uint64_t j = 0; j < n; j++) {
        double a = 0.0;
        for (int32_t k = 0; k < K; k++)
            a += (double)dec16(g[k][j], gbf16) / (double)hp->predivide;
        double x = a / (post * S);
        if (!isfinite(x))
            overflow = 1;
        sumsq += x * x;
    }
    double norm = sqrt(sumsq);
    if (!isfinite(norm))
        overflow = 1;
    orc_scaler_update(hp, sc, overflow);
    if (overflow) {
        *norm_out = INFINITY;
        return 1;
    }
    *norm_out = norm;
    sc->t += 1;
    double c = 1.0;
    if (hp->clip_norm > 0.0f) {
        c = (double)hp->clip_norm / (norm + 1e-6);
        if (c > 1.0) c = 1.0;
    }
    double b1 = hp->beta1, b2 = hp->beta2, eps = hp->eps, lrd = lr;
    double bc1 = 1.0 - pow(b1, (double)sc->t);
    double bc2 = 1.0 - pow(b2, (double)sc->t);
    for (uint64_t j = 0; j < n; j++) {
        double a = 0.0;
        for (int32_t k = 0; k < K; k++)
            a += (double)dec16(g[k][j], gbf16) / (double)hp->predivide;
        double gh = a / (post * S) * c;
        if (hp->optimizer == 1) {  /* SGD */
            double wd = segment_wd(segs, nsegs, j);
            master[j] = master[j] * (1.0 - lrd * wd) - lrd * gh;
            continue;
        }
        m[j] = b1 * m[j] + (1.0 - b1) * gh;
        v[j] = b2 * v[j] + (1.0 - b2) * gh * gh;
        double wd = segment_wd(segs, nsegs, j);
        double p = master[j] * (1.0 - lrd * wd);
        master[j] = p - lrd * (m[j] / bc1) / (sqrt(v[j] / bc2) + eps);
    }
    return 0;
}
