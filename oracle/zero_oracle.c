/*
 * zero_oracle.c -- plain float64 CPU oracle for the ZeRO-2/3 mixed-precision
 * Adam step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * library; the two meet only through the seeded synthetic inputs.
 *
 * Sources (three web pages on DeepSpeed ZeRO):
 *   [DS-ZeRO]  DeepSpeed documentation page "ZeRO" (code-docs zero3.rst),
 *              the numbered list of stages 1-3 and the AdamW config example.
 *   [QA]       "How does DeepSpeed ZeRO stage 1, 2, and 3 partition optimizer
 *              states, gradients, and parameters?", memory-footprint matrix.
 *   [DD]       "Deep dive: DeepSpeed" lesson, sections
 *              "Count state before choosing a stage",
 *              "Reduce first, then update the owned slice",
 *              "Resume training and export weights separately".
 *
 * Everything is float64 with scalar loops in the order the method states it.
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository as well):
 *   - AdamW uses decoupled decay on the pre-update weight:
 *       w <- w - lr * (mhat / (sqrt(vhat) + eps) + weight_decay * w);
 *     with weight_decay = 0 this is the [DD] scalar Adam exactly.
 *   - The reduced gradient is sum_r(n_r * g_r) / (sum_r(n_r) * S); equal
 *     weighting is n_r = 1 (the [DD] listing's sum / ranks), token weighting
 *     uses per-rank token counts n_r, S is the loss scale (1 unless fp16).
 *   - The overflow check covers every raw gradient of every rank; a skipped
 *     step changes no weight or moment, leaves t unchanged and halves S.
 *   - Growth of S (x2 after `growth_interval` consecutive applied steps when
 *     checking is on) is not described by the pages; it follows the stated
 *     loss-scaling reading and is pinned by a schedule derived by hand from
 *     that reading (tests/golden/loss_scale_schedule.txt), not by the pages.
 *   - 16-bit parameters are the round-to-nearest-even of the float64 master,
 *     rounded once, directly to the 16-bit format.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ZO_F64 0
#define ZO_F32 1
#define ZO_BF16 2
#define ZO_F16 3

#define ZO_OK 0
#define ZO_EINVAL (-1)

typedef struct zo_hparams {
    double lr, beta1, beta2, eps, weight_decay;
} zo_hparams;

typedef struct zo_ctrl {
    uint64_t t;               /* applied updates so far */
    uint64_t skipped;         /* skipped steps so far */
    double loss_scale;        /* S */
    uint32_t growth_tracker;  /* consecutive applied steps since the last change of S */
    uint32_t growth_interval; /* 0: S never grows */
    int32_t last_skipped;     /* 1 if the most recent step was skipped */
    int32_t pad;
} zo_ctrl;

/* ---------------------------------------------------------------- ownership */

/* [DD] "Reduce first, then update the owned slice": owner r holds the
 * contiguous indices floor(P*r/R) .. floor(P*(r+1)/R) - 1; a slice is empty
 * when the two bounds coincide (possible when R > P).  The products are taken
 * in 128-bit integers so that no P*r overflows. */
int zo_partition_bounds(uint64_t P, uint32_t R, uint64_t *lo, uint64_t *hi)
{
    if (R == 0 || lo == NULL || hi == NULL) return ZO_EINVAL;
    for (uint32_t r = 0; r < R; ++r) {
        lo[r] = (uint64_t)(((unsigned __int128)P * r) / R);
        hi[r] = (uint64_t)(((unsigned __int128)P * (r + 1)) / R);
    }
    return ZO_OK;
}

/* ------------------------------------------------------- number formats */

/* IEEE 754 binary16: sign, 5-bit exponent (bias 15), 10-bit fraction. */
double zo_f16_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double mag;
    if (e == 31)
        mag = f ? NAN : INFINITY;
    else if (e == 0)
        mag = ldexp((double)f, -24);           /* subnormal: f/1024 * 2^-14 */
    else
        mag = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return s ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double zo_bf16_to_double(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double zo_load(int dtype, const void *base, uint64_t k)
{
    switch (dtype) {
    case ZO_F64: return ((const double *)base)[k];
    case ZO_F32: return (double)((const float *)base)[k];
    case ZO_BF16: return zo_bf16_to_double(((const uint16_t *)base)[k]);
    default: return zo_f16_to_double(((const uint16_t *)base)[k]);
    }
}

/* Round x once to a binary format with `prec` significand bits (counting the
 * leading one), smallest normal exponent `emin` and largest finite `maxval`,
 * ties to even.  Returns the rounded value as a double (+-inf on overflow). */
static double zo_round_to_format(double x, int prec, int emin, double maxval)
{
    if (isnan(x) || isinf(x) || x == 0.0) return x;
    double a = fabs(x);
    int e;
    frexp(a, &e);               /* a = f * 2^e with f in [0.5, 1) */
    int lead = e - 1;           /* exponent of the leading bit */
    if (lead < emin) lead = emin; /* subnormal range: fixed spacing */
    double ulp = ldexp(1.0, lead - (prec - 1));
    double q = a / ulp;         /* exact: division by a power of two */
    double fl = floor(q);
    double frac = q - fl;       /* exact */
    double n;
    if (frac > 0.5)
        n = fl + 1.0;
    else if (frac < 0.5)
        n = fl;
    else
        n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: even */
    double y = n * ulp;
    if (y > maxval) y = INFINITY;
    return copysign(y, x);
}

/* bfloat16: 8 significand bits, emin = -126, max = (2 - 2^-7) * 2^127. */
uint16_t zo_rne_bf16(double x)
{
    if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFFC0u : 0x7FC0u);
    double y = zo_round_to_format(x, 8, -126, ldexp(255.0, 120));
    float f = (float)y; /* exact: y is a bfloat16 value */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

/* binary16: 11 significand bits, emin = -14, max = 65504. */
uint16_t zo_rne_f16(double x)
{
    if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFE00u : 0x7E00u);
    double y = zo_round_to_format(x, 11, -14, 65504.0);
    uint16_t sign = signbit(y) ? 0x8000u : 0u;
    double a = fabs(y);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) /* subnormal: a = f * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(a * ldexp(1.0, 24)));
    int e;
    double f = frexp(a, &e); /* a = f * 2^e, f in [0.5,1) */
    int lead = e - 1;
    uint16_t frac = (uint16_t)((2.0 * f - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((lead + 15) << 10) | frac);
}

/* Cast n masters to the 16-bit parameter format (bit patterns). */
int zo_cast_params(uint64_t n, const double *w, int dtype, uint16_t *out)
{
    if (dtype != ZO_BF16 && dtype != ZO_F16) return ZO_EINVAL;
    for (uint64_t k = 0; k < n; ++k)
        out[k] = (dtype == ZO_BF16) ? zo_rne_bf16(w[k]) : zo_rne_f16(w[k]);
    return ZO_OK;
}

/* -------------------------------------------------------------- Adam step */

/* [DD] "Reduce first, then update the owned slice", the scalar Adam update:
 * first and second moments, bias correction by 1 - beta^t, epsilon added
 * outside the square root.  weight_decay adds the decoupled AdamW term of the
 * [DS-ZeRO] optimizer config ("AdamW", weight_decay). */
void zo_adam_update(double *w, double *m, double *v, double g, uint64_t t,
                    const zo_hparams *h)
{
    *m = h->beta1 * *m + (1.0 - h->beta1) * g;
    *v = h->beta2 * *v + (1.0 - h->beta2) * g * g;
    double mhat = *m / (1.0 - pow(h->beta1, (double)t));
    double vhat = *v / (1.0 - pow(h->beta2, (double)t));
    *w = *w - h->lr * (mhat / (sqrt(vhat) + h->eps) + h->weight_decay * *w);
}

/* Does any gradient of any rank hold an inf or a NaN? */
int zo_any_nonfinite(uint64_t n, uint32_t R, int gdtype, const void *const *grads)
{
    int found = 0;
    for (uint32_t r = 0; r < R; ++r) {
#pragma omp parallel for reduction(| : found)
        for (uint64_t k = 0; k < n; ++k)
            if (!isfinite(zo_load(gdtype, grads[r], k))) found |= 1;
    }
    return found;
}

/* The reduced gradient of element k: the weighted mean over ranks in rank
 * order 0..R-1, divided by the loss scale. */
static double zo_reduce(uint32_t R, int gdtype, const void *const *grads,
                        const double *weights, double wsum, double S, uint64_t k)
{
    double s = 0.0;
    for (uint32_t r = 0; r < R; ++r)
        s += (weights ? weights[r] : 1.0) * zo_load(gdtype, grads[r], k);
    return s / (wsum * S);
}

static int zo_check_args(uint64_t n, uint32_t R, int gdtype, const void *const *grads,
                         const zo_hparams *h, zo_ctrl *c, double *w, double *m, double *v)
{
    if (R == 0 || grads == NULL || h == NULL || c == NULL) return ZO_EINVAL;
    if (gdtype < ZO_F64 || gdtype > ZO_F16) return ZO_EINVAL;
    if (n > 0 && (w == NULL || m == NULL || v == NULL)) return ZO_EINVAL;
    for (uint32_t r = 0; r < R; ++r)
        if (n > 0 && grads[r] == NULL) return ZO_EINVAL;
    return ZO_OK;
}

/* Skip bookkeeping: nothing is updated, t stays, S halves. */
static void zo_apply_skip(zo_ctrl *c)
{
    c->loss_scale *= 0.5;
    c->growth_tracker = 0;
    c->skipped += 1;
    c->last_skipped = 1;
}

static void zo_apply_success(zo_ctrl *c, uint64_t t, int check)
{
    c->t = t;
    c->last_skipped = 0;
    if (check) {
        c->growth_tracker += 1;
        if (c->growth_interval != 0 && c->growth_tracker == c->growth_interval) {
            c->loss_scale *= 2.0;
            c->growth_tracker = 0;
        }
    }
}

static double zo_weight_sum(uint32_t R, const double *weights)
{
    double wsum = 0.0;
    for (uint32_t r = 0; r < R; ++r) wsum += weights ? weights[r] : 1.0;
    return wsum;
}

/* One step, unsharded: every element is reduced over all ranks and updated.
 * n elements; grads[r] holds n gradients of rank r in dtype `gdtype`;
 * weights: R per-rank weights (token counts) or NULL for the equal mean.
 * Returns 1 if the step was skipped, 0 if applied, <0 on bad arguments. */
int zo_step_unsharded(uint64_t n, uint32_t R, int gdtype, const void *const *grads,
                      const double *weights, int check, const zo_hparams *h,
                      zo_ctrl *c, double *w, double *m, double *v)
{
    int rc = zo_check_args(n, R, gdtype, grads, h, c, w, m, v);
    if (rc) return rc;
    if (check && zo_any_nonfinite(n, R, gdtype, grads)) {
        zo_apply_skip(c);
        return 1;
    }
    uint64_t t = c->t + 1;
    double wsum = zo_weight_sum(R, weights), S = c->loss_scale;
#pragma omp parallel for
    for (uint64_t k = 0; k < n; ++k) {
        double g = zo_reduce(R, gdtype, grads, weights, wsum, S, k);
        zo_adam_update(&w[k], &m[k], &v[k], g, t, h);
    }
    zo_apply_success(c, t, check);
    return 0;
}

/* One step, sharded: owner r reduces only the indices it owns (a reference
 * reduce-scatter) and updates only its own slice of w, m, v.
 * The n elements stand at global positions idx[k] of a P-element parameter
 * vector (idx NULL: positions 0..n-1 with n == P), so that a sample of a large
 * vector can be checked element by element.  The overflow decision covers
 * every rank's gradients, as a flag combined across all ranks would. */
int zo_step_sharded(uint64_t P, uint64_t n, const uint64_t *idx, uint32_t R, int gdtype,
                    const void *const *grads, const double *weights, int check,
                    const zo_hparams *h, zo_ctrl *c, double *w, double *m, double *v,
                    uint64_t *lo, uint64_t *hi)
{
    int rc = zo_check_args(n, R, gdtype, grads, h, c, w, m, v);
    if (rc) return rc;
    if (lo == NULL || hi == NULL || (idx == NULL && n != P)) return ZO_EINVAL;
    zo_partition_bounds(P, R, lo, hi);
    if (check && zo_any_nonfinite(n, R, gdtype, grads)) {
        zo_apply_skip(c);
        return 1;
    }
    uint64_t t = c->t + 1;
    double wsum = zo_weight_sum(R, weights), S = c->loss_scale;
    for (uint32_t owner = 0; owner < R; ++owner) {
        if (idx == NULL) {
#pragma omp parallel for
            for (uint64_t k = lo[owner]; k < hi[owner]; ++k) {
                double g = zo_reduce(R, gdtype, grads, weights, wsum, S, k);
                zo_adam_update(&w[k], &m[k], &v[k], g, t, h);
            }
        } else {
#pragma omp parallel for
            for (uint64_t k = 0; k < n; ++k) {
                if (idx[k] < lo[owner] || idx[k] >= hi[owner]) continue;
                double g = zo_reduce(R, gdtype, grads, weights, wsum, S, k);
                zo_adam_update(&w[k], &m[k], &v[k], g, t, h);
            }
        }
    }
    zo_apply_success(c, t, check);
    return 0;
}

/* The reduced gradients themselves (the retained ZeRO-2 gradient slice), for
 * checking an optional reduced-gradient output. */
int zo_reduced_grads(uint64_t n, uint32_t R, int gdtype, const void *const *grads,
                     const double *weights, double S, double *out)
{
    if (R == 0 || grads == NULL || out == NULL) return ZO_EINVAL;
    double wsum = zo_weight_sum(R, weights);
    for (uint64_t k = 0; k < n; ++k)
        out[k] = zo_reduce(R, gdtype, grads, weights, wsum, S, k);
    return ZO_OK;
}

/* Micro-step gradient accumulation ("Deep dive: DeepSpeed", "Let the engine
 * own the microstep" and "Communication volume isn't elapsed time": ZeRO-2/3
 * reduce and partition the gradient on every backward call, and the owner
 * keeps only its slice between calls; "Count state before choosing a stage":
 * a 4-byte (fp32) accumulation array).  For each element:
 *   acc = (first ? 0 : acc) + scale * reduced gradient of this micro-batch
 * computed in float64 and stored rounded to the nearest float32 (the
 * accumulation dtype), so every micro-step rounds once.  The loss scale is
 * not undone here: the optimizer step does that on the accumulated sum. */
int zo_accumulate(uint64_t n, uint32_t R, int gdtype, const void *const *grads,
                  const double *weights, double scale, int first, float *acc)
{
    if (R == 0 || grads == NULL || (n > 0 && acc == NULL)) return ZO_EINVAL;
    if (gdtype < ZO_F64 || gdtype > ZO_F16) return ZO_EINVAL;
    double wsum = zo_weight_sum(R, weights);
#pragma omp parallel for
    for (uint64_t k = 0; k < n; ++k) {
        double g = zo_reduce(R, gdtype, grads, weights, wsum, 1.0, k);
        double prev = first ? 0.0 : (double)acc[k];
        acc[k] = (float)(prev + scale * g);
    }
    return ZO_OK;
}

int zo_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following OpenMP loops of this process (n >= 1); used to
 * time the oracle single-threaded and on all cores. */
void zo_set_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
