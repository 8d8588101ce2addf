/*
 * AWQ oracle: a plain, slow, obviously-correct CPU restatement of the
 * activation-aware scale search for one linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Sources (web pages; cited by title and section):
 *   [QAS-QA]   "Как работает quantization-aware scaling в AWQ для защиты
 *              важных весов?"  (Russian Q&A page)
 *   [AWQ-note] "AWQ: Activation-Aware Weight Quantization For On-Device LLM
 *              Compression AND Acceleration" (Chinese reading note)
 *   [Notes-52] "52 · AWQ, GPTQ và SmoothQuant" (Vietnamese notes)
 *   [GPTQ-AWQ] "GPTQ与AWQ" (Chinese markdown notes)
 *   [AWQ-wiki] "AWQ" encyclopedia page (French)
 *
 * Arithmetic conventions (the pages fix no precision; the decisions that turn
 * floating point into integer codes are taken in IEEE binary32, the kernel's
 * precision, and everything else is binary64):
 *   RN32(x)  = the binary64 value x rounded to binary32, ties to even.  Every
 *              binary32 +,-,*,/ is written as the binary64 operation followed
 *              by RN32; for one operation on binary32 inputs this equals the
 *              IEEE binary32 result (double rounding is innocuous because
 *              53 >= 2*24+2; S. Figueroa, "When is double rounding
 *              innocuous?", SIGNUM 1995).
 *   RN16(x)  = IEEE binary16 round-to-nearest-even, written below from the
 *              format's definition (subnormals kept, overflow to infinity).
 *   rint     = nearbyint() under the default FE_TONEAREST mode (ties to even).
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared.
 * Contraction must stay off so that no a*b+c is fused behind our back.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <float.h>

/* ------------------------------------------------------------------ */
/* binary16 and binary32 rounding                                      */
/* ------------------------------------------------------------------ */

static float rn32(double x) { return (float)x; }

/* Exact value of an IEEE binary16 bit pattern. */
double awq_oracle_h2d(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)       v = ldexp((double)m, -24);            /* subnormal / zero */
    else if (e == 31) v = m ? NAN : INFINITY;
    else              v = ldexp((double)(1024 + m), e - 25); /* (1.m) * 2^(e-15) */
    return sign ? -v : v;
}

/* IEEE binary16 round-to-nearest-even of a binary64 value. */
uint16_t awq_oracle_rn16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (isnan(x)) return 0x7E00;
    /* 65520 is the midpoint between 65504 (odd significand) and 2^16, so it
     * and everything above round to infinity. */
    if (ax >= 65520.0) return sign | 0x7C00;
    if (ax == 0.0) return sign;
    int e2;
    frexp(ax, &e2);                 /* ax = f * 2^e2, f in [0.5, 1) */
    int ue = e2 - 1;                /* floor(log2(ax)) */
    if (ue < -14) ue = -14;         /* subnormal range shares the 2^-24 quantum */
    double quantum = ldexp(1.0, ue - 10);
    double r = nearbyint(ax / quantum);   /* ax/quantum is exact (power of two) */
    double v = r * quantum;               /* exact */
    if (v < ldexp(1.0, -14)) return sign | (uint16_t)r;   /* subnormal: m = v / 2^-24 */
    int ev;
    double fv = frexp(v, &ev);      /* v = fv * 2^ev, fv in [0.5, 1) */
    int E = ev - 1;                 /* v = (2 fv) * 2^E, 2 fv in [1, 2) */
    uint16_t mant = (uint16_t)((2.0 * fv - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

/* The zero point as stored: the integer rint(-min/scale), saturated to the
 * largest finite binary16 magnitude (the zeros are kept in fp16), rounded to
 * binary16 (integers above 2048 are not all representable), and +0 in place
 * of -0.  The search, the packer and every consumer use this stored value. */
static double stored_zero(double z)
{
    if (z > 65504.0) z = 65504.0;
    if (z < -65504.0) z = -65504.0;
    z = awq_oracle_h2d(awq_oracle_rn16(z));
    return z == 0.0 ? 0.0 : z;
}

/* ------------------------------------------------------------------ */
/* Step a1: activation statistics                                      */
/*   [AWQ-note] "Measures": collect each layer's input X and take its  */
/*   average absolute value a; [GPTQ-AWQ] "量化方法": importance =      */
/*   X.abs().mean(dim=0) over in_features.  Per INPUT channel j.       */
/* ------------------------------------------------------------------ */

/* a[j] = RN32( (sum_t |X[t,j]|) / T ).  The sum is taken in binary64 in row
 * order; it is exact whenever sum < 2^29 because every binary16 value is a
 * multiple of 2^-24. */
void awq_oracle_act_stats(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, float *a)
{
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) s += fabs(awq_oracle_h2d(X[t * ldx + j]));
        a[j] = rn32(s / (double)T);
    }
}

/* ------------------------------------------------------------------ */
/* Step a2: search space  s_j = a_j ^ alpha                            */
/*   [AWQ-note] "Measures": for each candidate alpha compute a^alpha   */
/*   (one hyper-parameter per layer sets the protection strength).     */
/* ------------------------------------------------------------------ */

/* s[j] = RN32(pow(max(a_j, FLT_MIN), alpha)).  A channel that never fires
 * (a_j = 0) is lifted to the smallest normal binary32 so that pow stays
 * finite; alpha = 0 gives s = 1 exactly. */
void awq_oracle_scales(const float *a, int64_t K, float alpha, float *s)
{
    for (int64_t j = 0; j < K; ++j) {
        double aj = a[j] < FLT_MIN ? (double)FLT_MIN : (double)a[j];
        s[j] = rn32(pow(aj, (double)alpha));
    }
}

/* ------------------------------------------------------------------ */
/* Steps a3/a4: scale, group-wise round-to-nearest, dequant, unscale.  */
/*   [QAS-QA] §5: multiply the channel's weights by s, divide the      */
/*   activation by s, quantize with group-wise round-to-nearest; §9:   */
/*   quant_config zero_point=True, q_group_size=128, w_bit=4.           */
/*   [AWQ-wiki] "Fondements techniques": scaling before quantization,  */
/*   the inverse scaling after dequantization.                         */
/*   [AWQ-note] "Measures": Y = (W D)(D^-1 x); scale per input channel. */
/* Per row n and group G of g consecutive columns:                     */
/*   w'_k   = RN32(w_k * s_k)                                          */
/*   mn,mx  = min, max of w'_k over the group                          */
/* asymmetric (zero_point = 1):                                         */
/*   scale  = RN32(RN32(mx - mn) / qmax)                               */
/*   z      = RN16(sat(rint(-mn * r)))  (zero point = round(-min/scale),*/
/*            not clamped to the codes; sat() keeps it inside the      */
/*            finite fp16 range +-65504 it is stored in, and the       */
/*            stored fp16 value is the z used below, so the stored     */
/*            metadata reproduce what exactly; never -0)               */
/* symmetric (zero_point = 0; [AWQ-note] "Measures": the INT3 grid of  */
/* step max|w| / (2^(b-1) - 1)):                                        */
/*   scale  = RN32(max(-mn, mx) / (2^(b-1) - 1)),  z = 2^(b-1)          */
/* both:                                                               */
/*   sh     = RN16(clamp(scale, 2^-24, 65504))  (stored fp16 scale)    */
/*   r      = RN32(1 / sh)                                             */
/*   q_k    = clamp(rint(w'_k * r) + z, 0, qmax)                       */
/* The products inside rint are exact (binary32 x binary32 fits in      */
/* binary64): q = round(w'/scale) is rounded once, by rint itself.      */
/*   what_k = RN16(RN32(RN32((q_k - z) * sh) * RN32(1 / s_k)))         */
/* mask (may be NULL): channels k with mask[k] != 0 stay in fp16        */
/* ([AWQ-note] "Measures": keeping 1% of the channels in FP16): they    */
/* take no part in their group's min and max and what_k = w_k; a group  */
/* with every channel masked has mn = mx = 0.                           */
/* no_round != 0 replaces rint by the identity in q_k (and drops the   */
/* clamp), which turns quantization into an exact identity up to       */
/* binary32/binary16 rounding (a test hook).                           */
/* ------------------------------------------------------------------ */

void awq_oracle_quantize(const uint16_t *W, int64_t N, int64_t K, const float *s,
                         int bits, int g, int zero_point, const uint8_t *mask, int no_round,
                         uint8_t *q_out,        /* [N,K]  codes (may be NULL)        */
                         uint16_t *sh_out,      /* [N,K/g] fp16 bits (may be NULL)   */
                         float *z_out,          /* [N,K/g] zero points (may be NULL) */
                         uint16_t *what_out)    /* [N,K]  fp16 bits of W-hat         */
{
    const double qmax = (double)((1 << bits) - 1);
    const double qsym = (double)((1 << (bits - 1)) - 1);
    const int64_t G = K / g;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float wp[256];
        for (int64_t gi = 0; gi < G; ++gi) {
            const int64_t k0 = gi * g;
            float mn = INFINITY, mx = -INFINITY;
            for (int k = 0; k < g; ++k) {
                wp[k] = rn32(awq_oracle_h2d(W[n * K + k0 + k]) * (double)s[k0 + k]);
                if (mask && mask[k0 + k]) continue;
                if (wp[k] < mn) mn = wp[k];
                if (wp[k] > mx) mx = wp[k];
            }
            if (mn > mx) { mn = 0.0f; mx = 0.0f; }      /* every channel kept in fp16 */
            float scale;
            if (zero_point) {
                float range = rn32((double)mx - (double)mn);
                scale = rn32((double)range / qmax);
            } else {
                double amax = -(double)mn > (double)mx ? -(double)mn : (double)mx;
                scale = rn32(amax / qsym);
            }
            double sc = scale;
            if (sc < ldexp(1.0, -24)) sc = ldexp(1.0, -24);
            if (sc > 65504.0) sc = 65504.0;
            uint16_t shb = awq_oracle_rn16(sc);
            double sh = awq_oracle_h2d(shb);
            float r = rn32(1.0 / sh);
            double z;
            if (zero_point) {
                z = stored_zero(nearbyint(-(double)mn * (double)r));    /* exact product */
            } else {
                z = qsym + 1.0;                 /* 2^(b-1): the middle code */
            }
            if (sh_out) sh_out[n * G + gi] = shb;
            if (z_out) z_out[n * G + gi] = (float)z;
            for (int k = 0; k < g; ++k) {
                double t = (double)wp[k] * (double)r;          /* exact product */
                double q;
                if (no_round) {
                    q = t + z;
                } else {
                    q = nearbyint(t) + z;
                    if (q < 0.0) q = 0.0;
                    if (q > qmax) q = qmax;
                }
                float rs = rn32(1.0 / (double)s[k0 + k]);
                float deq = rn32((q - z) * sh);
                float un = rn32((double)deq * (double)rs);
                what_out[n * K + k0 + k] = (mask && mask[k0 + k]) ? W[n * K + k0 + k] : awq_oracle_rn16(un);
                if (q_out) q_out[n * K + k0 + k] = (uint8_t)q;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Channel selection for the FP16-protection baselines ([AWQ-note]     */
/* "Measures": keep the 1% most important channels, judged by the      */
/* activation, or -- the weaker choice -- by the weights).             */
/* mask[j] = 1 for the k channels of largest stat (ties: lower index    */
/* first; NaN ranks below every number), 0 elsewhere.  Plain O(K^2).    */
/* ------------------------------------------------------------------ */

void awq_oracle_topk(const float *stat, int64_t K, int64_t k, uint8_t *mask)
{
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < K; ++j) {
        int64_t above = 0;
        const int nj = isnan(stat[j]);
        for (int64_t i = 0; i < K; ++i) {
            if (i == j) continue;
            const int ni = isnan(stat[i]);
            int before;
            if (ni || nj) before = (!ni && nj) || (ni && nj && i < j);
            else before = stat[i] > stat[j] || (stat[i] == stat[j] && i < j);
            above += before;
        }
        mask[j] = above < k ? 1 : 0;
    }
}

/* ------------------------------------------------------------------ */
/* AWQ followed by GPTQ error compensation ([AWQ-note] "Measures": the  */
/* two are complementary, AWQ+GPTQ at INT2; [Notes-52] §4: round one    */
/* column at a time and push its error into the weights not yet         */
/* quantized, weighted by second-order statistics of the real input;    */
/* [GPTQ-AWQ] "GPTQ": column-wise, with a Cholesky factor prepared      */
/* once).  The sweep below takes U, the upper Cholesky factor of the    */
/* damped inverse Hessian (H^-1 = U^T U), as given, and works on the    */
/* scaled weights w = RN32(W s) of one row, in binary32:                 */
/*   for k = 0 .. K-1:                                                  */
/*     at the first column of a group: the group's parameters from the  */
/*       group's current weights (the quantizer above, w' = w);         */
/*     q_k  = clamp(rint(w_k r) + z, 0, qmax)     (exact product)       */
/*     wq_k = RN32((q_k - z) sh)                                        */
/*     e    = RN32(RN32(w_k - wq_k) / U_kk)                             */
/*     w_j  = fmaf(-e, U_kj, w_j)   for j = k+1 .. K-1, in order         */
/*   what_k = RN16(RN32(wq_k RN32(1 / s_k)))                            */
/* fixed_step > 0 replaces the group parameters by a fixed grid of that */
/* step (q = rint(w / step), no clamp; a test hook for the pages' toy   */
/* example).  stop_after >= 0 stops after that many columns and leaves  */
/* the current weights in w_out (a test hook for one update step).      */
/* ------------------------------------------------------------------ */

void awq_oracle_gptq(const uint16_t *W, int64_t N, int64_t K, const float *s, const float *U,
                     int bits, int g, int zero_point, double fixed_step, int64_t stop_after,
                     uint8_t *q_out, uint16_t *sh_out, float *z_out, uint16_t *what_out, float *w_out)
{
    const double qmax = (double)((1 << bits) - 1);
    const double qsym = (double)((1 << (bits - 1)) - 1);
    const int64_t G = K / g;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < N; ++n) {
        float *w = w_out + n * K;
        for (int64_t k = 0; k < K; ++k) w[k] = rn32(awq_oracle_h2d(W[n * K + k]) * (double)s[k]);
        double sh = 1.0, r = 1.0, z = 0.0;
        const int64_t last = stop_after >= 0 && stop_after < K ? stop_after : K;
        for (int64_t k = 0; k < last; ++k) {
            if (fixed_step <= 0.0 && k % g == 0) {
                float mn = INFINITY, mx = -INFINITY;
                for (int64_t j = k; j < k + g; ++j) {
                    if (w[j] < mn) mn = w[j];
                    if (w[j] > mx) mx = w[j];
                }
                float scale;
                if (zero_point) scale = rn32((double)rn32((double)mx - (double)mn) / qmax);
                else scale = rn32((-(double)mn > (double)mx ? -(double)mn : (double)mx) / qsym);
                double sc = scale;
                if (sc < ldexp(1.0, -24)) sc = ldexp(1.0, -24);
                if (sc > 65504.0) sc = 65504.0;
                uint16_t shb = awq_oracle_rn16(sc);
                sh = awq_oracle_h2d(shb);
                r = rn32(1.0 / sh);
                if (zero_point) {
                    z = stored_zero(nearbyint(-(double)mn * r));
                } else {
                    z = qsym + 1.0;
                }
                if (sh_out) sh_out[n * G + k / g] = shb;
                if (z_out) z_out[n * G + k / g] = (float)z;
            }
            double q, wq;
            if (fixed_step > 0.0) {
                q = nearbyint((double)w[k] / fixed_step);
                wq = rn32(q * fixed_step);
            } else {
                q = nearbyint((double)w[k] * r) + z;
                if (q < 0.0) q = 0.0;
                if (q > qmax) q = qmax;
                wq = rn32((q - z) * sh);
            }
            const float e = rn32((double)rn32((double)w[k] - wq) / (double)U[k * K + k]);
            for (int64_t j = k + 1; j < K; ++j) w[j] = fmaf(-e, U[k * K + j], w[j]);
            if (q_out) q_out[n * K + k] = (uint8_t)(q < 0 ? 0 : q);
            if (what_out) what_out[n * K + k] = awq_oracle_rn16(rn32(wq * (double)rn32(1.0 / (double)s[k])));
            w[k] = (float)wq;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Step a8: pack codes, LSB first.  The container is 4 bits for w_bit  */
/* 3 and 4 (8 codes per 32-bit word) and 2 bits for w_bit 2 (16 per    */
/* word): code of column k sits at bits c*(k mod 32/c) of word         */
/* k/(32/c).  ([AWQ-note] "Measures": save the quantized weights and   */
/* the necessary quantization metadata.)                               */
/* ------------------------------------------------------------------ */

void awq_oracle_pack_codes(const uint8_t *q, int64_t N, int64_t K, int bits, uint32_t *codes)
{
    const int c = bits == 2 ? 2 : 4;
    const int per = 32 / c;
    const int64_t words = K / per;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < words; ++w) {
            uint32_t v = 0;
            for (int i = 0; i < per; ++i)
                v |= (uint32_t)q[n * K + w * per + i] << (c * i);
            codes[n * words + w] = v;
        }
}

/* ------------------------------------------------------------------ */
/* Step a7: argmin over the grid, first index wins, NaN counts as +inf */
/* ([AWQ-note] "Measures": keep the best alpha of each layer).         */
/* ------------------------------------------------------------------ */

int awq_oracle_argmin(const double *losses, int n)
{
    int best = 0;
    double bv = INFINITY;
    int have = 0;
    for (int i = 0; i < n; ++i) {
        double v = isnan(losses[i]) ? INFINITY : losses[i];
        if (!have || v < bv) { bv = v; best = i; have = 1; }
    }
    return best;
}

/* ------------------------------------------------------------------ */
/* Worked-example primitives (real arithmetic, binary64).               */
/* [AWQ-note] "Measures": step 1/3 INT3 grid {0, 1/3, 2/3, 1}; the step */
/* grows to 2/3 when the group maximum grows to 2.0, i.e. a symmetric   */
/* absmax step max|w| / (2^(b-1) - 1).  [Notes-52] §3: round to a grid  */
/* of step 0.125.                                                       */
/* ------------------------------------------------------------------ */

double awq_oracle_round_to_step(double w, double step) { return nearbyint(w / step) * step; }

double awq_oracle_absmax_step(const double *w, int n, int bits)
{
    double m = 0.0;
    for (int i = 0; i < n; ++i) if (fabs(w[i]) > m) m = fabs(w[i]);
    return m / (double)((1 << (bits - 1)) - 1);
}
