/*
 * hqq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar fp32 CPU restatement of group-wise Half-Quadratic
 * Quantization (HQQ) with per-group early stopping, followed by bit packing and
 * dequantization.  Only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark may load this file's library; the product path never does,
 * and this file shares no code, header, table or constant with the CUDA path.
 *
 * Source of the method: "Half-Quadratic Quantization of Large Machine Learning
 * Models" (Dropbox tech blog, translated page), section 2 ("Half-Quadratic
 * Quantization"):
 *   - quantize / dequantize operators  Q(W) = round(W/s + z),  Q^-1(Wq) = s(Wq - z);
 *   - l_p (p < 1) error  phi(W - Q^-1(Q(W)));
 *   - half-quadratic split with s fixed, alternating sp1 / sp2, beta <- kappa*beta;
 *   - sp1 (section 2.1): W_e = shrink_lp(W - Q^-1(Q(W)), beta),
 *         shrink_lp(x, beta) = sign(x) relu(|x| - |x|^(p-1) / beta);
 *   - sp2 (section 2.2): z = mean over the group of (Wq - (W - W_e)/s), with the
 *         implementation holding 1/s rather than s;
 *   - section 4.1: p = 0.7, beta = 1, kappa = 1.01, 20 iterations, stop early
 *         once the error stops improving.
 * Readings taken where the page is silent:
 *   - min-max initialisation s = (max-min)/(2^b-1), z = -min * (1/s);
 *   - codes are clamped to [0, 2^b-1]; rounding is round-half-to-even;
 *   - early stopping is decided per group on the sum of |W - W_hat|^p (equal to
 *     comparing means, the group size being a power of two): the error of the z
 *     that produced this iteration's codes is computed before the sp1/sp2 update,
 *     the iteration is accepted only on a strict decrease, and the group then
 *     keeps the best z seen;
 *   - a constant group (max == min) uses s = 1, 1/s = 1.
 *
 * Canonical arithmetic (identical, op for op, to what the GPU path must do):
 * every operation is one IEEE-754 binary32 operation rounded to nearest-even;
 * fmaf() is the single-rounding fused multiply-add; sums over a group are the
 * pairwise sum over contiguous halves (PSUM).  The file must be compiled with
 * -ffp-contract=off and without -ffast-math.
 *
 * |x|^p is the table-driven power "powp" (in the spirit of P. T. P. Tang,
 * "Table-driven implementation of the exponential function", ACM TOMS 15(2),
 * 1989): x = 2^k * m, m in [1,2); c_j = 1 + (2j+1)/64 is the centre of m's
 * 1/32-wide cell; m^p = c_j^p (1+r)^p with r = m/c_j - 1, |r| <= 1/64, formed
 * as one fused multiply-add of m and fl(1/c_j), and (1+r)^p is the binomial
 * series to the cubic term.  The 2^(p k) and c_j^p entries are the
 * double-precision library values rounded once to binary32.  Zero and
 * subnormal x give 0 (p > 0), +inf (p < 0), 1 (p == 0).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HQQ_ORACLE_MAX_GROUP 256

/* ------------------------------------------------------------------------- */
/* fp16 <-> fp32 (GCC _Float16: conversions round to nearest-even)           */
/* ------------------------------------------------------------------------- */
static float half_bits_to_float(uint16_t h) {
    _Float16 v;
    memcpy(&v, &h, 2);
    return (float)v;
}

static uint16_t float_to_half_bits(float f) {
    _Float16 v = (_Float16)f;
    uint16_t h;
    memcpy(&h, &v, 2);
    return h;
}

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* ------------------------------------------------------------------------- */
/* powp: x^p for x >= 0 (see header comment)                                 */
/* ------------------------------------------------------------------------- */
typedef struct {
    float two_pk[256];  /* indexed by the biased exponent field of x */
    float cj_p[32];     /* c_j^p */
    float inv_cj[32];   /* fl(1 / c_j) */
    float a1, a2, a3;   /* binomial coefficients C(p,1), C(p,2), C(p,3) */
} powp_table;

static void powp_table_init(powp_table *t, float p) {
    const double pd = (double)p;
    for (int e = 0; e < 256; ++e) {
        if (e == 0)          /* +0 and subnormals */
            t->two_pk[e] = p > 0.0f ? 0.0f : (p < 0.0f ? INFINITY : 1.0f);
        else if (e == 255)   /* inf / nan: outside the method's domain */
            t->two_pk[e] = p > 0.0f ? INFINITY : (p < 0.0f ? 0.0f : 1.0f);
        else
            t->two_pk[e] = (float)exp2(pd * (double)(e - 127));
    }
    for (int j = 0; j < 32; ++j) {
        const double c = 1.0 + (double)(2 * j + 1) / 64.0;
        t->cj_p[j] = (float)pow(c, pd);
        t->inv_cj[j] = 1.0f / (float)c;
    }
    t->a1 = p;
    t->a2 = (float)(pd * (pd - 1.0) / 2.0);
    t->a3 = (float)(pd * (pd - 1.0) * (pd - 2.0) / 6.0);
}

static float powp(const powp_table *t, float x) {
    const uint32_t b = f2u(x);
    const uint32_t e = b >> 23;
    const uint32_t j = (b >> 18) & 31u;
    const float m = u2f((b & 0x007FFFFFu) | 0x3F800000u);   /* mantissa in [1,2) */
    const float r = fmaf(m, t->inv_cj[j], -1.0f);            /* m / c_j - 1       */
    const float poly = fmaf(fmaf(fmaf(r, t->a3, t->a2), r, t->a1), r, 1.0f);
    return (t->two_pk[e] * t->cj_p[j]) * poly;
}

/* ------------------------------------------------------------------------- */
/* PSUM: pairwise sum over contiguous halves, n a power of two               */
/* ------------------------------------------------------------------------- */
static float psum(const float *x, int n) {
    if (n == 1) return x[0];
    const int h = n / 2;
    return psum(x, h) + psum(x + h, h);
}

static float clamp_code(float v, float L) {
    /* round(.) of Q, half to even (current rounding mode is nearest), then
       clamped so that the code fits in b bits */
    return fminf(fmaxf(rintf(v), 0.0f), L);
}

/* ------------------------------------------------------------------------- */
/* One group of the solver                                                    */
/* ------------------------------------------------------------------------- */
typedef struct {
    float p, beta, kappa;
    int iters, G, nbits;
    powp_table tp;   /* exponent p     : the l_p error            */
    powp_table tq;   /* exponent p - 1 : the generalised shrink    */
} solver_cfg;

typedef struct {        /* optional per-iteration record of one group */
    float *z;           /* [iters] z used by evaluation t            */
    float *e;           /* [iters] error of evaluation t             */
    float *beta;        /* [iters] beta used by the shrink after t   */
    float *q;           /* [iters*G] codes of evaluation t           */
    float *d;           /* [iters*G] residual W - Q^-1(Q(W))         */
    float *we;          /* [iters*G] W_e from sp1 (accepted t only)  */
} group_trace;

typedef struct {
    float s, inv, z0, z_best, e_best;
    int accepted, evaluations;
} group_result;

static void solve_group(const float *w, const solver_cfg *cfg, uint8_t *codes,
                        group_result *res, group_trace *tr) {
    const int G = cfg->G;
    const float L = (float)((1 << cfg->nbits) - 1);
    float q[HQQ_ORACLE_MAX_GROUP], d[HQQ_ORACLE_MAX_GROUP];
    float pw[HQQ_ORACLE_MAX_GROUP], term[HQQ_ORACLE_MAX_GROUP];

    /* min-max initialisation */
    float mn = w[0], mx = w[0];
    for (int i = 1; i < G; ++i) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    const float rng = mx - mn;
    float s, inv;
    if (rng == 0.0f) {
        s = 1.0f;
        inv = 1.0f;
    } else {
        s = rng / L;
        inv = 1.0f / s;      /* the solver holds 1/s */
    }
    float z = -(mn * inv);
    float z_best = z, e_best = INFINITY, beta_t = cfg->beta;
    int accepted = 0, evaluations = 0;

    for (int t = 0; t < cfg->iters; ++t) {
        /* Wq = round(W/s + z);  residual W - s(Wq - z);  error sum |.|^p */
        for (int i = 0; i < G; ++i) {
            q[i] = clamp_code(fmaf(w[i], inv, z), L);
            d[i] = fmaf(z - q[i], s, w[i]);
            pw[i] = powp(&cfg->tp, fabsf(d[i]));
        }
        const float e = psum(pw, G);
        ++evaluations;
        if (tr) {
            tr->z[t] = z;
            tr->e[t] = e;
            tr->beta[t] = beta_t;
            memcpy(tr->q + (size_t)t * G, q, sizeof(float) * G);
            memcpy(tr->d + (size_t)t * G, d, sizeof(float) * G);
        }
        if (!(e < e_best)) break;           /* error stopped falling */
        e_best = e;
        z_best = z;
        ++accepted;

        /* sp1: W_e = shrink_lp(residual, beta);  sp2: z = <Wq - (W - W_e)/s> */
        for (int i = 0; i < G; ++i) {
            const float a = fabsf(d[i]);
            const float y = a - powp(&cfg->tq, a) / beta_t;
            const float we = copysignf(fmaxf(y, 0.0f), d[i]);
            if (tr) tr->we[(size_t)t * G + i] = we;
            term[i] = fmaf(-(w[i] - we), inv, q[i]);
        }
        z = psum(term, G) * (1.0f / (float)G);
        beta_t = beta_t * cfg->kappa;
    }

    for (int i = 0; i < G; ++i)
        codes[i] = (uint8_t)clamp_code(fmaf(w[i], inv, z_best), L);

    res->s = s;
    res->inv = inv;
    res->z0 = -(mn * inv);
    res->z_best = z_best;
    res->e_best = e_best;
    res->accepted = accepted;
    res->evaluations = evaluations;
}

/* ------------------------------------------------------------------------- */
/* The same solver in half precision                                         */
/* ------------------------------------------------------------------------- */
/* Section 2.2 of the page holds 1/s because it "is more stable in half
   precision", and section 3 runs the whole solve on the GPU in half precision.
   The page fixes no rounding step; the readings taken:
     - every element-wise step takes fp16 operands and rounds its result once
       to fp16 (round to nearest even), with no fused multiply-add; computing
       a +, -, * or / of fp16 values in binary32 and rounding to fp16 gives the
       correctly rounded fp16 result (24 >= 2*11 + 2 bits), so h(a op b) below
       is exact fp16 arithmetic;
     - the group reductions (the error and the sp2 mean) accumulate in
       binary32, in the PSUM order, and round the result once to fp16;
     - the error is the group MEAN of |W - s(Wq - z)|^p (never overflows
       fp16), compared in fp16;
     - |x|^p and |x|^(p-1) are powp of the fp16 value, rounded to fp16;
     - the hyper-parameters p, beta, kappa stay binary32 scalars: beta_t is
       the binary32 schedule of the single-precision solver, and the shrink
       divides its fp16 power by it and rounds to fp16;
     - initialisation: r = h(max - min), s = h(r / L), 1/s = h(1 / s),
       z = -h(min * (1/s)); a constant group has s = 1/s = 1, z = -min;
     - fp16 cannot hold every intermediate of every group: a group whose
       largest |W| exceeds 8192, whose s rounds to zero, or whose
       max|W| * (1/s) exceeds 2^14 (binary32 product) is solved by the
       single-precision solver above instead.  Inside those bounds the
       starting point and every update with W_e = 0 stay in the fp16 range
       (|W/s| <= 2^14, |z| <= 2^14 + L, |s (Wq - z)| <= 2 (max - min) +
       max|W|); an update that an active shrink drives out of range gives an
       infinite error at its evaluation and is never accepted. */
static float h16(float x) { return half_bits_to_float(float_to_half_bits(x)); }

/* 1 when the group is solved in half precision (see above), with its fp16
   s, 1/s and starting z. */
static int half_init(const float *w, int G, float L, float *s, float *inv, float *z) {
    float mn = w[0], mx = w[0];
    for (int i = 1; i < G; ++i) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    const float rng = h16(mx - mn);
    if (rng == 0.0f) {
        *s = 1.0f;
        *inv = 1.0f;
        *z = -mn;
        return 1;
    }
    const float m = fmaxf(fabsf(mn), fabsf(mx));
    *s = h16(rng / L);
    *inv = h16(1.0f / *s);
    if (!(m <= 8192.0f) || !(*s > 0.0f) || !(m * *inv <= 16384.0f)) return 0;
    *z = -h16(mn * *inv);
    return 1;
}

static void solve_group_half(const float *w, const solver_cfg *cfg, uint8_t *codes,
                             group_result *res, group_trace *tr, int *half) {
    const int G = cfg->G;
    const float L = (float)((1 << cfg->nbits) - 1);
    float s, inv, z;
    if (!half_init(w, G, L, &s, &inv, &z)) {
        *half = 0;
        solve_group(w, cfg, codes, res, tr);
        return;
    }
    *half = 1;
    float u[HQQ_ORACLE_MAX_GROUP], q[HQQ_ORACLE_MAX_GROUP], d[HQQ_ORACLE_MAX_GROUP];
    float pw[HQQ_ORACLE_MAX_GROUP], term[HQQ_ORACLE_MAX_GROUP];
    for (int i = 0; i < G; ++i) u[i] = h16(w[i] * inv);          /* W / s, held as W * (1/s) */
    const float z0 = z;
    float z_best = z, e_best = INFINITY, beta_t = cfg->beta;
    int accepted = 0, evaluations = 0;

    for (int t = 0; t < cfg->iters; ++t) {
        /* Wq = round(W/s + z);  residual W - s(Wq - z);  mean of |.|^p */
        for (int i = 0; i < G; ++i) {
            q[i] = clamp_code(h16(u[i] + z), L);
            d[i] = h16(w[i] - h16(s * h16(q[i] - z)));
            pw[i] = h16(powp(&cfg->tp, fabsf(d[i])));
        }
        const float e = h16(psum(pw, G) * (1.0f / (float)G));
        ++evaluations;
        if (tr) {
            tr->z[t] = z;
            tr->e[t] = e;
            tr->beta[t] = beta_t;
            memcpy(tr->q + (size_t)t * G, q, sizeof(float) * G);
            memcpy(tr->d + (size_t)t * G, d, sizeof(float) * G);
        }
        if (!(e < e_best)) break;           /* error stopped falling */
        e_best = e;
        z_best = z;
        ++accepted;

        /* sp1: W_e = shrink_lp(residual, beta);  sp2: z = <Wq - (W - W_e)/s> */
        for (int i = 0; i < G; ++i) {
            const float a = fabsf(d[i]);
            const float y = h16(a - h16(h16(powp(&cfg->tq, a)) / beta_t));
            const float we = copysignf(fmaxf(y, 0.0f), d[i]);
            if (tr) tr->we[(size_t)t * G + i] = we;
            term[i] = h16(q[i] - h16(h16(w[i] - we) * inv));
        }
        z = h16(psum(term, G) * (1.0f / (float)G));
        beta_t = beta_t * cfg->kappa;
    }

    for (int i = 0; i < G; ++i) codes[i] = (uint8_t)clamp_code(h16(u[i] + z_best), L);

    res->s = s;
    res->inv = inv;
    res->z0 = z0;
    res->z_best = z_best;
    res->e_best = e_best;
    res->accepted = accepted;
    res->evaluations = evaluations;
}

/* ------------------------------------------------------------------------- */
/* Exported entry points (test infrastructure)                               */
/* ------------------------------------------------------------------------- */
static int check_cfg(int nbits, int G, float p, float beta, float kappa, int iters) {
    if (nbits < 1 || nbits > 8) return 3;
    if (G < 1 || G > HQQ_ORACLE_MAX_GROUP || (G & (G - 1)) != 0) return 3;
    if (!(p > 0.0f && p <= 1.0f) || !(beta > 0.0f) || !(kappa > 0.0f)) return 4;
    if (iters < 0 || iters > 255) return 4;
    return 0;
}

static void cfg_init(solver_cfg *cfg, int nbits, int G, float p, float beta,
                     float kappa, int iters) {
    cfg->p = p;
    cfg->beta = beta;
    cfg->kappa = kappa;
    cfg->iters = iters;
    cfg->G = G;
    cfg->nbits = nbits;
    powp_table_init(&cfg->tp, p);
    powp_table_init(&cfg->tq, p - 1.0f);
}

typedef struct {
    const solver_cfg *cfg;
    const uint16_t *W;
    int64_t g0, g1;
    uint8_t *codes;
    uint16_t *scale, *zero;
    float *zero_f32, *scale_f32, *err;
    uint8_t *iters_out;
    int half;            /* 1: the half-precision solver                 */
    uint8_t *half_out;   /* per group: 1 when it was solved in fp16      */
} work_range;

static void *run_range(void *arg) {
    const work_range *wr = (const work_range *)arg;
    const int G = wr->cfg->G;
    float w[HQQ_ORACLE_MAX_GROUP];
    for (int64_t g = wr->g0; g < wr->g1; ++g) {
        const uint16_t *src = wr->W + g * G;
        for (int i = 0; i < G; ++i) w[i] = half_bits_to_float(src[i]);
        group_result r;
        int h = 0;
        if (wr->half)
            solve_group_half(w, wr->cfg, wr->codes + g * G, &r, NULL, &h);
        else
            solve_group(w, wr->cfg, wr->codes + g * G, &r, NULL);
        if (wr->half_out) wr->half_out[g] = (uint8_t)h;
        wr->scale[g] = float_to_half_bits(r.s);
        wr->zero[g] = float_to_half_bits(r.z_best);
        if (wr->zero_f32) wr->zero_f32[g] = r.z_best;
        if (wr->scale_f32) wr->scale_f32[g] = r.s;
        if (wr->err) wr->err[g] = r.e_best;
        if (wr->iters_out) wr->iters_out[g] = (uint8_t)r.accepted;
    }
    return NULL;
}

/* Quantize n_groups contiguous groups of G fp16 weights (row-major [out,in]
   with in % G == 0 is exactly this flat layout).  codes: one byte per weight.
   scale/zero: fp16 bits per group.  zero_f32/scale_f32/err/iters_out nullable;
   err is the accepted minimum of the error sum (+inf when iters = 0). */
static int quantize_groups(const uint16_t *W, int64_t n_groups, int G, int nbits,
                           float p, float beta, float kappa, int iters, int nthreads,
                           uint8_t *codes, uint16_t *scale, uint16_t *zero,
                           float *zero_f32, float *scale_f32, float *err, uint8_t *iters_out,
                           int half, uint8_t *half_out) {
    const int st = check_cfg(nbits, G, p, beta, kappa, iters);
    if (st) return st;
    if (n_groups <= 0) return 0;
    solver_cfg cfg;
    cfg_init(&cfg, nbits, G, p, beta, kappa, iters);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > n_groups) nthreads = (int)n_groups;
    pthread_t th[256];
    work_range wr[256];
    for (int k = 0; k < nthreads; ++k) {
        wr[k].cfg = &cfg;
        wr[k].W = W;
        wr[k].g0 = n_groups * k / nthreads;
        wr[k].g1 = n_groups * (k + 1) / nthreads;
        wr[k].codes = codes;
        wr[k].scale = scale;
        wr[k].zero = zero;
        wr[k].zero_f32 = zero_f32;
        wr[k].scale_f32 = scale_f32;
        wr[k].err = err;
        wr[k].iters_out = iters_out;
        wr[k].half = half;
        wr[k].half_out = half_out;
    }
    if (nthreads == 1) {
        run_range(&wr[0]);
        return 0;
    }
    for (int k = 0; k < nthreads; ++k) pthread_create(&th[k], NULL, run_range, &wr[k]);
    for (int k = 0; k < nthreads; ++k) pthread_join(th[k], NULL);
    return 0;
}

int hqq_oracle_quantize(const uint16_t *W, int64_t n_groups, int G, int nbits,
                        float p, float beta, float kappa, int iters, int nthreads,
                        uint8_t *codes, uint16_t *scale, uint16_t *zero,
                        float *zero_f32, float *scale_f32, float *err, uint8_t *iters_out) {
    return quantize_groups(W, n_groups, G, nbits, p, beta, kappa, iters, nthreads, codes,
                           scale, zero, zero_f32, scale_f32, err, iters_out, 0, NULL);
}

/* The half-precision solver over the same layout; err is the accepted minimum
   of the group's mean error in fp16 (of its binary32 error sum for a group
   outside the fp16 bounds, which half_out marks 0). */
int hqq_oracle_quantize_half(const uint16_t *W, int64_t n_groups, int G, int nbits,
                             float p, float beta, float kappa, int iters, int nthreads,
                             uint8_t *codes, uint16_t *scale, uint16_t *zero,
                             float *zero_f32, float *scale_f32, float *err,
                             uint8_t *iters_out, uint8_t *half_out) {
    return quantize_groups(W, n_groups, G, nbits, p, beta, kappa, iters, nthreads, codes,
                           scale, zero, zero_f32, scale_f32, err, iters_out, 1, half_out);
}

/* One group in fp32 with its full per-iteration record (for the pins). */
int hqq_oracle_trace_group(const float *w, int G, int nbits, float p, float beta,
                           float kappa, int iters, uint8_t *codes, float *out6,
                           int *counts2, float *z, float *e, float *beta_hist,
                           float *q, float *d, float *we) {
    const int st = check_cfg(nbits, G, p, beta, kappa, iters);
    if (st) return st;
    solver_cfg cfg;
    cfg_init(&cfg, nbits, G, p, beta, kappa, iters);
    group_trace tr = {z, e, beta_hist, q, d, we};
    group_result r;
    solve_group(w, &cfg, codes, &r, &tr);
    out6[0] = r.s;
    out6[1] = r.inv;
    out6[2] = r.z0;
    out6[3] = r.z_best;
    out6[4] = r.e_best;
    out6[5] = 0.0f;
    counts2[0] = r.accepted;
    counts2[1] = r.evaluations;
    return 0;
}

/* One group of the half-precision solver with its record; counts2[2] receives
   1 when the group was solved in fp16. */
int hqq_oracle_trace_group_half(const float *w, int G, int nbits, float p, float beta,
                                float kappa, int iters, uint8_t *codes, float *out6,
                                int *counts3, float *z, float *e, float *beta_hist,
                                float *q, float *d, float *we) {
    const int st = check_cfg(nbits, G, p, beta, kappa, iters);
    if (st) return st;
    solver_cfg cfg;
    cfg_init(&cfg, nbits, G, p, beta, kappa, iters);
    group_trace tr = {z, e, beta_hist, q, d, we};
    group_result r;
    int h = 0;
    solve_group_half(w, &cfg, codes, &r, &tr, &h);
    out6[0] = r.s;
    out6[1] = r.inv;
    out6[2] = r.z0;
    out6[3] = r.z_best;
    out6[4] = r.e_best;
    out6[5] = 0.0f;
    counts3[0] = r.accepted;
    counts3[1] = r.evaluations;
    counts3[2] = h;
    return 0;
}

/* The sp1 operator alone: we[i] = shrink_lp(x[i], beta) with exponent p. */
void hqq_oracle_shrink(const float *x, int64_t n, float p, float beta, float *we) {
    powp_table tq;
    powp_table_init(&tq, p - 1.0f);
    for (int64_t i = 0; i < n; ++i) {
        const float a = fabsf(x[i]);
        const float y = a - powp(&tq, a) / beta;
        we[i] = copysignf(fmaxf(y, 0.0f), x[i]);
    }
}

/* The sp2 update alone for one group: z = PSUM(Wq - (W - W_e)/s) / G. */
float hqq_oracle_z_update(const float *w, const float *q, const float *we, int G,
                          float inv) {
    float term[HQQ_ORACLE_MAX_GROUP];
    for (int i = 0; i < G; ++i) term[i] = fmaf(-(w[i] - we[i]), inv, q[i]);
    return psum(term, G) * (1.0f / (float)G);
}

/* y[i] = powp(x[i], p), and the table entries used (for the pins). */
void hqq_oracle_powp(const float *x, int64_t n, float p, float *y) {
    powp_table t;
    powp_table_init(&t, p);
    for (int64_t i = 0; i < n; ++i) y[i] = powp(&t, x[i]);
}

void hqq_oracle_powp_table(float p, float *two_pk256, float *cj_p32, float *inv_cj32,
                           float *a3) {
    powp_table t;
    powp_table_init(&t, p);
    memcpy(two_pk256, t.two_pk, sizeof t.two_pk);
    memcpy(cj_p32, t.cj_p, sizeof t.cj_p);
    memcpy(inv_cj32, t.inv_cj, sizeof t.inv_cj);
    a3[0] = t.a1;
    a3[1] = t.a2;
    a3[2] = t.a3;
}

/* Pairwise sum (exposed so the pins can check its order). */
float hqq_oracle_psum(const float *x, int n) { return psum(x, n); }

/* Packing over the flat row-major element index.
   8 bit: one code per byte.
   4 bit: two codes per byte, even index in the low nibble.
   2 bit: four codes per byte, first code in the least significant bits.
   1 bit: eight codes per byte, first code in the least significant bit.
   3 bit: ten codes per little-endian 32-bit word in bits 0..29; bits 30..31
          and the codes past the end of the last word are zero. */
int64_t hqq_oracle_packed_bytes(int64_t n, int nbits) {
    if (n < 0) return -1;
    if (nbits == 8) return n;
    if (nbits == 4) return (n + 1) / 2;
    if (nbits == 2) return (n + 3) / 4;
    if (nbits == 1) return (n + 7) / 8;
    if (nbits == 3) return 4 * ((n + 9) / 10);
    return -1;
}

int hqq_oracle_pack(const uint8_t *codes, int64_t n, int nbits, uint8_t *out) {
    const int64_t nb = hqq_oracle_packed_bytes(n, nbits);
    if (nb < 0) return 3;
    memset(out, 0, (size_t)nb);
    for (int64_t i = 0; i < n; ++i) {
        const uint32_t c = codes[i];
        if (nbits < 8 && (c >> nbits)) return 4;
        if (nbits == 8) {
            out[i] = (uint8_t)c;
        } else if (nbits == 1) {
            out[i / 8] |= (uint8_t)(c << (i % 8));
        } else if (nbits == 4) {
            out[i / 2] |= (uint8_t)(c << (4 * (i % 2)));
        } else if (nbits == 2) {
            out[i / 4] |= (uint8_t)(c << (2 * (i % 4)));
        } else {
            const int64_t word = i / 10;
            const uint32_t bit = 3u * (uint32_t)(i % 10);
            const uint32_t v = c << bit;
            for (int k = 0; k < 4; ++k) out[4 * word + k] |= (uint8_t)(v >> (8 * k));
        }
    }
    return 0;
}

int hqq_oracle_unpack(const uint8_t *packed, int64_t n, int nbits, uint8_t *codes) {
    if (hqq_oracle_packed_bytes(n, nbits) < 0) return 3;
    for (int64_t i = 0; i < n; ++i) {
        if (nbits == 8) {
            codes[i] = packed[i];
        } else if (nbits == 1) {
            codes[i] = (packed[i / 8] >> (i % 8)) & 1u;
        } else if (nbits == 4) {
            codes[i] = (packed[i / 2] >> (4 * (i % 2))) & 15u;
        } else if (nbits == 2) {
            codes[i] = (packed[i / 4] >> (2 * (i % 4))) & 3u;
        } else {
            const int64_t word = i / 10;
            uint32_t v = 0;
            for (int k = 0; k < 4; ++k) v |= (uint32_t)packed[4 * word + k] << (8 * k);
            codes[i] = (v >> (3u * (uint32_t)(i % 10))) & 7u;
        }
    }
    return 0;
}

/* Q^-1: W_hat = fp16( (c - z) * s ) with z, s the stored fp16 values. */
int hqq_oracle_dequantize(const uint8_t *codes, const uint16_t *scale,
                          const uint16_t *zero, int64_t n, int G, uint16_t *W_hat) {
    if (G < 1) return 3;
    for (int64_t i = 0; i < n; ++i) {
        const float s = half_bits_to_float(scale[i / G]);
        const float z = half_bits_to_float(zero[i / G]);
        W_hat[i] = float_to_half_bits(((float)codes[i] - z) * s);
    }
    return 0;
}

/* fp16 conversions exposed for the pins. */
void hqq_oracle_f32_to_f16(const float *x, int64_t n, uint16_t *h) {
    for (int64_t i = 0; i < n; ++i) h[i] = float_to_half_bits(x[i]);
}

/* ------------------------------------------------------------------------- */
/* 8-bit meta-quantization of the stored zero points and scales              */
/* ------------------------------------------------------------------------- */
/* Section 4.1 ("Llama-2 benchmarks") of the page quantizes the zero points to
   8 bits with neither grouping nor optimisation, and in its table's starred
   row also the scales, to 8 bits in groups of 128.  Readings taken:
     - "without optimisation" is section 2's Q with its min-max start and no
       solver iterations: s = (max-min)/255 (s = 1 for a constant group),
       1/s held, z = -min * (1/s), c = clamp(round(x * (1/s) + z), 0, 255);
     - the input is the stored fp16 tensor in flat row-major order; groups are
       `group` consecutive values and the last one may be shorter; group 0
       means one group over all n values ("without grouping");
     - each group's own scale and zero are stored in fp16 like the weights';
     - the arithmetic is the weights' canonical binary32 sequence. */
int hqq_oracle_meta_quantize(const uint16_t *x, int64_t n, int64_t group,
                             uint8_t *codes, uint16_t *scale, uint16_t *zero) {
    if (n < 0 || group < 0) return 3;
    const float L = 255.0f;
    const int64_t len = group == 0 ? n : group;
    for (int64_t g0 = 0, gi = 0; g0 < n; g0 += len, ++gi) {
        const int64_t m = n - g0 < len ? n - g0 : len;
        float mn = half_bits_to_float(x[g0]), mx = mn;
        for (int64_t i = 1; i < m; ++i) {
            const float v = half_bits_to_float(x[g0 + i]);
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        const float rng = mx - mn;
        float s, inv;
        if (rng == 0.0f) {
            s = 1.0f;
            inv = 1.0f;
        } else {
            s = rng / L;
            inv = 1.0f / s;
        }
        const float z = -(mn * inv);
        for (int64_t i = 0; i < m; ++i)
            codes[g0 + i] = (uint8_t)clamp_code(fmaf(half_bits_to_float(x[g0 + i]), inv, z), L);
        scale[gi] = float_to_half_bits(s);
        zero[gi] = float_to_half_bits(z);
    }
    return 0;
}

/* Its inverse, section 2's Q^-1 on the 8-bit codes: fp16((c - z) * s) with the
   group's stored fp16 s and z (group 0: one group over all n values). */
int hqq_oracle_meta_dequantize(const uint8_t *codes, const uint16_t *scale,
                               const uint16_t *zero, int64_t n, int64_t group,
                               uint16_t *out) {
    if (n < 0 || group < 0) return 3;
    const int64_t len = group == 0 ? (n > 0 ? n : 1) : group;
    for (int64_t i = 0; i < n; ++i) {
        const float s = half_bits_to_float(scale[i / len]);
        const float z = half_bits_to_float(zero[i / len]);
        out[i] = float_to_half_bits(((float)codes[i] - z) * s);
    }
    return 0;
}
