/*
 * lapsum_oracle.c -- plain, slow fp64 CPU oracle for the exact-budget LapSum
 * soft top-k ("Fast LapSum: Exact Differentiable Top-k at Million Scale").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: it is used by tests/, by __graft_entry__.smoke() and by the
 * CPU-baseline leg of bench.py.  It shares no code with the CUDA library.
 *
 * What it computes (page "gist.science/paper/2608.06912", Technical Summary):
 *   section 2.1 -- memberships p_i = F((r_i - b)/alpha), F the Laplace CDF,
 *                  with b fixed by  sum_i p_i = k;  an analytic VJP backward.
 *   section 2.2 -- full-sort solver: sort, one prefix/suffix pass over the
 *                  sorted scores, look up the interval where the budget
 *                  balances, closed-form root inside it.
 *   section 2.2 -- localization: kernel-noised samples and binomial order
 *                  statistics give a bracket [a_L, a_R) around b; the stream
 *                  step aggregates the scores outside it into tail sums.
 *
 * Conventions (plainest reading of the pages):
 *   F(z) = exp(z)/2 for z < 0, 1 - exp(-z)/2 for z >= 0; alpha is the Laplace
 *   scale t; k is real with 0 < k < n; larger scores get larger p.
 *   Backward: differentiating sum_i F((r_i - b)/alpha) = k gives
 *   db/dr_j = f_j / sum f, hence grad_j = f_j (g_j - lambda) with
 *   f_j = exp(-|r_j - b|/alpha) / (2 alpha), lambda = sum g f / sum f,
 *   and dL/dk = lambda.
 *   The noise kernel is Laplace(0, alpha), so P(r_I + eps > b) = k/n exactly.
 *   Random numbers: splitmix64 (Steele, Lea & Flood, "Fast splittable
 *   pseudorandom number generators", OOPSLA 2014), used counter-style.
 *
 * Every function works in fp64.  Plausible-mistake variants for the pin tests
 * are compiled in only with -DLO_MUTANT=<n>; the default build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef LO_MUTANT
#define LO_MUTANT 0
#endif

#define LO_OK 0
#define LO_EINVAL 1
#define LO_EBADK 2
#define LO_EBADALPHA 3
#define LO_ENOMEM 4
#define LO_ENONFINITE 5

/* ------------------------------------------------------------------ */
/* small helpers                                                       */
/* ------------------------------------------------------------------ */

/* Laplace CDF, section 2.1 */
static double lap_cdf(double z) { return z < 0.0 ? 0.5 * exp(z) : 1.0 - 0.5 * exp(-z); }

/* Neumaier-compensated running sum */
typedef struct { double s, c; } nsum;
static void nsum_add(nsum* a, double x) {
    double t = a->s + x;
    if (fabs(a->s) >= fabs(x)) a->c += (a->s - t) + x;
    else a->c += (x - t) + a->s;
    a->s = t;
}
static double nsum_get(const nsum* a) { return a->s + a->c; }

static int cmp_double(const void* pa, const void* pb) {
    double a = *(const double*)pa, b = *(const double*)pb;
    return (a > b) - (a < b);
}

/* IEEE totalOrder on finite floats: -0 sorts before +0 */
static int cmp_float_total(const void* pa, const void* pb) {
    float a = *(const float*)pa, b = *(const float*)pb;
    if (a < b) return -1;
    if (a > b) return 1;
    int sa = signbit(a) != 0, sb = signbit(b) != 0;
    return sb - sa;
}

static int check_args(int64_t n, double k, double alpha) {
    if (n < 1) return LO_EINVAL;
    if (!isfinite(k) || !(k > 0.0) || !(k < (double)n)) return LO_EBADK;
    if (!isfinite(alpha) || !(alpha > 0.0)) return LO_EBADALPHA;
    return LO_OK;
}

/* ln(m + sqrt(m^2 + e^L)) for m >= 0, without overflow or underflow. */
static double lnsum(double m, double L) {
    if (m == 0.0) return 0.5 * L;
    double lm = log(m);
    double D = L - 2.0 * lm;
    if (D > 0.0) return 0.5 * L + log(exp(-0.5 * D) + sqrt(exp(-D) + 1.0));
    return lm + log(1.0 + sqrt(1.0 + exp(D)));
}

/* ------------------------------------------------------------------ */
/* the threshold b: full sort + threshold curve + closed-form root     */
/* ------------------------------------------------------------------ */

/*
 * Sorted scores x_0 <= ... <= x_{n-1}.  For a knot j:
 *   A_j  = sum_{l <= j} exp((x_l - x_j)/alpha)       (prefix, anchored at x_j)
 *   Bp_j = sum_{l >= j} exp((x_j - x_l)/alpha)       (suffix, anchored at x_j)
 *   S(x_j) = A_j/2 + (n-1-j) - (Bp_{j+1} exp((x_j - x_{j+1})/alpha))/2
 * S is strictly decreasing in b, so the root lies in [x_j*, x_j*+1) with j*
 * the last knot where S(x_j) >= k (j* = -1 when b < x_0).  On that interval,
 * with u = exp((b - x_j)/alpha), c = n-1-j and mu = c - k, the budget equation
 * A/(2u) + c - B u/2 = k becomes B u^2 - 2 mu u - A = 0 (B the strict suffix).
 * The positive root is taken anchored at the right knot when mu >= 0 and at
 * the left knot when mu < 0, in log form so that neither anchor overflows.
 */
int lo_threshold_f64(const double* r, int64_t n, double k, double alpha, double* b_out) {
    int rc = check_args(n, k, alpha);
    if (rc) return rc;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(r[i])) return LO_ENONFINITE;
    double* x = (double*)malloc(sizeof(double) * (size_t)n);
    double* Bp = (double*)malloc(sizeof(double) * (size_t)n);
    if (!x || !Bp) { free(x); free(Bp); return LO_ENOMEM; }
    memcpy(x, r, sizeof(double) * (size_t)n);
    qsort(x, (size_t)n, sizeof(double), cmp_double);

    /* suffix pass */
    Bp[n - 1] = 1.0;
    for (int64_t j = n - 2; j >= 0; --j) {
#if LO_MUTANT == 2
        Bp[j] = Bp[j + 1] * exp((x[j + 1] - x[j]) / alpha) + 1.0; /* wrong sign */
#else
        Bp[j] = Bp[j + 1] * exp((x[j] - x[j + 1]) / alpha) + 1.0;
#endif
    }

    /* prefix pass + knot values */
    int64_t jstar = -1;
    double Astar = 0.0, A = 0.0;
    for (int64_t j = 0; j < n; ++j) {
#if LO_MUTANT == 1
        A = (j == 0) ? 1.0 : A * exp((x[j - 1] - x[j]) / alpha); /* dropped +1 */
#else
        A = (j == 0) ? 1.0 : A * exp((x[j - 1] - x[j]) / alpha) + 1.0;
#endif
        double Bs = (j + 1 < n) ? Bp[j + 1] * exp((x[j] - x[j + 1]) / alpha) : 0.0;
        double S = 0.5 * A + (double)(n - 1 - j) - 0.5 * Bs;
        if (S >= k) { jstar = j; Astar = A; }
        else break;
    }

    double c = (double)(n - 1 - jstar);
    double mu = c - k;
    double lnA = (jstar >= 0) ? log(Astar) : -INFINITY;
    double lnBp = (jstar + 1 < n) ? log(Bp[jstar + 1]) : -INFINITY;
    double L = -INFINITY;
    if (jstar >= 0 && jstar + 1 < n) L = lnA + lnBp - (x[jstar + 1] - x[jstar]) / alpha;
    double b;
#if LO_MUTANT == 3
    if (jstar >= 0) b = x[jstar] + alpha * (lnA - lnsum(fabs(mu), L)); /* ignores sign of mu */
    else b = x[0] + alpha * (lnsum(mu, L) - lnBp);
#else
    if (mu >= 0.0) b = x[jstar + 1] + alpha * (lnsum(mu, L) - lnBp);
    else b = x[jstar] + alpha * (lnA - lnsum(-mu, L));
#endif
    if (jstar >= 0 && b < x[jstar]) b = x[jstar];
    if (jstar + 1 < n && b > x[jstar + 1]) b = x[jstar + 1];
    *b_out = b;
    free(x);
    free(Bp);
    return LO_OK;
}

/* S(b) = sum_i F((r_i - b)/alpha), summed directly with compensation. */
double lo_S_f64(const double* r, int64_t n, double b, double alpha) {
    nsum a = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) nsum_add(&a, lap_cdf((r[i] - b) / alpha));
    return nsum_get(&a);
}

/* memberships p (fp64) and sum_i f_i for the solved b */
int lo_forward_f64(const double* r, int64_t n, double k, double alpha,
                   double* p_out, double* b_out, double* sumf_out) {
    double b;
    int rc = lo_threshold_f64(r, n, k, alpha, &b);
    if (rc) return rc;
    nsum sf = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
        double z = (r[i] - b) / alpha;
        if (p_out) p_out[i] = lap_cdf(z);
        nsum_add(&sf, 0.5 * exp(-fabs(z)) / alpha);
    }
    if (b_out) *b_out = b;
    if (sumf_out) *sumf_out = nsum_get(&sf);
    return LO_OK;
}

/* VJP: grad_j = f_j (g_j - lambda), lambda = sum g f / sum f  (= dL/dk) */
int lo_backward_f64(const double* r, const double* g, int64_t n, double b, double alpha,
                    double* grad_out, double* lambda_out, double* sumf_out) {
    if (n < 1) return LO_EINVAL;
    if (!isfinite(alpha) || !(alpha > 0.0)) return LO_EBADALPHA;
    nsum sgf = {0.0, 0.0}, sf = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
        double f = 0.5 * exp(-fabs(r[i] - b) / alpha) / alpha;
        nsum_add(&sf, f);
        nsum_add(&sgf, g[i] * f);
    }
    double SF = nsum_get(&sf);
    double lam = nsum_get(&sgf) / SF;
    for (int64_t i = 0; i < n; ++i) {
        double f = 0.5 * exp(-fabs(r[i] - b) / alpha) / alpha;
#if LO_MUTANT == 4
        grad_out[i] = f * g[i]; /* dropped the budget term */
#else
        grad_out[i] = f * (g[i] - lam);
#endif
    }
    if (lambda_out) *lambda_out = lam;
    if (sumf_out) *sumf_out = SF;
    return LO_OK;
}

/*
 * dL/dalpha for the loss L = sum_j g_j p_j (technical summary section 2.1:
 * the budget constraint ties b to alpha).  Differentiating
 * sum_i F((r_i - b)/alpha) = k with respect to alpha gives
 *     db/dalpha = - sum_i f_i z_i / sum_i f_i,   z_i = (r_i - b)/alpha,
 * and then, term by term,
 *     dp_j/dalpha = f_j (-db/dalpha - z_j),
 *     dL/dalpha   = sum_j g_j dp_j/dalpha.
 */
int lo_backward_alpha_f64(const double* r, const double* g, int64_t n, double b, double alpha,
                          double* dalpha_out) {
    if (n < 1) return LO_EINVAL;
    if (!isfinite(alpha) || !(alpha > 0.0)) return LO_EBADALPHA;
    nsum sf = {0.0, 0.0}, sfz = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
        const double z = (r[i] - b) / alpha;
        const double f = 0.5 * exp(-fabs(z)) / alpha;
        nsum_add(&sf, f);
        nsum_add(&sfz, f * z);
    }
    const double db = -nsum_get(&sfz) / nsum_get(&sf);
    nsum dl = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
        const double z = (r[i] - b) / alpha;
        const double f = 0.5 * exp(-fabs(z)) / alpha;
#if LO_MUTANT == 5
        const double dp = f * (-z); /* dropped the move of b */
#else
        const double dp = f * (-db - z);
#endif
        nsum_add(&dl, g[i] * dp);
    }
    if (dalpha_out) *dalpha_out = nsum_get(&dl);
    return LO_OK;
}

/* ------------------------------------------------------------------ */
/* fp32-input wrappers (the GPU path reads fp32 scores)                */
/* ------------------------------------------------------------------ */

static double* widen(const float* r, int64_t n) {
    double* d = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!d) return NULL;
    for (int64_t i = 0; i < n; ++i) d[i] = (double)r[i];
    return d;
}

int lo_threshold_f32(const float* r, int64_t n, double k, double alpha, double* b_out) {
    double* d = widen(r, n);
    if (!d) return LO_ENOMEM;
    int rc = lo_threshold_f64(d, n, k, alpha, b_out);
    free(d);
    return rc;
}

int lo_forward_f32(const float* r, int64_t n, double k, double alpha,
                   double* p_out, double* b_out, double* sumf_out) {
    double* d = widen(r, n);
    if (!d) return LO_ENOMEM;
    int rc = lo_forward_f64(d, n, k, alpha, p_out, b_out, sumf_out);
    free(d);
    return rc;
}

int lo_backward_f32(const float* r, const float* g, int64_t n, double b, double alpha,
                    double* grad_out, double* lambda_out, double* sumf_out) {
    double* d = widen(r, n);
    double* e = widen(g, n);
    if (!d || !e) { free(d); free(e); return LO_ENOMEM; }
    int rc = lo_backward_f64(d, e, n, b, alpha, grad_out, lambda_out, sumf_out);
    free(d);
    free(e);
    return rc;
}

int lo_backward_alpha_f32(const float* r, const float* g, int64_t n, double b, double alpha,
                          double* dalpha_out) {
    double* d = widen(r, n);
    double* e = widen(g, n);
    if (!d || !e) { free(d); free(e); return LO_ENOMEM; }
    int rc = lo_backward_alpha_f64(d, e, n, b, alpha, dalpha_out);
    free(d);
    free(e);
    return rc;
}

double lo_S_f32(const float* r, int64_t n, double b, double alpha) {
    nsum a = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) nsum_add(&a, lap_cdf(((double)r[i] - b) / alpha));
    return nsum_get(&a);
}

/* ------------------------------------------------------------------ */
/* localization: kernel-noised samples and binomial order statistics   */
/* ------------------------------------------------------------------ */

static const uint64_t SM64_GAMMA = 0x9E3779B97F4A7C15ull;

uint64_t lo_sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* i-th output (i >= 1) of a splitmix64 generator whose state starts at s */
uint64_t lo_sm64_out(uint64_t s, uint64_t i) { return lo_sm64_mix(s + i * SM64_GAMMA); }

/* per-row stream: the (row+1)-th output of a generator seeded with `seed` */
uint64_t lo_row_stream(uint64_t seed, uint64_t row) { return lo_sm64_out(seed, row + 1); }

/*
 * Sample j of a row uses draws 2j+1 (index) and 2j+2 (noise) of the row's
 * stream.  Index: the high 64 bits of draw * n (uniform on [0, n), with
 * replacement).  Noise: u = ((draw >> 11) + 1/2) 2^-53 in (0,1), then the
 * Laplace inverse CDF alpha * (u < 1/2 ? ln(2u) : -ln(2 - 2u)).
 * Y_j = r[I_j] + eps_j is formed in fp64 and rounded to fp32.
 */
void lo_sample(const float* r, int64_t n, double alpha, uint64_t seed, int64_t row, int64_t m,
               float* Y_out, int64_t* idx_out, double* eps_out) {
    uint64_t s = lo_row_stream(seed, (uint64_t)row);
    for (int64_t j = 0; j < m; ++j) {
        uint64_t d1 = lo_sm64_out(s, (uint64_t)(2 * j + 1));
        uint64_t d2 = lo_sm64_out(s, (uint64_t)(2 * j + 2));
        uint64_t I = (uint64_t)(((unsigned __int128)d1 * (unsigned __int128)(uint64_t)n) >> 64);
        double u = ((double)(d2 >> 11) + 0.5) * 0x1p-53;
        double e = (u < 0.5) ? log(2.0 * u) : -log(2.0 - 2.0 * u);
        double eps = alpha * e;
        double Y = (double)r[I] + eps;
        if (Y_out) Y_out[j] = (float)Y;
        if (idx_out) idx_out[j] = (int64_t)I;
        if (eps_out) eps_out[j] = eps;
    }
}

/*
 * #{Y_j > b} ~ Binomial(m, q = k/n).  Ranks (descending, 1-based):
 *   c_lo = floor(mq - z sigma), c_hi = ceil(mq + z sigma), sigma = sqrt(mq(1-q)).
 */
void lo_sample_ranks(int64_t n, double k, int64_t m, double z, int64_t* c_lo, int64_t* c_hi) {
    double q = k / (double)n;
    double mq = (double)m * q;
#if LO_MUTANT == 6
    double sigma = sqrt(mq);  /* MUTANT: the (1 - q) factor of the variance dropped */
#else
    double sigma = sqrt(mq * (1.0 - q));
#endif
    *c_lo = (int64_t)floor(mq - z * sigma);
#if LO_MUTANT == 7
    *c_hi = (int64_t)ceil(mq);  /* MUTANT: the half-width applied on one side only */
#else
    *c_hi = (int64_t)ceil(mq + z * sigma);
#endif
}

/*
 * Bracket [a_L, a_R): a_R is the c_lo-th largest Y (+inf when c_lo < 1),
 * a_L the (c_hi+1)-th largest (-inf when c_hi + 1 > m).
 */
int lo_bracket(const float* r, int64_t n, double k, double alpha, int64_t m, double z,
               uint64_t seed, int64_t row, float* aL, float* aR, int64_t* c_lo_out,
               int64_t* c_hi_out) {
    int rc = check_args(n, k, alpha);
    if (rc) return rc;
    if (m < 1) return LO_EINVAL;
    float* Y = (float*)malloc(sizeof(float) * (size_t)m);
    if (!Y) return LO_ENOMEM;
    lo_sample(r, n, alpha, seed, row, m, Y, NULL, NULL);
    qsort(Y, (size_t)m, sizeof(float), cmp_float_total);
    int64_t c_lo, c_hi;
    lo_sample_ranks(n, k, m, z, &c_lo, &c_hi);
    *aR = (c_lo >= 1) ? Y[m - c_lo] : INFINITY;
    *aL = (c_hi + 1 <= m) ? Y[m - c_hi - 1] : -INFINITY;
    if (c_lo_out) *c_lo_out = c_lo;
    if (c_hi_out) *c_hi_out = c_hi;
    free(Y);
    return LO_OK;
}

/*
 * Stream-and-filter aggregates for a bracket [a_L, a_R):
 *   n_L, S_L = sum_{r < a_L} exp((r - a_L)/alpha);
 *   n_R, S_R = sum_{r >= a_R} exp((a_R - r)/alpha);  M = #{a_L <= r < a_R}.
 */
void lo_tails(const float* r, int64_t n, float aL, float aR, double alpha,
              int64_t* nL, double* SL, int64_t* nR, double* SR, int64_t* M) {
    nsum sl = {0.0, 0.0}, sr = {0.0, 0.0};
    int64_t cl = 0, cr = 0, cm = 0;
    for (int64_t i = 0; i < n; ++i) {
        float x = r[i];
        if (x < aL) { ++cl; nsum_add(&sl, exp(((double)x - (double)aL) / alpha)); }
        else if (x >= aR) { ++cr; nsum_add(&sr, exp(((double)aR - (double)x) / alpha)); }
        else ++cm;
    }
    *nL = cl; *SL = nsum_get(&sl); *nR = cr; *SR = nsum_get(&sr); *M = cm;
}

/*
 * DFTopK-style threshold (section 2.3): the midpoint of the k-th and (k+1)-th
 * largest scores, integer k in [1, n-1].  Used as the zero-temperature limit.
 */
int lo_dftopk_threshold_f32(const float* r, int64_t n, int64_t k, double* b_out) {
    if (n < 2 || k < 1 || k >= n) return LO_EBADK;
    double* x = widen(r, n);
    if (!x) return LO_ENOMEM;
    qsort(x, (size_t)n, sizeof(double), cmp_double);
    *b_out = 0.5 * (x[n - k] + x[n - k - 1]);
    free(x);
    return LO_OK;
}


/*
 * The DFTopK relaxation (technical summary section 2.3): the threshold is
 * fixed at that midpoint instead of solving the budget, and the memberships
 * are the same Laplace CDF at scale alpha; their mass sum_i p_i is then free
 * to drift from k.
 */
int lo_dftopk_forward_f32(const float* r, int64_t n, int64_t k, double alpha, double* p_out, double* b_out,
                          double* mass_out) {
    if (!isfinite(alpha) || !(alpha > 0.0)) return LO_EBADALPHA;
    double b;
    int rc = lo_dftopk_threshold_f32(r, n, k, &b);
    if (rc != LO_OK) return rc;
    nsum mass = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
        const double p = lap_cdf(((double)r[i] - b) / alpha);
        if (p_out) p_out[i] = p;
        nsum_add(&mass, p);
    }
    if (b_out) *b_out = b;
    if (mass_out) *mass_out = nsum_get(&mass);
    return LO_OK;
}
