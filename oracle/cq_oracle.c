/*
 * Exhaustive CPU oracle for exact minimax FP16 group-scale selection.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA path.
 *
 * What it computes (CliffQuant project page, "What CliffQuant changes"):
 * for a group of weights w_i and E environment diagonals d_{e,i}, the scale
 *
 *     s* = argmin_s  max_e  sum_i d_{e,i} * (w_i - s * q_i(s))^2
 *
 * over every positive finite IEEE binary16 value s (bit patterns 0x0001 ..
 * 0x7BFF, the page's 31,743 values), with
 *
 *     q_i(s) = clip(round-half-even(w_i / s), qmin, qmax),   qmin=-8, qmax=7
 *
 * (QuantizerSpec(qmin=-8, qmax=7) in the page's "Use the solver" example),
 * and an exact objective tie going to the lower FP16 bit pattern.
 *
 * The objective is evaluated in fp64 (the pages fix no precision; the
 * exhaustive reference they describe enumerates every FP16 value).  For each
 * scale the order is fixed: codes first, then for every environment e
 *     acc = 0;  for i = 0..n-1:  r = w_i - s*q_i;  acc = acc + d_{e,i}*(r*r)
 * and f = max_e acc.  Build with -ffp-contract=off and without -ffast-math so
 * that no product is fused into a sum.  Division is IEEE fp64 and rounding is
 * nearbyint() under the default round-to-nearest-even mode.
 *
 * Parity pins: see the oracle tests (exact-rational brute force on tiny
 * groups, closed forms, invariants).  The functions here carry no pruning,
 * blocking or reordering beyond the definition above.
 */
#include <fenv.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CQO_MAX_E 64
#define CQO_FIRST_SCALE 0x0001u
#define CQO_LAST_SCALE 0x7BFFu

/* Exact value of a binary16 bit pattern (IEEE 754-2008 binary16 layout:
 * 1 sign bit, 5 exponent bits with bias 15, 10 fraction bits). */
double cqo_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (ex == 0)
        v = ldexp((double)man, -24);          /* subnormal: man * 2^-24 */
    else if (ex == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(man | 0x400), ex - 25);  /* (1024+man) * 2^(ex-25) */
    return sign ? -v : v;
}

/* Nearest binary16 to a finite x >= 0, ties to the even bit pattern; values at
 * or beyond 65520 give the infinity pattern 0x7C00.  Plain search over the
 * ordered positive patterns: find b with half(b) <= x < half(b+1), then
 * compare the two (exact, Sterbenz) distances. */
uint16_t cqo_double_to_half_rne(double x)
{
    if (!(x > 0.0))
        return 0;
    if (x >= 65520.0)
        return 0x7C00;
    uint32_t lo = 0, hi = 0x7BFF;   /* invariant: half(lo) <= x */
    if (x >= cqo_half_to_double(0x7BFF))
        lo = 0x7BFF;
    else {
        while (hi - lo > 1) {       /* half(lo) <= x < half(hi) */
            uint32_t mid = (lo + hi) / 2;
            if (cqo_half_to_double((uint16_t)mid) <= x)
                lo = mid;
            else
                hi = mid;
        }
    }
    if (lo == 0x7BFF) {             /* between 65504 and 65520: to 65504 */
        return 0x7BFF;
    }
    double a = x - cqo_half_to_double((uint16_t)lo);
    double b = cqo_half_to_double((uint16_t)(lo + 1)) - x;
    if (a < b)
        return (uint16_t)lo;
    if (b < a)
        return (uint16_t)(lo + 1);
    return (lo & 1) ? (uint16_t)(lo + 1) : (uint16_t)lo;
}

/* Codes of one group at scale s: q_i = clip(nearbyint(w_i / s), qmin, qmax). */
static void codes_at(const double *w, int n, double s, int qmin, int qmax, int *q)
{
    for (int i = 0; i < n; i++) {
        double r = nearbyint(w[i] / s);
        if (r < (double)qmin)
            r = (double)qmin;
        if (r > (double)qmax)
            r = (double)qmax;
        q[i] = (int)r;
    }
}

/* Per-environment objective sum_i d_{e,i} (w_i - s q_i)^2 in the fixed order
 * i = 0..n-1.  The environments are independent sums; looping over them in
 * the inner loop does not change any single sum's order. */
static void env_objectives(const double *w, const float *const *d, int E, int n,
                           double s, const int *q, double *obj)
{
    for (int e = 0; e < E; e++)
        obj[e] = 0.0;
    for (int i = 0; i < n; i++) {
        double r = w[i] - s * (double)q[i];
        double rr = r * r;
        for (int e = 0; e < E; e++)
            obj[e] = obj[e] + (double)d[e][i] * rr;
    }
}

static double max_env(const double *obj, int E)
{
    double f = obj[0];
    for (int e = 1; e < E; e++)
        if (obj[e] > f)
            f = obj[e];
    return f;
}

/* Objective at one scale bit pattern.  d[e] points at environment e's n
 * diagonal values for this group.  Writes codes (nullable) and per-env sums
 * (nullable); returns max_e. */
double cqo_objective(const uint16_t *w_bits, const float *const *d, int E, int n,
                     uint16_t scale_bits, int qmin, int qmax, int8_t *codes,
                     double *per_env)
{
    double w[4096];
    int q[4096];
    double obj[CQO_MAX_E];
    if (n > 4096 || E > CQO_MAX_E || E < 1)
        return NAN;
    for (int i = 0; i < n; i++)
        w[i] = cqo_half_to_double(w_bits[i]);
    double s = cqo_half_to_double(scale_bits);
    codes_at(w, n, s, qmin, qmax, q);
    env_objectives(w, d, E, n, s, q, obj);
    if (codes)
        for (int i = 0; i < n; i++)
            codes[i] = (int8_t)q[i];
    if (per_env)
        for (int e = 0; e < E; e++)
            per_env[e] = obj[e];
    return max_env(obj, E);
}

/* Exhaustive solve of one group over all 31,743 scales, ascending bit
 * patterns.  Keeps the best (f, b) with strict "<", so the lowest pattern wins
 * an exact tie, and the runner-up: the smallest f among all other patterns
 * (equal to the best when the best is tied). */
int cqo_solve_group(const uint16_t *w_bits, const float *const *d, int E, int n,
                    int qmin, int qmax, uint16_t *best_bits, double *best_obj,
                    uint16_t *runner_bits, double *runner_obj, int8_t *codes)
{
    double w[4096];
    int q[4096];
    double obj[CQO_MAX_E];
    if (n < 0 || n > 4096 || E < 1 || E > CQO_MAX_E)
        return 1;
    if (fegetround() != FE_TONEAREST)
        return 2;
    for (int i = 0; i < n; i++)
        w[i] = cqo_half_to_double(w_bits[i]);

    double best = INFINITY, runner = INFINITY;
    uint32_t bb = 0, rb = 0;
    for (uint32_t b = CQO_FIRST_SCALE; b <= CQO_LAST_SCALE; b++) {
        double s = cqo_half_to_double((uint16_t)b);
        codes_at(w, n, s, qmin, qmax, q);
        env_objectives(w, d, E, n, s, q, obj);
        double f = max_env(obj, E);
        if (f < best) {
            runner = best;
            rb = bb;
            best = f;
            bb = b;
        } else if (f < runner) {
            runner = f;
            rb = b;
        }
    }
    if (best_bits)
        *best_bits = (uint16_t)bb;
    if (best_obj)
        *best_obj = best;
    if (runner_bits)
        *runner_bits = (uint16_t)rb;
    if (runner_obj)
        *runner_obj = runner;
    if (codes) {
        codes_at(w, n, cqo_half_to_double((uint16_t)bb), qmin, qmax, q);
        for (int i = 0; i < n; i++)
            codes[i] = (int8_t)q[i];
    }
    return 0;
}

/* Pack 8 codes per uint32, low nibble first, each stored as (q + 8). */
void cqo_pack_codes(const int8_t *q, int n, uint32_t *words)
{
    for (int j = 0; j < n / 8; j++) {
        uint32_t word = 0;
        for (int t = 0; t < 8; t++)
            word |= (uint32_t)((q[8 * j + t] + 8) & 0xF) << (4 * t);
        words[j] = word;
    }
}

/* AbsMax scale: binary16 nearest (ties even) to max_i |w_i| / qmax in fp64. */
uint16_t cqo_absmax_scale(const uint16_t *w_bits, int n, int qmax)
{
    double m = 0.0;
    for (int i = 0; i < n; i++) {
        double a = fabs(cqo_half_to_double(w_bits[i]));
        if (a > m)
            m = a;
    }
    return cqo_double_to_half_rne(m / (double)qmax);
}

/* ---- batch driver: threads over groups ---------------------------------- */

typedef struct {
    const uint16_t *W;   /* [G][n] */
    const float *D;      /* K>0: [E][K] per column; K==0: [E][G][n] */
    const int64_t *sel;  /* nullable: which groups to solve */
    int64_t count, G, K;
    int n, E, qmin, qmax;
    uint16_t *best_bits;
    double *best_obj;
    uint16_t *runner_bits;
    double *runner_obj;
    int8_t *codes;       /* nullable [count][n] */
    int64_t next;
    pthread_mutex_t lock;
    int status;
} batch_job;

static void group_diag_ptrs(const batch_job *jb, int64_t g, const float **dp)
{
    for (int e = 0; e < jb->E; e++) {
        if (jb->K > 0) {
            int64_t gpr = jb->K / jb->n;
            dp[e] = jb->D + (int64_t)e * jb->K + (g % gpr) * jb->n;
        } else {
            dp[e] = jb->D + ((int64_t)e * jb->G + g) * jb->n;
        }
    }
}

static void *batch_worker(void *arg)
{
    batch_job *jb = (batch_job *)arg;
    const float *dp[CQO_MAX_E];
    for (;;) {
        pthread_mutex_lock(&jb->lock);
        int64_t k = jb->next++;
        pthread_mutex_unlock(&jb->lock);
        if (k >= jb->count)
            break;
        int64_t g = jb->sel ? jb->sel[k] : k;
        group_diag_ptrs(jb, g, dp);
        int st = cqo_solve_group(jb->W + g * jb->n, dp, jb->E, jb->n, jb->qmin, jb->qmax,
                                 jb->best_bits ? jb->best_bits + k : NULL,
                                 jb->best_obj ? jb->best_obj + k : NULL,
                                 jb->runner_bits ? jb->runner_bits + k : NULL,
                                 jb->runner_obj ? jb->runner_obj + k : NULL,
                                 jb->codes ? jb->codes + k * jb->n : NULL);
        if (st)
            jb->status = st;
    }
    return NULL;
}

/* Solve `count` groups (all G when sel is NULL, count must then equal G).
 * Results are written at position k of each output for the k-th solved group.
 * Returns 0, or nonzero on bad arguments. */
int cqo_solve_batch(const uint16_t *W, int64_t G, int n, const float *D, int E, int64_t K,
                    const int64_t *sel, int64_t count, int qmin, int qmax,
                    uint16_t *best_bits, double *best_obj, uint16_t *runner_bits,
                    double *runner_obj, int8_t *codes, int nthreads)
{
    if (n < 1 || n > 4096 || E < 1 || E > CQO_MAX_E || G < 0 || count < 0)
        return 1;
    if (K > 0 && (K % n != 0))
        return 1;
    if (!sel && count != G)
        return 1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 512)
        nthreads = 512;
    batch_job jb;
    memset(&jb, 0, sizeof(jb));
    jb.W = W;
    jb.D = D;
    jb.sel = sel;
    jb.count = count;
    jb.G = G;
    jb.K = K;
    jb.n = n;
    jb.E = E;
    jb.qmin = qmin;
    jb.qmax = qmax;
    jb.best_bits = best_bits;
    jb.best_obj = best_obj;
    jb.runner_bits = runner_bits;
    jb.runner_obj = runner_obj;
    jb.codes = codes;
    pthread_mutex_init(&jb.lock, NULL);
    pthread_t th[512];
    int started = 0;
    for (int t = 0; t < nthreads; t++) {
        if (pthread_create(&th[t], NULL, batch_worker, &jb) != 0)
            break;
        started++;
    }
    if (started == 0)
        batch_worker(&jb);
    for (int t = 0; t < started; t++)
        pthread_join(th[t], NULL);
    pthread_mutex_destroy(&jb.lock);
    return jb.status;
}
