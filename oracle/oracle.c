/*
 * fp64 CPU oracle for ReplaySSM decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm use it.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * What it computes (plain, slow, obviously correct; double precision; libm
 * exp; no fast-math, no fused contractions -- built with -ffp-contract=off):
 *
 *  - The eager recurrences that ReplaySSM must reproduce.  The pages state
 *    that they do not give the SSM equations ("ReplaySSM for hybrid
 *    SSM-Transformer stacks", section "What is not documented"); the standard
 *    published forms of the two layer kinds the abstract names are used:
 *      Mamba-2 (Transformers are SSMs / structured state space duality):
 *          h_t = exp(dt_t * A) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D x_t
 *          with h in R^{P x N}, x in R^P, B, C in R^N, scalar dt, A, D per head.
 *      Gated DeltaNet (Gated Delta Networks: Improving Mamba2 with Delta Rule):
 *          S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *          o_t = scale * S_t q_t
 *          with S in R^{dv x dk}, q, k in R^dk, v in R^dv, scalar alpha, beta.
 *  - The replay (unrolled) form of the same outputs: a checkpoint S0 plus the
 *    buffered inputs since it ("ReplaySSM: Cache SSM Inputs, Not State",
 *    Abstract: the state is represented as a checkpoint and a buffer of recent
 *    SSM inputs; "ReplaySSM for hybrid SSM-Transformer stacks", How ReplaySSM
 *    works, step 2).  Used only to pin the algebra against the eager form.
 *  - bf16 round-to-nearest-even and OCP FP8 E4M3 (satfinite, RNE) encoders,
 *    written from the format definitions; used by the tests that check that
 *    the low-precision output copy is exactly the quantisation of the master
 *    ("How ReplaySSM works", step 5: the high-precision checkpoint is never
 *    derived from the low-precision one).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Mamba-2                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Eager Mamba-2 recurrence for one (sequence, head), T steps.
 *   h  [P][N]  state, updated in place (row p = head channel, column n = state dim)
 *   x  [T][P], dt [T], Bm [T][N], Cm [T][N]
 *   y  [T][P]  output (may be NULL: a pure fold, as a commit does)
 */
void oracle_mamba2_eager(int P, int N, int T, double A, double D,
                         const double *x, const double *dt,
                         const double *Bm, const double *Cm,
                         double *h, double *y)
{
    for (int t = 0; t < T; ++t) {
        const double decay = exp(dt[t] * A);
        const double *xt = x + (size_t)t * P;
        const double *bt = Bm + (size_t)t * N;
        const double *ct = Cm + (size_t)t * N;
        for (int p = 0; p < P; ++p) {
            double *hp = h + (size_t)p * N;
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                /* h_t[p][n] = exp(dt A) h_{t-1}[p][n] + dt * x[p] * B[n] */
                hp[n] = decay * hp[n] + dt[t] * xt[p] * bt[n];
                acc += hp[n] * ct[n];
            }
            if (y) y[(size_t)t * P + p] = acc + D * xt[p];
        }
    }
}

/*
 * Replay form: output of the newest buffered entry from a checkpoint S0 and
 * the L buffered entries since it (entry L-1 is the current token).
 *   y = exp(A sum_{j} dt_j) (S0 C_L)
 *       + sum_i exp(A sum_{j>i} dt_j) dt_i (B_i . C_L) x_i + D x_L
 * S0 is not modified and no intermediate state is formed.
 */
void oracle_mamba2_replay(int P, int N, int L, double A, double D,
                          const double *S0, const double *x, const double *dt,
                          const double *Bm, const double *Cm, double *y)
{
    const double *c = Cm + (size_t)(L - 1) * N;
    double total = 0.0;
    for (int j = 0; j < L; ++j) total += dt[j];
    const double decay_all = exp(A * total);
    for (int p = 0; p < P; ++p) {
        double s0c = 0.0;
        for (int n = 0; n < N; ++n) s0c += S0[(size_t)p * N + n] * c[n];
        double acc = decay_all * s0c;
        for (int i = 0; i < L; ++i) {
            double after = 0.0;                 /* sum of dt over entries newer than i */
            for (int j = i + 1; j < L; ++j) after += dt[j];
            double bc = 0.0;
            for (int n = 0; n < N; ++n) bc += Bm[(size_t)i * N + n] * c[n];
            acc += exp(A * after) * dt[i] * bc * x[(size_t)i * P + p];
        }
        y[p] = acc + D * x[(size_t)(L - 1) * P + p];
    }
}

/* ------------------------------------------------------------------------ */
/* Gated DeltaNet                                                            */
/* ------------------------------------------------------------------------ */

/*
 * Eager Gated DeltaNet recurrence for one (sequence, head), T steps.
 *   S [DV][DK] state, updated in place (row r indexes v, column c indexes k)
 *   q, k [T][DK], v [T][DV], alpha, beta [T]
 *   o [T][DV] (may be NULL)
 * Row r of S (I - beta k k^T) is s_r - beta (s_r . k) k^T, so the update of
 * row r is  s_r <- alpha (s_r - beta (s_r . k) k) + beta v[r] k.
 */
void oracle_gdn_eager(int DV, int DK, int T, double scale,
                      const double *q, const double *k, const double *v,
                      const double *alpha, const double *beta,
                      double *S, double *o)
{
    for (int t = 0; t < T; ++t) {
        const double *qt = q + (size_t)t * DK;
        const double *kt = k + (size_t)t * DK;
        const double *vt = v + (size_t)t * DV;
        for (int r = 0; r < DV; ++r) {
            double *sr = S + (size_t)r * DK;
            double sk = 0.0;
            for (int c = 0; c < DK; ++c) sk += sr[c] * kt[c];
            double acc = 0.0;
            for (int c = 0; c < DK; ++c) {
                sr[c] = alpha[t] * (sr[c] - beta[t] * sk * kt[c]) + beta[t] * vt[r] * kt[c];
                acc += sr[c] * qt[c];
            }
            if (o) o[(size_t)t * DV + r] = scale * acc;
        }
    }
}

/*
 * Replay form for Gated DeltaNet.  With M_j = alpha_j (I - beta_j k_j k_j^T)
 * the state after the buffer is S0 M_1..M_L + sum_i beta_i v_i k_i^T M_{i+1}..M_L,
 * so  o = S0 (M_1..M_L q) + sum_i c_i v_i  with  c_i = beta_i k_i^T (M_{i+1}..M_L q).
 * The transformed query is formed by one backward sweep over the buffer:
 *   u <- q;  for j = L..1:  c_j = beta_j (k_j . u);  u <- alpha_j (u - beta_j (k_j . u) k_j)
 * q is the current (newest) entry's query.
 */
void oracle_gdn_replay(int DV, int DK, int L, double scale, const double *S0,
                       const double *k, const double *v,
                       const double *alpha, const double *beta,
                       const double *q, double *o)
{
    double *u = (double *)malloc(sizeof(double) * (size_t)DK);
    double *coef = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int c = 0; c < DK; ++c) u[c] = q[c];
    for (int j = L - 1; j >= 0; --j) {
        const double *kj = k + (size_t)j * DK;
        double ku = 0.0;
        for (int c = 0; c < DK; ++c) ku += kj[c] * u[c];
        coef[j] = beta[j] * ku;
        for (int c = 0; c < DK; ++c) u[c] = alpha[j] * (u[c] - beta[j] * ku * kj[c]);
    }
    for (int r = 0; r < DV; ++r) {
        double acc = 0.0;
        for (int c = 0; c < DK; ++c) acc += S0[(size_t)r * DK + c] * u[c];
        for (int j = 0; j < L; ++j) acc += coef[j] * v[(size_t)j * DV + r];
        o[r] = scale * acc;
    }
    free(coef);
    free(u);
}

/* ------------------------------------------------------------------------ */
/* Batched drivers: independent (sequence, head) pairs split over threads.   */
/* Pair-major layouts: x [npairs][T][P], dt [npairs][T], ...                 */
/* Threading only partitions independent pairs; per-pair arithmetic is the   */
/* single-pair function above, unchanged.                                    */
/* ------------------------------------------------------------------------ */

typedef struct {
    int kind;           /* 0 = Mamba-2, 1 = GDN */
    int first, last;    /* pair range [first, last) */
    int R, Cc, T;       /* rows, columns, steps */
    const double *p0, *p1;                  /* Mamba-2: A, D per pair; GDN: scale (p0[0]) */
    const double *a0, *a1, *a2, *a3, *a4;   /* per-step inputs */
    double *state, *out;
} oracle_job;

static void *oracle_worker(void *arg)
{
    const oracle_job *j = (const oracle_job *)arg;
    const size_t RC = (size_t)j->R * j->Cc;
    const size_t T = (size_t)j->T;
    for (int i = j->first; i < j->last; ++i) {
        double *out = j->out ? j->out + (size_t)i * T * j->R : NULL;
        if (j->kind == 0) {
            oracle_mamba2_eager(j->R, j->Cc, j->T, j->p0[i], j->p1[i],
                                j->a0 + (size_t)i * T * j->R,  /* x  */
                                j->a1 + (size_t)i * T,         /* dt */
                                j->a2 + (size_t)i * T * j->Cc, /* B  */
                                j->a3 + (size_t)i * T * j->Cc, /* C  */
                                j->state + (size_t)i * RC, out);
        } else {
            oracle_gdn_eager(j->R, j->Cc, j->T, j->p0[0],
                             j->a0 + (size_t)i * T * j->Cc,    /* q */
                             j->a1 + (size_t)i * T * j->Cc,    /* k */
                             j->a2 + (size_t)i * T * j->R,     /* v */
                             j->a3 + (size_t)i * T,            /* alpha */
                             j->a4 + (size_t)i * T,            /* beta  */
                             j->state + (size_t)i * RC, out);
        }
    }
    return NULL;
}

static int oracle_run_jobs(oracle_job base, int npairs, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > npairs) nthreads = npairs > 0 ? npairs : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    oracle_job *jobs = (oracle_job *)malloc(sizeof(oracle_job) * (size_t)nthreads);
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = base;
        jobs[t].first = (int)(((long long)npairs * t) / nthreads);
        jobs[t].last = (int)(((long long)npairs * (t + 1)) / nthreads);
        if (pthread_create(&th[t], NULL, oracle_worker, &jobs[t]) != 0) {
            oracle_worker(&jobs[t]);   /* run inline if a thread cannot start */
            th[t] = 0;
            rc = 1;
        } else {
            ++started;
        }
    }
    for (int t = 0; t < nthreads; ++t)
        if (th[t]) pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    (void)started;
    return rc;
}

int oracle_mamba2_eager_batch(int npairs, int P, int N, int T,
                              const double *A, const double *D,
                              const double *x, const double *dt,
                              const double *Bm, const double *Cm,
                              double *h, double *y, int nthreads)
{
    oracle_job j;
    memset(&j, 0, sizeof j);
    j.kind = 0; j.R = P; j.Cc = N; j.T = T;
    j.p0 = A; j.p1 = D; j.a0 = x; j.a1 = dt; j.a2 = Bm; j.a3 = Cm;
    j.state = h; j.out = y;
    return oracle_run_jobs(j, npairs, nthreads);
}

int oracle_gdn_eager_batch(int npairs, int DV, int DK, int T, double scale,
                           const double *q, const double *k, const double *v,
                           const double *alpha, const double *beta,
                           double *S, double *o, int nthreads)
{
    oracle_job j;
    memset(&j, 0, sizeof j);
    j.kind = 1; j.R = DV; j.Cc = DK; j.T = T;
    j.p0 = &scale;
    j.a0 = q; j.a1 = k; j.a2 = v; j.a3 = alpha; j.a4 = beta;
    j.state = S; j.out = o;
    return oracle_run_jobs(j, npairs, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 = the upper 16 bits of an IEEE binary32, rounded to nearest, ties to
 * even.  NaN maps to a quiet NaN of the same sign. */
uint16_t oracle_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7fc0u);
    uint32_t lower = u & 0xffffu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

void oracle_bf16_rne_array(const float *in, uint16_t *out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = oracle_bf16_rne(in[i]);
}

/*
 * OCP 8-bit floating point, E4M3 ("fn": no infinities).  Bias 7, 3 mantissa
 * bits, largest finite 448 = 1.75 * 2^8, smallest normal 2^-6, subnormal step
 * 2^-9, 0x7f / 0xff are NaN.  Rounding is to nearest with ties to even; the
 * satfinite mode clamps every finite magnitude above 448 (and infinities) to
 * 448.  The rounding is done exactly in double: |f| / quantum is a float times
 * a power of two, nearbyint() rounds it half-to-even.
 */
uint8_t oracle_e4m3_rne_satfinite(float f)
{
    if (isnan(f)) return (uint8_t)(signbit(f) ? 0xff : 0x7f);
    const uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a == 0.0) return sign;
    if (isinf(a) || a >= 448.0) return (uint8_t)(sign | 0x7e);
    int e;
    (void)frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1): floor(log2 a) = e - 1 */
    int ex = e - 1;
    if (ex < -6) ex = -6;          /* subnormal range shares the 2^-6 binade's quantum */
    const double quantum = ldexp(1.0, ex - 3);
    double qa = nearbyint(a / quantum) * quantum;
    if (qa >= 448.0) return (uint8_t)(sign | 0x7e);
    if (qa == 0.0) return sign;
    if (qa < ldexp(1.0, -6)) {     /* subnormal: value = m * 2^-9, m in 1..7 */
        int m = (int)(qa / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    int e2;
    (void)frexp(qa, &e2);
    int ef = e2 - 1;               /* qa in [2^ef, 2^(ef+1)) */
    int m = (int)(qa / ldexp(1.0, ef - 3)) - 8;
    return (uint8_t)(sign | ((ef + 7) << 3) | m);
}

float oracle_e4m3_decode(uint8_t b)
{
    const int s = b >> 7, ef = (b >> 3) & 0xf, m = b & 7;
    if (ef == 0xf && m == 7) return NAN;
    double v = ef == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, ef - 7 - 3);
    return (float)(s ? -v : v);
}

void oracle_e4m3_rne_satfinite_array(const float *in, uint8_t *out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = oracle_e4m3_rne_satfinite(in[i]);
}

void oracle_e4m3_decode_array(const uint8_t *in, float *out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(in[i]);
}
