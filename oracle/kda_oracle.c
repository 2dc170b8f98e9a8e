/*
 * kda_oracle.c -- plain, slow, sequential fp64 reference of the KDA recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the checker for the CUDA library; it
 * is never part of the product path. Only tests, the smoke check and the CPU
 * baseline leg of the benchmark may load it. It shares no code, header or
 * table with the CUDA path.
 *
 * What it computes (Kimi Delta Attention, KDA):
 *   Per (batch b, head h) there is a d_k x d_v state S. For each token t:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t
 *   with alpha_t = exp(log_alpha_t) in (0,1]^{d_k} a per-channel forget gate.
 *
 * Where the pages state it (Kimi Linear summary, es.news.hada.io/topic?id=31936):
 *   - section "De la atencion lineal a Gated DeltaNet": a matrix-valued state
 *     used as fast weights (linear attention); the delta rule corrects the
 *     stored association with a rank-1 update that is a generalised
 *     Householder transform (DeltaNet); GDN adds a scalar forget gate alpha_t.
 *   - section "Control fino de memoria en Kimi Delta Attention": KDA replaces
 *     the scalar gate by a diagonal, per-channel gate Diag(alpha_t) and keeps
 *     the delta rule, giving a Diagonal-Plus-Low-Rank transition.
 *   - section "Algoritmo paralelo por chunks": the chunked algorithm reaches
 *     the same state and outputs as this token-by-token recurrence; the
 *     oracle therefore is the recurrence itself, not the chunked algorithm.
 *
 * The update is evaluated in the plain order the formula gives:
 *     S' = Diag(alpha_t) S            (decay every row i of S by alpha_t[i])
 *     r  = S'^T k_t                   (what the state recalls for k_t)
 *     u  = beta_w v_t - beta_e r      (erase-then-write, rank-1)
 *     S  = S' + k_t u^T
 *     o  = S^T q_t                    (read from the post-update state)
 * Expanding: S' + k (beta v - beta k^T S')^T = (I - beta k k^T) S' + beta k v^T.
 * For KDA beta_e = beta_w = beta. Separate erase and write strengths exist
 * only so that tests can reach the special cases the pages name (gated
 * linear attention and plain linear attention have no erase term).
 *
 * Inputs q, k, v are fp32 or bf16 (raw 16-bit patterns, widened exactly);
 * gates and the state are read as given; everything is computed in fp64.
 * Layouts (contiguous, token-major, heads interleaved):
 *   q, k, log_alpha [B,T,H,dk]; v, out [B,T,H,dv]; beta [B,T,H];
 *   S0, ST [B,H,dk,dv].
 *
 * Parity status: pinned. The tests check this recurrence against linear
 * attention, gated linear attention, scalar-gate GDN, DeltaNet with basis
 * keys, the beta = 0 closed form, brute-force products of dense transition
 * matrices, a hand-worked example, and invariants (splitting, permutations,
 * the Householder norm bound).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Widen element i of an input array of type in_dtype (0 = fp32, 1 = bf16). */
static double widen(const void *p, long i, int in_dtype)
{
    if (in_dtype == 0)
        return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * One (b, h) pair, all T tokens.
 * Returns 0, or -1 if scratch memory could not be allocated.
 */
static int run_head(const void *q, const void *k, const void *v, int in_dtype,
                    const float *log_alpha, const float *beta_e, const float *beta_w,
                    const double *S0, double *out, double *ST,
                    long b, long h, long T, long H, long dk, long dv)
{
    double *S = (double *)calloc((size_t)(dk * dv), sizeof(double));
    double *kt = (double *)malloc(sizeof(double) * (size_t)dk);
    double *qt = (double *)malloc(sizeof(double) * (size_t)dk);
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !kt || !qt || !r || !u) {
        free(S); free(kt); free(qt); free(r); free(u);
        return -1;
    }
    if (S0) {
        const double *s0 = S0 + (b * H + h) * dk * dv;
        for (long e = 0; e < dk * dv; ++e)
            S[e] = s0[e];
    }
    for (long t = 0; t < T; ++t) {
        long row = (b * T + t) * H + h;          /* index of (b, t, h) */
        double be = (double)beta_e[row];
        double bw = beta_w ? (double)beta_w[row] : be;
        for (long i = 0; i < dk; ++i) {
            kt[i] = widen(k, row * dk + i, in_dtype);
            qt[i] = widen(q, row * dk + i, in_dtype);
        }
        /* S' = Diag(alpha_t) S */
        for (long i = 0; i < dk; ++i) {
            double a = exp((double)log_alpha[row * dk + i]);
            for (long j = 0; j < dv; ++j)
                S[i * dv + j] *= a;
        }
        /* r = S'^T k_t */
        for (long j = 0; j < dv; ++j)
            r[j] = 0.0;
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                r[j] += S[i * dv + j] * kt[i];
        /* u = beta_w v_t - beta_e r ; S = S' + k_t u^T */
        for (long j = 0; j < dv; ++j)
            u[j] = bw * widen(v, row * dv + j, in_dtype) - be * r[j];
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j)
                S[i * dv + j] += kt[i] * u[j];
        /* o_t = S_t^T q_t */
        for (long j = 0; j < dv; ++j) {
            double o = 0.0;
            for (long i = 0; i < dk; ++i)
                o += S[i * dv + j] * qt[i];
            out[row * dv + j] = o;
        }
    }
    if (ST) {
        double *st = ST + (b * H + h) * dk * dv;
        for (long e = 0; e < dk * dv; ++e)
            st[e] = S[e];
    }
    free(S); free(kt); free(qt); free(r); free(u);
    return 0;
}

/*
 * Full forward over the heads listed in `heads` (flat indices b*H + h), or
 * over all B*H heads when heads == NULL. Rows of `out` and blocks of `ST`
 * that belong to heads not listed are left untouched. beta_w may be NULL
 * (then beta_w = beta_e, which is KDA). S0 may be NULL (zero state); ST may
 * be NULL (not written). nthreads <= 0 uses the OpenMP default.
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int kda_oracle_fwd(const void *q, const void *k, const void *v, int in_dtype,
                   const float *log_alpha, const float *beta_e, const float *beta_w,
                   const double *S0, double *out, double *ST,
                   long B, long T, long H, long dk, long dv,
                   const int64_t *heads, long nheads, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta_e || !out)
        return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0 || (in_dtype != 0 && in_dtype != 1))
        return -1;
    long n = heads ? nheads : B * H;
    for (long i = 0; heads && i < n; ++i)
        if (heads[i] < 0 || heads[i] >= B * H)
            return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (long i = 0; i < n; ++i) {
        long bh = heads ? (long)heads[i] : i;
        failed |= run_head(q, k, v, in_dtype, log_alpha, beta_e, beta_w, S0, out, ST,
                           bh / H, bh % H, T, H, dk, dv) != 0;
    }
    (void)nthreads;
    return failed ? -1 : 0;
}

/* Number of threads an OpenMP parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
