/*
 * gdn_oracle.c -- fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm may load this library.  It shares no code,
 * header or constant with the CUDA path.
 *
 * What it computes: the plain token-by-token recurrence, no chunking.
 *
 *   Delta rule as one step of online gradient descent on
 *   f_t(S) = 1/2 ||S k_t - v_t||^2  ("OSDN: Improving Delta Rule with Provable
 *   Online Preconditioning in Linear Attention", sec. 1 Problem Statement):
 *       S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T
 *   Scalar forget gate ("Moonshot AI's New Attention Architecture: Key
 *   Innovations Explained", sec. 2 Core Operator, Gated DeltaNet form):
 *       S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t v_t k_t^T
 *   Per-dimension gate (same page, sec. 2, the architecture's own operator):
 *       S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t v_t k_t^T
 *   Output o_t = S_t q_t (the post-update state).
 *
 * Storage: M = S^T, row-major [Dk][Dv] per (batch, head).  In M form one token
 * is (a = exp(g_t), decay before the erase):
 *     1. M <- Diag(a) M            (scalar gate: every row times the same a)
 *     2. x = M^T k_t               (what the decayed memory recalls for k_t)
 *     3. r = beta_t (v_t - x)      (the gradient-step residual)
 *     4. M <- M + k_t r^T          (erase-then-write in one rank-1 update)
 *     5. o_t = M^T q_t
 * Steps 2-4 are exactly (I - beta k k^T) M + beta k v^T.
 *
 * Layouts (all dense, row-major):
 *   q, k [B][T][H][Dk]; v [B][T][H][Dv]; beta [B][T][H];
 *   g    [B][T][H] (gate_kind 1) or [B][T][H][Dk] (gate_kind 2), g = log a;
 *   S0   [B][H][Dk][Dv] or NULL (zero); o [B][T][H][Dv]; S_out [B][H][Dk][Dv].
 * Summation order is fixed (ascending index); build without -ffast-math.
 *
 * gdn_oracle_recurrent_wk is the same recurrence with a separate write key
 * kw_t (the preconditioned key of "OSDN ...", sec. 2.1: right-preconditioning
 * the gradient step by D_t = diag(d_t) is the update
 *     S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) (d_t (.) k_t)^T,
 * so the residual is read with k_t and written along kw_t = d_t (.) k_t).  In
 * M form step 4 becomes M <- M + kw_t r^T; every other step is unchanged.
 * With kw = k it is gdn_oracle_recurrent exactly (same operations, same order).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GATE_NONE 0
#define ORACLE_GATE_SCALAR 1
#define ORACLE_GATE_PER_DIM 2

static int recurrent_impl(const double* q, const double* k, const double* kw,
                          const double* v, const double* beta, const double* g,
                          int gate_kind, const double* S0, double* o, double* S_out,
                          long B, long T, long H, long Dk, long Dv, int nthreads)
{
    if (!q || !k || !kw || !v || !beta || !o || !S_out) return 1;
    if (gate_kind != ORACLE_GATE_NONE && !g) return 1;
    if (gate_kind < 0 || gate_kind > 2) return 1;
    if (B < 0 || T < 0 || H < 0 || Dk < 1 || Dv < 1) return 1;
    if (nthreads < 1) nthreads = 1;
    int failed = 0;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (long bh = 0; bh < B * H; ++bh) {
        const long b = bh / H, h = bh % H;
        double* M = S_out + bh * Dk * Dv;
        double* x = (double*)malloc(sizeof(double) * (size_t)Dv);
        double* r = (double*)malloc(sizeof(double) * (size_t)Dv);
        if (!x || !r) {
            free(x); free(r);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (S0) memcpy(M, S0 + bh * Dk * Dv, sizeof(double) * (size_t)(Dk * Dv));
        else memset(M, 0, sizeof(double) * (size_t)(Dk * Dv));

        for (long t = 0; t < T; ++t) {
            const long tok = (b * T + t) * H + h;
            const double* qt = q + tok * Dk;
            const double* kt = k + tok * Dk;
            const double* kwt = kw + tok * Dk;
            const double* vt = v + tok * Dv;
            const double bt = beta[tok];

            /* 1. decay */
            if (gate_kind == ORACLE_GATE_SCALAR) {
                const double a = exp(g[tok]);
                for (long i = 0; i < Dk * Dv; ++i) M[i] *= a;
            } else if (gate_kind == ORACLE_GATE_PER_DIM) {
                for (long i = 0; i < Dk; ++i) {
                    const double a = exp(g[tok * Dk + i]);
                    for (long j = 0; j < Dv; ++j) M[i * Dv + j] *= a;
                }
            }
            /* 2. x = M^T k */
            for (long j = 0; j < Dv; ++j) x[j] = 0.0;
            for (long i = 0; i < Dk; ++i) {
                const double ki = kt[i];
                for (long j = 0; j < Dv; ++j) x[j] += M[i * Dv + j] * ki;
            }
            /* 3. r = beta (v - x) */
            for (long j = 0; j < Dv; ++j) r[j] = bt * (vt[j] - x[j]);
            /* 4. M += kw r^T (the write key; kw = k for the plain rule) */
            for (long i = 0; i < Dk; ++i) {
                const double ki = kwt[i];
                for (long j = 0; j < Dv; ++j) M[i * Dv + j] += ki * r[j];
            }
            /* 5. o = M^T q */
            double* ot = o + tok * Dv;
            for (long j = 0; j < Dv; ++j) ot[j] = 0.0;
            for (long i = 0; i < Dk; ++i) {
                const double qi = qt[i];
                for (long j = 0; j < Dv; ++j) ot[j] += M[i * Dv + j] * qi;
            }
        }
        free(x);
        free(r);
    }
    return failed ? 2 : 0;
}

int gdn_oracle_recurrent(const double* q, const double* k, const double* v,
                         const double* beta, const double* g, int gate_kind,
                         const double* S0, double* o, double* S_out,
                         long B, long T, long H, long Dk, long Dv, int nthreads)
{
    return recurrent_impl(q, k, k, v, beta, g, gate_kind, S0, o, S_out, B, T, H, Dk, Dv,
                          nthreads);
}

int gdn_oracle_recurrent_wk(const double* q, const double* k, const double* kw,
                            const double* v, const double* beta, const double* g,
                            int gate_kind, const double* S0, double* o, double* S_out,
                            long B, long T, long H, long Dk, long Dv, int nthreads)
{
    return recurrent_impl(q, k, kw, v, beta, g, gate_kind, S0, o, S_out, B, T, H, Dk, Dv,
                          nthreads);
}
