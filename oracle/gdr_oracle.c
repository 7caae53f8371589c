/*
 * gdr_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta-rule forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, link or
 * call this file.  It is used by tests/, by __graft_entry__.smoke() and by the
 * CPU-baseline / reference legs of bench.py, and nowhere else.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section/equation):
 *  [SLA]  "Systolic Linear Attention: Co-Designing Tile-Grouped Gated Delta
 *         Attention for TPUs".
 *  [MOMI] "When Good Enough Is Optimal: Multiplication-Only Matrix Inversion
 *         Approximation for Quantized Gated DeltaNet".
 *
 * Layouts (all row-major, contiguous, fp64):
 *   q, k   [B, Hk, T, dk]      query / key of key head hk
 *   v      [B, Hv, T, dv]      value of value head hv; hv uses key head hv / R,
 *                              R = Hv / Hk (grouped value heads, [SLA] §2.3,
 *                              §2.4.1)
 *   g      [B, Hk, T, G]       log forget gate (<= 0); channel i of a key head
 *                              uses group floor(i * G / dk)  ([SLA] §2.1 GDN
 *                              G=1, KDA G=dk; §2.3 four 64-channel tiles)
 *   beta   [B, Hk, T]          write gate, shared by the R value heads
 *   S0     [B, Hv, dk, dv]     initial state, or NULL for zeros
 *   o      [B, Hv, T, dv]      output o_t = S_t^T q_t (post-update state)
 *   S_final[B, Hv, dk, dv]     state after the last token
 *
 * Routines: gdro_recurrent (the definition: token recurrence), gdro_chunked
 * (the chunkwise WY form with the exact, truncated-Neumann or 1-Step Neumann
 * inverse), gdro_chunked_momentum (the same with chunk-boundary momentum,
 * [SLA] §2.3), gdro_recurrent_grad (the exact gradient of the token recurrence,
 * a reverse sweep: what a backward, [SLA] §2.5, must reproduce), the chunk
 * inverses alone (gdro_tril_inverse, gdro_neumann_inverse,
 * gdro_block_neumann1_inverse), the chunk's factor matrices
 * (gdro_chunk_matrices) and the readout epilogue (gdro_output_gate_rmsnorm,
 * [SLA] §2.3 Eq. (5)).
 *
 * Every function returns 0 on success and a negative code on a bad argument.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GDRO_ERR_ARG (-1)
#define GDRO_ERR_NOMEM (-2)

/* Inverse modes and Neumann variant bits (mirrors nothing; the CUDA library
 * defines its own enums). */
#define GDRO_INV_EXACT 0
#define GDRO_INV_NEUMANN 1
#define GDRO_INV_NEUMANN1 2  /* [SLA] 1-Step Neumann, blocks of GDRO_BLK1 rows */
#define GDRO_BLK1 16
#define GDRO_NV_REFINE 1   /* residual step uses X0 instead of X_k        */
#define GDRO_NV_BANDCUT 2  /* zero X0 outside the band i - j <= order      */

static int check_dims(int B, int T, int Hk, int Hv, int dk, int dv, int G)
{
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || G <= 0)
        return GDRO_ERR_ARG;
    if (Hv % Hk != 0 || dk % G != 0)
        return GDRO_ERR_ARG;
    return 0;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int gdro_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Token-by-token recurrence, the definition of the operation.
 * [SLA] §2.1, Eq. (2), prediction-error form:
 *     S_t = F_t S_{t-1} + beta_t k_t (v_t - (F_t S_{t-1})^T k_t)^T,
 *     o_t = S_t^T q_t,   F_t = diag(exp(g_t expanded to dk channels)).
 * Each step: decay the rows of S, read the current prediction r = S^T k,
 * write beta * k (v - r)^T, read out with q.
 */
int gdro_recurrent(int B, int T, int Hk, int Hv, int dk, int dv, int G,
                   const double *q, const double *k, const double *v,
                   const double *g, const double *beta, const double *S0,
                   double *o, double *S_final, int nthreads)
{
    if (check_dims(B, T, Hk, Hv, dk, dv, G))
        return GDRO_ERR_ARG;
    const int R = Hv / Hk;
    const long nseq = (long)B * Hv;
    int err = 0;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (long s = 0; s < nseq; ++s) {
        const long b = s / Hv, hv = s % Hv, hk = hv / R;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *f = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !r || !f) {
            free(S); free(r); free(f);
#pragma omp atomic write
            err = GDRO_ERR_NOMEM;
            continue;
        }
        if (S0)
            memcpy(S, S0 + s * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        const long kh = b * Hk + hk;
        for (long t = 0; t < T; ++t) {
            const double *qt = q + (kh * T + t) * dk;
            const double *kt = k + (kh * T + t) * dk;
            const double *vt = v + (s * T + t) * dv;
            const double *gt = g + (kh * T + t) * G;
            const double bt = beta[kh * T + t];
            for (int i = 0; i < dk; ++i)
                f[i] = exp(gt[(long)i * G / dk]);
            /* decay: S <- F_t S */
            for (int i = 0; i < dk; ++i)
                for (int n = 0; n < dv; ++n)
                    S[i * dv + n] *= f[i];
            /* current prediction r = S^T k */
            for (int n = 0; n < dv; ++n)
                r[n] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int n = 0; n < dv; ++n)
                    r[n] += S[i * dv + n] * kt[i];
            /* delta write */
            for (int i = 0; i < dk; ++i) {
                const double bk = bt * kt[i];
                for (int n = 0; n < dv; ++n)
                    S[i * dv + n] += bk * (vt[n] - r[n]);
            }
            /* readout with the post-update state */
            double *ot = o + (s * T + t) * dv;
            for (int n = 0; n < dv; ++n)
                ot[n] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int n = 0; n < dv; ++n)
                    ot[n] += S[i * dv + n] * qt[i];
        }
        if (S_final)
            memcpy(S_final + s * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(r); free(f);
    }
    return err;
}

/*
 * X = (I + N)^{-1} for strictly lower-triangular N (n x n, row-major), by
 * forward substitution (row t of X from rows j < t).  This is the
 * "sequential substitution" that [SLA] §2.2 Bottleneck 3 describes; it is a
 * different algorithm from the block-doubling the GPU uses.
 */
int gdro_tril_inverse(int n, const double *N, double *X)
{
    if (n < 0)
        return GDRO_ERR_ARG;
    for (int t = 0; t < n; ++t) {
        for (int c = 0; c < n; ++c) {
            double acc = (t == c) ? 1.0 : 0.0;
            for (int j = c; j < t; ++j)
                acc -= N[t * n + j] * X[j * n + c];
            X[t * n + c] = (c <= t) ? acc : 0.0;
        }
    }
    return 0;
}

static void matmul_nn(int n, const double *A, const double *B, double *C)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int l = 0; l < n; ++l)
                acc += A[i * n + l] * B[l * n + j];
            C[i * n + j] = acc;
        }
}

/*
 * Truncated Neumann approximation of (I + N)^{-1}, N strictly lower
 * triangular, following [MOMI] (abstract; Lemma 3.1; §4.1 settings):
 *   1. powers with structural masking: P_1 = N, P_p = mask_p(P_{p-1} N),
 *      mask_p zeroing entries with i - j < p (Lemma 3.1: those entries of
 *      N^p vanish, so the mask keeps only the structurally non-zero band);
 *   2. X_0 = sum_{p=0}^{order} (-1)^p P_p;
 *   3. residual correction, `resid` times:
 *        Newton (default):  X_{s+1} = X_s + X_s (I - (I + N) X_s)
 *        refine (flag 1) :  X_{s+1} = X_s + X_0 (I - (I + N) X_s)
 *      (identical for one step).
 * Flag 2 zeroes X_0 outside the band i - j <= order before the correction.
 */
int gdro_neumann_inverse(int n, const double *N, int order, int resid, int variant,
                         double *X)
{
    if (n < 0 || order < 0 || resid < 0)
        return GDRO_ERR_ARG;
    const size_t nn = (size_t)n * n;
    double *P = (double *)malloc(sizeof(double) * (nn ? nn : 1));
    double *T1 = (double *)malloc(sizeof(double) * (nn ? nn : 1));
    double *X0 = (double *)malloc(sizeof(double) * (nn ? nn : 1));
    double *Rm = (double *)malloc(sizeof(double) * (nn ? nn : 1));
    if (!P || !T1 || !X0 || !Rm) {
        free(P); free(T1); free(X0); free(Rm);
        return GDRO_ERR_NOMEM;
    }
    /* X0 = I (p = 0) */
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            X0[i * n + j] = (i == j) ? 1.0 : 0.0;
    if (order >= 1) {
        memcpy(P, N, sizeof(double) * nn);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j)
                if (i - j < 1)
                    P[i * n + j] = 0.0;
        for (size_t e = 0; e < nn; ++e)
            X0[e] -= P[e];
    }
    for (int p = 2; p <= order; ++p) {
        matmul_nn(n, P, N, T1);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j)
                if (i - j < p)
                    T1[i * n + j] = 0.0;
        memcpy(P, T1, sizeof(double) * nn);
        const double sgn = (p % 2 == 0) ? 1.0 : -1.0;
        for (size_t e = 0; e < nn; ++e)
            X0[e] += sgn * P[e];
    }
    if (variant & GDRO_NV_BANDCUT)
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j)
                if (i - j > order)
                    X0[i * n + j] = 0.0;
    memcpy(X, X0, sizeof(double) * nn);
    for (int s = 0; s < resid; ++s) {
        /* Rm = I - (I + N) X = -(N X) + (I - X) */
        matmul_nn(n, N, X, T1);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j)
                Rm[i * n + j] = ((i == j) ? 1.0 : 0.0) - X[i * n + j] - T1[i * n + j];
        matmul_nn(n, (variant & GDRO_NV_REFINE) ? X0 : X, Rm, T1);
        for (size_t e = 0; e < nn; ++e)
            X[e] += T1[e];
    }
    free(P); free(T1); free(X0); free(Rm);
    return 0;
}

/*
 * 1-Step Neumann of [SLA] §2.4.3 ("Block-doubling and block-Neumann
 * factorization").  Write I + N = D (I + Nb): D is the block-diagonal part of
 * I + N in blocks of `blk` rows (the last block may be shorter) and
 * Nb = D^{-1} N_off, N_off the part of N below the diagonal blocks.  Nb is
 * nilpotent, so (I + N)^{-1} = sum_s (-Nb)^s D^{-1}; the 1-Step variant keeps the
 * terms s = 0 and 1:
 *   X = (I - Nb) D^{-1}.
 * D^{-1} block by block by forward substitution (gdro_tril_inverse).
 */
int gdro_block_neumann1_inverse(int n, const double *N, int blk, double *X)
{
    if (n < 0 || blk < 1)
        return GDRO_ERR_ARG;
    const size_t nn = (size_t)n * n;
    double *Dinv = (double *)calloc(nn ? nn : 1, sizeof(double));
    double *Noff = (double *)calloc(nn ? nn : 1, sizeof(double));
    double *Nb = (double *)malloc(sizeof(double) * (nn ? nn : 1));
    double *Bi = (double *)malloc(sizeof(double) * (size_t)blk * blk);
    double *Bx = (double *)malloc(sizeof(double) * (size_t)blk * blk);
    if (!Dinv || !Noff || !Nb || !Bi || !Bx) {
        free(Dinv); free(Noff); free(Nb); free(Bi); free(Bx);
        return GDRO_ERR_NOMEM;
    }
    for (int b0 = 0; b0 < n; b0 += blk) {
        const int nb = (n - b0 < blk) ? n - b0 : blk;
        for (int i = 0; i < nb; ++i)
            for (int j = 0; j < nb; ++j)
                Bi[i * nb + j] = N[(b0 + i) * n + b0 + j];
        gdro_tril_inverse(nb, Bi, Bx);
        for (int i = 0; i < nb; ++i)
            for (int j = 0; j < nb; ++j)
                Dinv[(b0 + i) * n + b0 + j] = Bx[i * nb + j];
    }
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            if (j / blk < i / blk)
                Noff[i * n + j] = N[i * n + j];
    matmul_nn(n, Dinv, Noff, Nb);
    matmul_nn(n, Nb, Dinv, X);            /* Nb D^{-1} */
    for (size_t e = 0; e < nn; ++e)
        X[e] = Dinv[e] - X[e];            /* (I - Nb) D^{-1} */
    free(Dinv); free(Noff); free(Nb); free(Bi); free(Bx);
    return 0;
}

/*
 * Chunk matrices of one chunk for one key head, [SLA] §2.2 Bottleneck 2 and
 * §2.3 Table 2 (Gram M, score L, cumulative log-decay Lambda):
 *   Lam[t][i] = sum_{s<=t} g_s(i)                       (summed, never log o exp)
 *   M[t][j]   = 1[t>j]  beta_j sum_i k_ti k_ji exp(Lam_ti - Lam_ji)
 *   L[t][j]   = 1[t>=j]        sum_i q_ti k_ji exp(Lam_ti - Lam_ji)
 * The exponent is always of a difference with t >= j, so it is <= 0 and
 * needs no pivot in fp64.  Arrays: qc,kc [Cl][dk], gc [Cl][G], bc [Cl].
 */
static void chunk_matrices(int Cl, int dk, int G, const double *qc, const double *kc,
                           const double *gc, const double *bc, double *Lam,
                           double *M, double *L)
{
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int t = 0; t < Cl; ++t) {
            acc += gc[(long)t * G + (long)i * G / dk];
            Lam[t * dk + i] = acc;
        }
    }
    for (int t = 0; t < Cl; ++t)
        for (int j = 0; j < Cl; ++j) {
            double m = 0.0, l = 0.0;
            if (j <= t) {
                for (int i = 0; i < dk; ++i) {
                    const double d = exp(Lam[t * dk + i] - Lam[j * dk + i]);
                    m += kc[t * dk + i] * kc[j * dk + i] * d;
                    l += qc[t * dk + i] * kc[j * dk + i] * d;
                }
            }
            M[t * Cl + j] = (j < t) ? bc[j] * m : 0.0;
            L[t * Cl + j] = (j <= t) ? l : 0.0;
        }
}

int gdro_chunk_matrices(int Cl, int dk, int G, const double *qc, const double *kc,
                        const double *gc, const double *bc, double *Lam, double *M,
                        double *L)
{
    if (Cl < 0 || dk <= 0 || G <= 0 || dk % G != 0)
        return GDRO_ERR_ARG;
    chunk_matrices(Cl, dk, G, qc, kc, gc, bc, Lam, M, L);
    return 0;
}

/*
 * Chunkwise WY form ([SLA] §2.1 "Chunkwise WY parallelization", §2.3 Table 2,
 * §2.4.2 "Proof of tile-grouped packed WY equivalence", §2.5):
 *   A  = (I + M)^{-1}                     (exact: forward substitution;
 *                                          NEUMANN: gdro_neumann_inverse)
 *   Kb = P_{t<-0} k_t,  Qb = P_{t<-0} q_t,  Kh = P_{C<-t} k_t,  F = P_{C<-0}
 *   E  = diag(beta) A (V - Kb S)          (= U - W S with U, W of Table 2)
 *   O  = Qb S + L E
 *   S <- F S + Kh^T E
 * A ragged last chunk (T % C != 0) is a chunk of length T - start.
 * Processed per value head (one S of dk x dv), so the packed grouped-value
 * form is reached by running the R value heads of a key head separately.
 */
static int chunked_impl(int B, int T, int Hk, int Hv, int dk, int dv, int G, int C,
                        int inverse_mode, int neumann_order, int neumann_resid,
                        int neumann_variant, int momentum, double mu, const int *kappa,
                        const double *q, const double *k, const double *v, const double *g,
                        const double *beta, const double *S0, double *o, double *S_final,
                        int nthreads)
{
    if (check_dims(B, T, Hk, Hv, dk, dv, G) || C <= 0)
        return GDRO_ERR_ARG;
    if (inverse_mode != GDRO_INV_EXACT && inverse_mode != GDRO_INV_NEUMANN &&
        inverse_mode != GDRO_INV_NEUMANN1)
        return GDRO_ERR_ARG;
    if (inverse_mode == GDRO_INV_NEUMANN && (neumann_order < 0 || neumann_resid < 0))
        return GDRO_ERR_ARG;
    const int R = Hv / Hk;
    const long nseq = (long)B * Hv;
    int err = 0;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (long s = 0; s < nseq; ++s) {
        const long b = s / Hv, hv = s % Hv, hk = hv / R;
        const long kh = b * Hk + hk;
        const size_t CC = (size_t)C * C;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *Lam = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *M = (double *)malloc(sizeof(double) * CC);
        double *L = (double *)malloc(sizeof(double) * CC);
        double *A = (double *)malloc(sizeof(double) * CC);
        double *RHS = (double *)malloc(sizeof(double) * (size_t)C * dv);
        double *E = (double *)malloc(sizeof(double) * (size_t)C * dv);
        double *Kb = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *Qb = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *Kh = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *F = (double *)malloc(sizeof(double) * (size_t)dk);
        /* momentum: the chunk-entry state and the velocity buffer Z (zero at the start) */
        double *Sp = momentum ? (double *)malloc(sizeof(double) * (size_t)dk * dv) : NULL;
        double *Z = momentum ? (double *)calloc((size_t)dk * dv, sizeof(double)) : NULL;
        if (!S || !Lam || !M || !L || !A || !RHS || !E || !Kb || !Qb || !Kh || !F ||
            (momentum && (!Sp || !Z))) {
            free(S); free(Lam); free(M); free(L); free(A); free(RHS); free(E);
            free(Kb); free(Qb); free(Kh); free(F); free(Sp); free(Z);
#pragma omp atomic write
            err = GDRO_ERR_NOMEM;
            continue;
        }
        if (S0)
            memcpy(S, S0 + s * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (long c0 = 0; c0 < T; c0 += C) {
            const int Cl = (int)((T - c0 < C) ? (T - c0) : C);
            const double *qc = q + (kh * T + c0) * dk;
            const double *kc = k + (kh * T + c0) * dk;
            const double *vc = v + (s * T + c0) * dv;
            const double *gc = g + (kh * T + c0) * G;
            const double *bc = beta + kh * T + c0;
            chunk_matrices(Cl, dk, G, qc, kc, gc, bc, Lam, M, L);
            if (inverse_mode == GDRO_INV_EXACT)
                gdro_tril_inverse(Cl, M, A);
            else if (inverse_mode == GDRO_INV_NEUMANN1) {
                if (gdro_block_neumann1_inverse(Cl, M, GDRO_BLK1, A) != 0) {
#pragma omp atomic write
                    err = GDRO_ERR_NOMEM;
                    break;
                }
            } else if (gdro_neumann_inverse(Cl, M, neumann_order, neumann_resid,
                                          neumann_variant, A) != 0) {
#pragma omp atomic write
                err = GDRO_ERR_NOMEM;
                break;
            }
            /* decayed operands: Kb_t = P_{t<-0} k_t, Qb_t = P_{t<-0} q_t,
             * Kh_t = P_{C<-t} k_t, F = P_{C<-0} (Table 2 of [SLA] §2.3) */
            for (int i = 0; i < dk; ++i) {
                const double LamC = Lam[(Cl - 1) * dk + i];
                F[i] = exp(LamC);
                for (int t = 0; t < Cl; ++t) {
                    Kb[t * dk + i] = kc[t * dk + i] * exp(Lam[t * dk + i]);
                    Qb[t * dk + i] = qc[t * dk + i] * exp(Lam[t * dk + i]);
                    Kh[t * dk + i] = kc[t * dk + i] * exp(LamC - Lam[t * dk + i]);
                }
            }
            /* RHS = V - Kb S */
            for (int t = 0; t < Cl; ++t)
                for (int n = 0; n < dv; ++n) {
                    double acc = vc[t * dv + n];
                    for (int i = 0; i < dk; ++i)
                        acc -= Kb[t * dk + i] * S[i * dv + n];
                    RHS[t * dv + n] = acc;
                }
            /* E = diag(beta) A RHS */
            for (int t = 0; t < Cl; ++t)
                for (int n = 0; n < dv; ++n) {
                    double acc = 0.0;
                    for (int j = 0; j < Cl; ++j)
                        acc += A[t * Cl + j] * RHS[j * dv + n];
                    E[t * dv + n] = bc[t] * acc;
                }
            /* O = Qb S + L E (uses the chunk-entry state) */
            for (int t = 0; t < Cl; ++t) {
                double *ot = o + (s * T + c0 + t) * dv;
                for (int n = 0; n < dv; ++n) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i)
                        acc += Qb[t * dk + i] * S[i * dv + n];
                    for (int j = 0; j <= t; ++j)
                        acc += L[t * Cl + j] * E[j * dv + n];
                    ot[n] = acc;
                }
            }
            if (momentum)
                memcpy(Sp, S, sizeof(double) * (size_t)dk * dv);
            /* S <- F S + Kh^T E */
            for (int i = 0; i < dk; ++i)
                for (int n = 0; n < dv; ++n) {
                    double acc = F[i] * S[i * dv + n];
                    for (int t = 0; t < Cl; ++t)
                        acc += Kh[t * dk + i] * E[t * dv + n];
                    S[i * dv + n] = acc;
                }
            if (momentum) {
                /* chunk-boundary momentum ([SLA] §2.3): with S the chunk update just
                 * formed (S~_c) and Sp the chunk-entry state S_{c-1},
                 *   Z_c = mu kappa_c Z_{c-1} + (S~_c - F_c S_{c-1}),  S_c = F_c S_{c-1} + Z_c */
                const long nch = (T + C - 1) / C;
                const double mk = mu * (kappa ? (double)kappa[b * nch + c0 / C] : 1.0);
                for (int i = 0; i < dk; ++i)
                    for (int n = 0; n < dv; ++n) {
                        const double fs = F[i] * Sp[i * dv + n];
                        Z[i * dv + n] = mk * Z[i * dv + n] + (S[i * dv + n] - fs);
                        S[i * dv + n] = fs + Z[i * dv + n];
                    }
            }
        }
        if (S_final)
            memcpy(S_final + s * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(Lam); free(M); free(L); free(A); free(RHS); free(E);
        free(Kb); free(Qb); free(Kh); free(F); free(Sp); free(Z);
    }
    return err;
}

int gdro_chunked(int B, int T, int Hk, int Hv, int dk, int dv, int G, int C,
                 int inverse_mode, int neumann_order, int neumann_resid,
                 int neumann_variant, const double *q, const double *k,
                 const double *v, const double *g, const double *beta,
                 const double *S0, double *o, double *S_final, int nthreads)
{
    return chunked_impl(B, T, Hk, Hv, dk, dv, G, C, inverse_mode, neumann_order, neumann_resid,
                        neumann_variant, 0, 0.0, NULL, q, k, v, g, beta, S0, o, S_final,
                        nthreads);
}

/*
 * The chunked form with chunk-boundary momentum ([SLA] §2.3, the momentum
 * equation after Eq. (5), and §2.3's notation table): every chunk's state update
 * S~_c (the chunked form above, from S_{c-1}) is blended with a velocity buffer,
 *   Z_c = mu kappa_c Z_{c-1} + (S~_c - F_c S_{c-1}),  S_c = F_c S_{c-1} + Z_c,
 * Z_0 = 0.  kappa: [B][ceil(T / C)] reset indicators (0 where a document reset
 * falls inside the chunk), or NULL for ones.  The outputs of chunk c come from
 * the chunk computation started at S_{c-1}, as without momentum.
 */
int gdro_chunked_momentum(int B, int T, int Hk, int Hv, int dk, int dv, int G, int C,
                          int inverse_mode, int neumann_order, int neumann_resid,
                          int neumann_variant, double mu, const int *kappa, const double *q,
                          const double *k, const double *v, const double *g,
                          const double *beta, const double *S0, double *o, double *S_final,
                          int nthreads)
{
    return chunked_impl(B, T, Hk, Hv, dk, dv, G, C, inverse_mode, neumann_order, neumann_resid,
                        neumann_variant, 1, mu, kappa, q, k, v, g, beta, S0, o, S_final,
                        nthreads);
}

/*
 * Output gate and per-value-head RMSNorm of the readout, [SLA] §2.3 Eq. (5):
 *   out_t = sigmoid(z_t) * RMSNorm(o_t),  RMSNorm(x) = x / sqrt(mean_i x_i^2 + eps) * w
 * over the dv channels of one (token, value head) row.  o, z, out: [rows][dv];
 * w: [dv] per-channel weight, or NULL for ones.  out may alias o.
 */
int gdro_output_gate_rmsnorm(int rows, int dv, const double *o, const double *z, const double *w,
                             double eps, double *out)
{
    if (rows < 0 || dv < 1 || eps < 0.0)
        return GDRO_ERR_ARG;
    for (int r = 0; r < rows; ++r) {
        const double *x = o + (size_t)r * dv;
        double ss = 0.0;
        for (int i = 0; i < dv; ++i)
            ss += x[i] * x[i];
        const double inv = 1.0 / sqrt(ss / dv + eps);
        for (int i = 0; i < dv; ++i) {
            const double gate = 1.0 / (1.0 + exp(-z[(size_t)r * dv + i]));
            out[(size_t)r * dv + i] = gate * x[i] * inv * (w ? w[i] : 1.0);
        }
    }
    return 0;
}

/* f_i = exp(g of channel i's group) for one token's gate row gt[G] */
static void decay_factors(double *f, const double *gt, int dk, int G)
{
    for (int i = 0; i < dk; ++i) {
        const long grp = (long)i * G / dk;
        f[i] = exp(gt[grp]);
    }
}

/*
 * Gradients of the token recurrence ([SLA] §2.1 Eq. (2), the definition the
 * oracle's forward follows) by a reverse sweep over the tokens: for upstream
 * gradients dO [B,Hv,T,dv] and dSf [B,Hv,dk,dv] (NULL for zero), the gradients
 * of sum(dO * o) + sum(dSf * S_final) with respect to q, k [B,Hk,T,dk],
 * v [B,Hv,T,dv], g [B,Hk,T,G], beta [B,Hk,T] and S0 [B,Hv,dk,dv] (the initial
 * state, zero when S0 is NULL).  Per token, with S' = F_t S_{t-1}, u = v - S'^T k,
 * S_t = S' + beta k u^T and o = S_t^T q, backwards:
 *   dS += q do^T, dq = S_t do;
 *   du = beta dS^T k, dbeta = k^T dS u, dk = beta dS u - S' du, dv = du,
 *   dS' = dS - k du^T;
 *   dS_{t-1} = F_t dS', dg (per group) += sum_{i in group} f_i sum_n dS'_in S_{t-1,in}.
 * Key-head inputs collect the gradients of all their value heads.  The states
 * are recomputed forward and kept per token (T dk dv doubles per value head).
 */
int gdro_recurrent_grad(int B, int T, int Hk, int Hv, int dk, int dv, int G, const double *q,
                        const double *k, const double *v, const double *g, const double *beta,
                        const double *S0, const double *dO, const double *dSf, double *dq,
                        double *dkk, double *dvv, double *dg, double *dbeta, double *dS0,
                        int nthreads)
{
    if (check_dims(B, T, Hk, Hv, dk, dv, G) || !dO)
        return GDRO_ERR_ARG;
    const int R = Hv / Hk;
    const long nkh = (long)B * Hk;
    const size_t SS = (size_t)dk * dv;
    int err = 0;
    memset(dq, 0, sizeof(double) * (size_t)nkh * T * dk);
    memset(dkk, 0, sizeof(double) * (size_t)nkh * T * dk);
    memset(dg, 0, sizeof(double) * (size_t)nkh * T * G);
    memset(dbeta, 0, sizeof(double) * (size_t)nkh * T);
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (long kh = 0; kh < nkh; ++kh) {   /* one key head and its R value heads */
        const long b = kh / Hk, hk = kh % Hk;
        double *Sall = (double *)malloc(sizeof(double) * SS * (size_t)(T + 1));
        double *Sp = (double *)malloc(sizeof(double) * SS);
        double *dS = (double *)malloc(sizeof(double) * SS);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *du = (double *)malloc(sizeof(double) * (size_t)dv);
        double *f = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!Sall || !Sp || !dS || !u || !du || !f) {
            free(Sall); free(Sp); free(dS); free(u); free(du); free(f);
#pragma omp atomic write
            err = GDRO_ERR_NOMEM;
            continue;
        }
        for (int m = 0; m < R; ++m) {
            const long s = b * Hv + hk * R + m;   /* value-head sequence */
            /* forward, keeping S_{t-1} of every token in Sall[t] */
            if (S0)
                memcpy(Sall, S0 + s * (long)SS, sizeof(double) * SS);
            else
                memset(Sall, 0, sizeof(double) * SS);
            for (long t = 0; t < T; ++t) {
                const double *kt = k + (kh * T + t) * dk, *vt = v + (s * T + t) * dv;
                const double *gt = g + (kh * T + t) * G;
                const double bt = beta[kh * T + t];
                const double *Sprev = Sall + SS * t;
                double *Snew = Sall + SS * (t + 1);
                decay_factors(f, gt, dk, G);
                for (int n = 0; n < dv; ++n) {
                    double r = 0.0;
                    for (int i = 0; i < dk; ++i)
                        r += f[i] * Sprev[i * dv + n] * kt[i];
                    u[n] = vt[n] - r;
                }
                for (int i = 0; i < dk; ++i)
                    for (int n = 0; n < dv; ++n)
                        Snew[i * dv + n] = f[i] * Sprev[i * dv + n] + bt * kt[i] * u[n];
            }
            /* reverse sweep */
            if (dSf)
                memcpy(dS, dSf + s * (long)SS, sizeof(double) * SS);
            else
                memset(dS, 0, sizeof(double) * SS);
            for (long t = T - 1; t >= 0; --t) {
                const double *qt = q + (kh * T + t) * dk, *kt = k + (kh * T + t) * dk;
                const double *vt = v + (s * T + t) * dv, *gt = g + (kh * T + t) * G;
                const double *dot = dO + (s * T + t) * dv;
                const double bt = beta[kh * T + t];
                const double *Sprev = Sall + SS * t, *Snew = Sall + SS * (t + 1);
                double *dqt = dq + (kh * T + t) * dk, *dkt = dkk + (kh * T + t) * dk;
                double *dvt = dvv + (s * T + t) * dv, *dgt = dg + (kh * T + t) * G;
                decay_factors(f, gt, dk, G);
                for (int i = 0; i < dk; ++i)
                    for (int n = 0; n < dv; ++n)
                        Sp[i * dv + n] = f[i] * Sprev[i * dv + n];
                for (int n = 0; n < dv; ++n) {
                    double r = 0.0;
                    for (int i = 0; i < dk; ++i)
                        r += Sp[i * dv + n] * kt[i];
                    u[n] = vt[n] - r;
                }
                /* readout o = S_t^T q */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int n = 0; n < dv; ++n) {
                        dS[i * dv + n] += qt[i] * dot[n];
                        acc += Snew[i * dv + n] * dot[n];
                    }
                    dqt[i] += acc;
                }
                /* write S_t = S' + beta k u^T, u = v - S'^T k */
                double db = 0.0;
                for (int n = 0; n < dv; ++n) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i)
                        acc += kt[i] * dS[i * dv + n];
                    du[n] = bt * acc;
                    db += acc * u[n];
                    dvt[n] = du[n];
                }
                dbeta[kh * T + t] += db;
                for (int i = 0; i < dk; ++i) {
                    double a1 = 0.0, a2 = 0.0;
                    for (int n = 0; n < dv; ++n) {
                        a1 += dS[i * dv + n] * u[n];
                        a2 += Sp[i * dv + n] * du[n];
                    }
                    dkt[i] += bt * a1 - a2;
                }
                /* dS' = dS - k du^T, then through the decay S' = F_t S_{t-1} */
                for (int i = 0; i < dk; ++i) {
                    double df = 0.0;
                    for (int n = 0; n < dv; ++n) {
                        const double dsp = dS[i * dv + n] - kt[i] * du[n];
                        df += dsp * Sprev[i * dv + n];
                        dS[i * dv + n] = f[i] * dsp;
                    }
                    dgt[(long)i * G / dk] += df * f[i];
                }
            }
            memcpy(dS0 + s * (long)SS, dS, sizeof(double) * SS);
        }
        free(Sall); free(Sp); free(dS); free(u); free(du); free(f);
    }
    return err;
}
