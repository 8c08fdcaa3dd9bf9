/*
 * la_oracle.c — fp64 CPU oracle for kernelized linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (all in double precision, one attention head at a time,
 * tensors laid out [B, H, N, D] with D innermost):
 *
 *   a_i = phi(q_i),  b_j = phi(k_j)                       (elementwise phi)
 *   S_i = sum_{j in J(i)} b_j v_j^T      (D x D)
 *   z_i = sum_{j in J(i)} b_j            (D)
 *   o_i = S_i^T a_i / (a_i . z_i)
 *
 * with J(i) = {all j} (non-causal) or {j <= i} (causal).  This is the
 * kernel-decomposition form of attention stated in "Efficient Transformers
 * Survey", section Linear Attention, Proposition "Linear Attention via
 * Kernel Decomposition" (Statement), evaluated with the token-by-token
 * update of S and z described in the same proposition's "Why It Matters"
 * paragraph (recurrent computation, constant memory per step).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - phi is elementwise with m = D; id 0 is elu(x)+1 (alpha = 1), id 1 is
 *     max(x,0) + 1e-6.  The pages leave phi generic.  Id 2 is the identity:
 *     the inputs are feature vectors already (positive random features of
 *     the Performer, computed by the caller; phi' = 1).
 *   - causal sums include the diagonal (j <= i).
 *   - no epsilon is added to the denominator; both maps are > 0.
 *   - phi'(0) is taken from the x <= 0 branch (exp(0) = 1 for elu+1, 0 for
 *     the ReLU map).
 *
 * Functions:
 *   oracle_forward    the recurrence above (the plain definition).
 *   oracle_quadratic  the same attention evaluated the quadratic way,
 *                     W = (A B^T) masked, O = diag(W 1)^-1 W V; this is the
 *                     form the Proof Sketch starts from, kept separate so the
 *                     two can be checked against each other.
 *   oracle_backward   dQ, dK, dV of L = sum(dO * O) by the closed-form
 *                     gradient of the definition (derived by hand; the pages
 *                     print no gradient).  Pinned by finite differences.
 *   oracle_decode_step one in-place recurrent step on a caller's (S, z).
 *
 * Decayed (gated) variants, causal only: every step first scales the state
 * by a per-head factor gamma in [0, 1], S_i = gamma S_{i-1} + b_i v_i^T and
 * z_i = gamma z_{i-1} + b_i, and the query reads it as above.  The pages
 * name gating and decay factors as the change linear-attention models need
 * to match softmax quality ("Efficient Transformers Survey", Common
 * Confusions, "Watch Out: Linear attention is not a drop-in replacement")
 * without fixing a form; this is the plainest one (a constant per head,
 * applied to both sums so that o_i stays a weighted average of the v_j with
 * weights gamma^(i-j) a_i.b_j).
 *   oracle_forward_decay      the decayed recurrence.
 *   oracle_quadratic_decay    w_ij = gamma^(i-j) a_i . b_j for j <= i.
 *   oracle_backward_decay     its closed-form gradient (decayed prefix and
 *                             suffix states), pinned by finite differences.
 *   oracle_decode_step_decay  one decayed step on a caller's (S, z).
 *
 * Heads are independent; an OpenMP loop runs over them.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PHI_ELU1 0
#define ORACLE_PHI_RELU_EPS 1
#define ORACLE_PHI_IDENTITY 2

static double phi_of(double x, int phi)
{
    if (phi == ORACLE_PHI_ELU1)
        return x > 0.0 ? x + 1.0 : exp(x);
    if (phi == ORACLE_PHI_IDENTITY)
        return x;
    return (x > 0.0 ? x : 0.0) + 1e-6;
}

static double dphi_of(double x, int phi)
{
    if (phi == ORACLE_PHI_ELU1)
        return x > 0.0 ? 1.0 : exp(x);
    if (phi == ORACLE_PHI_IDENTITY)
        return 1.0;
    return x > 0.0 ? 1.0 : 0.0;
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Forward.  q, k, v, o: [B,H,N,D].  S_out: [B,H,D,D] (row = feature f,
 * column = value index), z_out: [B,H,D]; either may be NULL.  They receive
 * the state after all N tokens.
 */
void oracle_forward(const double *q, const double *k, const double *v,
                    double *o, double *S_out, double *z_out,
                    int64_t B, int64_t H, int64_t N, int64_t D,
                    int causal, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        double *oh = o + h * N * D;
        double *S = calloc((size_t)(D * D), sizeof(double));
        double *z = calloc((size_t)D, sizeof(double));
        double *a = malloc((size_t)D * sizeof(double));
        double *b = malloc((size_t)D * sizeof(double));

        if (!causal) {
            /* S = sum_j b_j v_j^T, z = sum_j b_j over every key first. */
            for (int64_t j = 0; j < N; ++j) {
                for (int64_t f = 0; f < D; ++f)
                    b[f] = phi_of(kh[j * D + f], phi);
                for (int64_t f = 0; f < D; ++f) {
                    z[f] += b[f];
                    for (int64_t e = 0; e < D; ++e)
                        S[f * D + e] += b[f] * vh[j * D + e];
                }
            }
        }
        for (int64_t i = 0; i < N; ++i) {
            if (causal) {
                /* add token i to the running state, then query it */
                for (int64_t f = 0; f < D; ++f)
                    b[f] = phi_of(kh[i * D + f], phi);
                for (int64_t f = 0; f < D; ++f) {
                    z[f] += b[f];
                    for (int64_t e = 0; e < D; ++e)
                        S[f * D + e] += b[f] * vh[i * D + e];
                }
            }
            double den = 0.0;
            for (int64_t f = 0; f < D; ++f) {
                a[f] = phi_of(qh[i * D + f], phi);
                den += a[f] * z[f];
            }
            for (int64_t e = 0; e < D; ++e) {
                double num = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    num += a[f] * S[f * D + e];
                oh[i * D + e] = num / den;
            }
        }
        if (S_out)
            memcpy(S_out + h * D * D, S, (size_t)(D * D) * sizeof(double));
        if (z_out)
            memcpy(z_out + h * D, z, (size_t)D * sizeof(double));
        free(S);
        free(z);
        free(a);
        free(b);
    }
}

/*
 * Quadratic form: w_ij = a_i . b_j for j in J(i), o_i = sum_j w_ij v_j /
 * sum_j w_ij.  O(N^2 D); meant for small N.
 */
void oracle_quadratic(const double *q, const double *k, const double *v,
                      double *o, int64_t B, int64_t H, int64_t N, int64_t D,
                      int causal, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        double *oh = o + h * N * D;
        double *A = malloc((size_t)(N * D) * sizeof(double));
        double *Bm = malloc((size_t)(N * D) * sizeof(double));
        for (int64_t t = 0; t < N * D; ++t) {
            A[t] = phi_of(qh[t], phi);
            Bm[t] = phi_of(kh[t], phi);
        }
        for (int64_t i = 0; i < N; ++i) {
            const int64_t jmax = causal ? i + 1 : N;
            double rowsum = 0.0;
            for (int64_t e = 0; e < D; ++e)
                oh[i * D + e] = 0.0;
            for (int64_t j = 0; j < jmax; ++j) {
                double w = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    w += A[i * D + f] * Bm[j * D + f];
                rowsum += w;
                for (int64_t e = 0; e < D; ++e)
                    oh[i * D + e] += w * vh[j * D + e];
            }
            for (int64_t e = 0; e < D; ++e)
                oh[i * D + e] /= rowsum;
        }
        free(A);
        free(Bm);
    }
}

/*
 * Backward of L = sum_i dO_i . o_i.  With u_i = S_i^T a_i and g_i = a_i.z_i
 * (so o_i = u_i / g_i):
 *
 *   du_i = dO_i / g_i                       dg_i = -(dO_i . o_i) / g_i
 *   dA_i = S_i du_i + z_i dg_i                                   (D)
 *   dB_j = sum_{i : j in J(i)} a_i (v_j . du_i + dg_i)            (D)
 *   dV_j = sum_{i : j in J(i)} (a_i . b_j) du_i                   (D)
 *   dQ = dA * phi'(Q),  dK = dB * phi'(K)
 *
 * dA uses the same prefix (or total) state as the forward.  dB and dV use
 * the reverse-direction sums R = sum a_i du_i^T (D x D) and r = sum a_i dg_i
 * (D) over the queries that see key j:  dB_j = R v_j + r,  dV_j = R^T b_j.
 */
void oracle_backward(const double *q, const double *k, const double *v,
                     const double *dO, double *dq, double *dk, double *dv,
                     int64_t B, int64_t H, int64_t N, int64_t D,
                     int causal, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        const double *gh = dO + h * N * D;
        double *dqh = dq + h * N * D;
        double *dkh = dk + h * N * D;
        double *dvh = dv + h * N * D;

        double *S = calloc((size_t)(D * D), sizeof(double));
        double *z = calloc((size_t)D, sizeof(double));
        double *R = calloc((size_t)(D * D), sizeof(double));
        double *r = calloc((size_t)D, sizeof(double));
        double *b = malloc((size_t)D * sizeof(double));
        /* per-token quantities reused by the reverse sweep */
        double *A = malloc((size_t)(N * D) * sizeof(double));
        double *DU = malloc((size_t)(N * D) * sizeof(double));
        double *DG = malloc((size_t)N * sizeof(double));

        if (!causal) {
            for (int64_t j = 0; j < N; ++j) {
                for (int64_t f = 0; f < D; ++f)
                    b[f] = phi_of(kh[j * D + f], phi);
                for (int64_t f = 0; f < D; ++f) {
                    z[f] += b[f];
                    for (int64_t e = 0; e < D; ++e)
                        S[f * D + e] += b[f] * vh[j * D + e];
                }
            }
        }
        /* forward sweep: g, o, du, dg and dA -> dQ */
        for (int64_t i = 0; i < N; ++i) {
            if (causal) {
                for (int64_t f = 0; f < D; ++f)
                    b[f] = phi_of(kh[i * D + f], phi);
                for (int64_t f = 0; f < D; ++f) {
                    z[f] += b[f];
                    for (int64_t e = 0; e < D; ++e)
                        S[f * D + e] += b[f] * vh[i * D + e];
                }
            }
            double *a = A + i * D;
            double g = 0.0;
            for (int64_t f = 0; f < D; ++f) {
                a[f] = phi_of(qh[i * D + f], phi);
                g += a[f] * z[f];
            }
            double dot = 0.0; /* dO_i . o_i */
            for (int64_t e = 0; e < D; ++e) {
                double u = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    u += a[f] * S[f * D + e];
                dot += gh[i * D + e] * (u / g);
                DU[i * D + e] = gh[i * D + e] / g;
            }
            DG[i] = -dot / g;
            for (int64_t f = 0; f < D; ++f) {
                double da = z[f] * DG[i];
                for (int64_t e = 0; e < D; ++e)
                    da += S[f * D + e] * DU[i * D + e];
                dqh[i * D + f] = da * dphi_of(qh[i * D + f], phi);
            }
        }
        if (!causal) {
            /* every query sees every key: R, r are totals */
            for (int64_t i = 0; i < N; ++i)
                for (int64_t f = 0; f < D; ++f) {
                    r[f] += A[i * D + f] * DG[i];
                    for (int64_t e = 0; e < D; ++e)
                        R[f * D + e] += A[i * D + f] * DU[i * D + e];
                }
        }
        /* reverse sweep: dB -> dK and dV */
        for (int64_t j = N - 1; j >= 0; --j) {
            if (causal) {
                /* queries i >= j see key j: add query j, then use */
                for (int64_t f = 0; f < D; ++f) {
                    r[f] += A[j * D + f] * DG[j];
                    for (int64_t e = 0; e < D; ++e)
                        R[f * D + e] += A[j * D + f] * DU[j * D + e];
                }
            }
            for (int64_t f = 0; f < D; ++f)
                b[f] = phi_of(kh[j * D + f], phi);
            for (int64_t f = 0; f < D; ++f) {
                double db = r[f];
                for (int64_t e = 0; e < D; ++e)
                    db += R[f * D + e] * vh[j * D + e];
                dkh[j * D + f] = db * dphi_of(kh[j * D + f], phi);
            }
            for (int64_t e = 0; e < D; ++e) {
                double acc = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    acc += R[f * D + e] * b[f];
                dvh[j * D + e] = acc;
            }
        }
        free(S);
        free(z);
        free(R);
        free(r);
        free(b);
        free(A);
        free(DU);
        free(DG);
    }
}

/*
 * One recurrent step, in place: S += b v^T, z += b, then
 * o = S^T a / (a . z) with the updated state.  S: [B,H,D,D], z: [B,H,D],
 * q, k, v, o: [B,H,D].
 */
void oracle_decode_step(double *S, double *z, const double *q,
                        const double *k, const double *v, double *o,
                        int64_t B, int64_t H, int64_t D, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < heads; ++h) {
        double *Sh = S + h * D * D;
        double *zh = z + h * D;
        const double *qh = q + h * D, *kh = k + h * D, *vh = v + h * D;
        double *oh = o + h * D;
        for (int64_t f = 0; f < D; ++f) {
            const double bf = phi_of(kh[f], phi);
            zh[f] += bf;
            for (int64_t e = 0; e < D; ++e)
                Sh[f * D + e] += bf * vh[e];
        }
        double den = 0.0;
        for (int64_t f = 0; f < D; ++f)
            den += phi_of(qh[f], phi) * zh[f];
        for (int64_t e = 0; e < D; ++e) {
            double num = 0.0;
            for (int64_t f = 0; f < D; ++f)
                num += phi_of(qh[f], phi) * Sh[f * D + e];
            oh[e] = num / den;
        }
    }
}

/*
 * Decayed causal forward: per head h (flattened b*H + h), gamma[h % H].
 * S_i = gamma S_{i-1} + b_i v_i^T, z_i = gamma z_{i-1} + b_i, o_i = S_i^T a_i
 * / (a_i . z_i).  S_out, z_out as for oracle_forward (nullable).
 */
void oracle_forward_decay(const double *q, const double *k, const double *v,
                          const double *gamma, double *o, double *S_out,
                          double *z_out, int64_t B, int64_t H, int64_t N,
                          int64_t D, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double gm = gamma[h % H];
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        double *oh = o + h * N * D;
        double *S = calloc((size_t)(D * D), sizeof(double));
        double *z = calloc((size_t)D, sizeof(double));
        double *a = malloc((size_t)D * sizeof(double));
        double *b = malloc((size_t)D * sizeof(double));
        for (int64_t i = 0; i < N; ++i) {
            for (int64_t f = 0; f < D; ++f)
                b[f] = phi_of(kh[i * D + f], phi);
            for (int64_t f = 0; f < D; ++f) {
                z[f] = gm * z[f] + b[f];
                for (int64_t e = 0; e < D; ++e)
                    S[f * D + e] = gm * S[f * D + e] + b[f] * vh[i * D + e];
            }
            double den = 0.0;
            for (int64_t f = 0; f < D; ++f) {
                a[f] = phi_of(qh[i * D + f], phi);
                den += a[f] * z[f];
            }
            for (int64_t e = 0; e < D; ++e) {
                double num = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    num += a[f] * S[f * D + e];
                oh[i * D + e] = num / den;
            }
        }
        if (S_out)
            memcpy(S_out + h * D * D, S, (size_t)(D * D) * sizeof(double));
        if (z_out)
            memcpy(z_out + h * D, z, (size_t)D * sizeof(double));
        free(S);
        free(z);
        free(a);
        free(b);
    }
}

/*
 * Decayed quadratic form: w_ij = gamma^(i-j) a_i . b_j for j <= i, o_i =
 * sum_j w_ij v_j / sum_j w_ij (pow(0, 0) = 1: with gamma = 0 only the
 * diagonal remains).  O(N^2 D); small N only.
 */
void oracle_quadratic_decay(const double *q, const double *k, const double *v,
                            const double *gamma, double *o, int64_t B,
                            int64_t H, int64_t N, int64_t D, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double gm = gamma[h % H];
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        double *oh = o + h * N * D;
        for (int64_t i = 0; i < N; ++i) {
            double rowsum = 0.0;
            for (int64_t e = 0; e < D; ++e)
                oh[i * D + e] = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                double w = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    w += phi_of(qh[i * D + f], phi) * phi_of(kh[j * D + f], phi);
                w *= pow(gm, (double)(i - j));
                rowsum += w;
                for (int64_t e = 0; e < D; ++e)
                    oh[i * D + e] += w * vh[j * D + e];
            }
            for (int64_t e = 0; e < D; ++e)
                oh[i * D + e] /= rowsum;
        }
    }
}

/*
 * Backward of L = sum_i dO_i . o_i for the decayed forward.  The forward's
 * sums carry weights gamma^(i-j), so with the decayed prefix state (S_i,
 * z_i) of the forward and the decayed suffix sums
 *   R_j = sum_{i >= j} gamma^(i-j) a_i du_i^T = gamma R_{j+1} + a_j du_j^T
 *   r_j = sum_{i >= j} gamma^(i-j) a_i dg_i   = gamma r_{j+1} + a_j dg_j
 * the gradient keeps the undecayed form:
 *   du_i = dO_i / g_i, dg_i = -(dO_i . o_i) / g_i,
 *   dA_i = S_i du_i + z_i dg_i,  dB_j = R_j v_j + r_j,  dV_j = R_j^T b_j,
 *   dQ = dA * phi'(Q), dK = dB * phi'(K).
 */
void oracle_backward_decay(const double *q, const double *k, const double *v,
                           const double *dO, const double *gamma, double *dq,
                           double *dk, double *dv, int64_t B, int64_t H,
                           int64_t N, int64_t D, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < heads; ++h) {
        const double gm = gamma[h % H];
        const double *qh = q + h * N * D;
        const double *kh = k + h * N * D;
        const double *vh = v + h * N * D;
        const double *gh = dO + h * N * D;
        double *dqh = dq + h * N * D;
        double *dkh = dk + h * N * D;
        double *dvh = dv + h * N * D;
        double *S = calloc((size_t)(D * D), sizeof(double));
        double *z = calloc((size_t)D, sizeof(double));
        double *R = calloc((size_t)(D * D), sizeof(double));
        double *r = calloc((size_t)D, sizeof(double));
        double *b = malloc((size_t)D * sizeof(double));
        double *A = malloc((size_t)(N * D) * sizeof(double));
        double *DU = malloc((size_t)(N * D) * sizeof(double));
        double *DG = malloc((size_t)N * sizeof(double));
        /* forward sweep: decayed prefix state, g, o, du, dg, dA -> dQ */
        for (int64_t i = 0; i < N; ++i) {
            for (int64_t f = 0; f < D; ++f)
                b[f] = phi_of(kh[i * D + f], phi);
            for (int64_t f = 0; f < D; ++f) {
                z[f] = gm * z[f] + b[f];
                for (int64_t e = 0; e < D; ++e)
                    S[f * D + e] = gm * S[f * D + e] + b[f] * vh[i * D + e];
            }
            double *a = A + i * D;
            double g = 0.0;
            for (int64_t f = 0; f < D; ++f) {
                a[f] = phi_of(qh[i * D + f], phi);
                g += a[f] * z[f];
            }
            double dot = 0.0;
            for (int64_t e = 0; e < D; ++e) {
                double u = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    u += a[f] * S[f * D + e];
                dot += gh[i * D + e] * (u / g);
                DU[i * D + e] = gh[i * D + e] / g;
            }
            DG[i] = -dot / g;
            for (int64_t f = 0; f < D; ++f) {
                double da = z[f] * DG[i];
                for (int64_t e = 0; e < D; ++e)
                    da += S[f * D + e] * DU[i * D + e];
                dqh[i * D + f] = da * dphi_of(qh[i * D + f], phi);
            }
        }
        /* reverse sweep: decayed suffix sums, dB -> dK and dV */
        for (int64_t j = N - 1; j >= 0; --j) {
            for (int64_t f = 0; f < D; ++f) {
                r[f] = gm * r[f] + A[j * D + f] * DG[j];
                for (int64_t e = 0; e < D; ++e)
                    R[f * D + e] = gm * R[f * D + e] + A[j * D + f] * DU[j * D + e];
            }
            for (int64_t f = 0; f < D; ++f)
                b[f] = phi_of(kh[j * D + f], phi);
            for (int64_t f = 0; f < D; ++f) {
                double db = r[f];
                for (int64_t e = 0; e < D; ++e)
                    db += R[f * D + e] * vh[j * D + e];
                dkh[j * D + f] = db * dphi_of(kh[j * D + f], phi);
            }
            for (int64_t e = 0; e < D; ++e) {
                double acc = 0.0;
                for (int64_t f = 0; f < D; ++f)
                    acc += R[f * D + e] * b[f];
                dvh[j * D + e] = acc;
            }
        }
        free(S);
        free(z);
        free(R);
        free(r);
        free(b);
        free(A);
        free(DU);
        free(DG);
    }
}

/*
 * One decayed recurrent step, in place: S = gamma S + b v^T, z = gamma z +
 * b, then o = S^T a / (a . z).  Shapes as oracle_decode_step; gamma[H].
 */
void oracle_decode_step_decay(double *S, double *z, const double *q,
                              const double *k, const double *v,
                              const double *gamma, double *o, int64_t B,
                              int64_t H, int64_t D, int phi)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < heads; ++h) {
        const double gm = gamma[h % H];
        double *Sh = S + h * D * D;
        double *zh = z + h * D;
        const double *qh = q + h * D, *kh = k + h * D, *vh = v + h * D;
        double *oh = o + h * D;
        for (int64_t f = 0; f < D; ++f) {
            const double bf = phi_of(kh[f], phi);
            zh[f] = gm * zh[f] + bf;
            for (int64_t e = 0; e < D; ++e)
                Sh[f * D + e] = gm * Sh[f * D + e] + bf * vh[e];
        }
        double den = 0.0;
        for (int64_t f = 0; f < D; ++f)
            den += phi_of(qh[f], phi) * zh[f];
        for (int64_t e = 0; e < D; ++e) {
            double num = 0.0;
            for (int64_t f = 0; f < D; ++f)
                num += phi_of(qh[f], phi) * Sh[f * D + e];
            oh[e] = num / den;
        }
    }
}
