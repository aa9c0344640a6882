/*
 * gdr_oracle.c -- fp64 CPU oracle for the key-axis-gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA path computes.  Only the test suite, the smoke
 * check and the bench's CPU-baseline / reference arm may load it.  It shares no
 * code, header, table or constant with the CUDA library and never calls it.
 *
 * What it computes (one head of one sequence, tokens t = 1..T):
 *
 *   S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + w_t v_t k_t^T,   o_t = S_t (scale q_t)
 *
 * with S_t in R^{dv x dk} (value rows, key columns), erase strength beta_t and write
 * strength w_t (w_t = beta_t, the tied delta rule, unless a separate w is given).  Sources:
 *   - "Semidirect Fourier Delta Attention" page, section "Core architecture":
 *     the update decays first, then erases along k_t, then writes beta_t k_t v_t^*;
 *     the state there is the transpose of ours (dk x dv, acting from the left).
 *     Transposing it gives the row-vector form used here.
 *   - same section, "real implementation": the complex diagonal Lambda_t =
 *     diag(alpha_t * exp(i theta_t)) is a direct sum of 2x2 rotation-decay blocks.
 *   - "CARVE" page, section 2.3: the decay is a key-axis exponential gate,
 *     D_t = diag(exp(g_t)) with g_t <= 0.
 *   - the readout o_t = S_t q_t uses the post-update state, so o_t sees the token's
 *     own write (the convention of this library; the CARVE page writes S_{t-1} q_t in
 *     section 2.1).
 *   - "CARVE" page, sections 2.1-2.2: an erase gate b_t and a separate scalar value
 *     write gate w_{h,t} per head and token.  Read here as the erase strength that
 *     multiplies the removal along k_t and the write strength that multiplies v_t k_t^T;
 *     with both equal the update is the original delta rule (section 3, Theorem 1).
 *
 * The token step, in the order the SFDA page gives it (decay, erase, write):
 *   1. alpha = exp(g_t) per key dim (rotation mode: per key pair j, with angle
 *      theta_{t,j}; the pair (2j, 2j+1) of every row of S is read as the complex
 *      number x + i y and multiplied by alpha e^{i theta}).  This is the
 *      transpose of Lambda_t acting on the left of the SFDA state.
 *   2. X = S D_t.
 *   3. e = w_t v_t - beta_t X k_t              (erase along k_t, write v_t)
 *   4. S = X + e k_t^T                          (write)
 *   5. o_t = S (scale q_t)
 *
 * Gate modes: GATE_LOGDECAY (0) takes g as given; GATE_NEG_SOFTPLUS (1) takes a
 * raw gate a and uses g = -softplus(a) = -(max(a,0) + log1p(exp(-|a|))),
 * the activation the configurations state ("g = -softplus(N(0,1))").
 *
 * Layouts (row-major, last index fastest):
 *   q, k [B,T,H,dk]; v, o [B,T,H,dv]; g [B,T,H,dk] ([B,T,H,dk/2] in rotation
 *   mode); beta, w [B,T,H]; theta [B,T,H,dk/2]; S0, S_T [B,H,dv,dk].
 * All arrays are double; bf16 or fp32 inputs are widened exactly by the caller.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static double oracle_log_decay(double g_in, int gate_mode)
{
    if (gate_mode == 1) {
        double a = g_in;
        double sp = (a > 0.0 ? a : 0.0) + log1p(exp(-fabs(a)));
        return -sp;
    }
    return g_in;
}

/*
 * One token of the recurrence on one head's state S (dv x dk, row-major).
 * g points at this token's dk (or dk/2) gate values, theta at dk/2 angles
 * (rotation mode only).  Writes o (dv values).
 */
static void oracle_token_step(int dk, int dv, int gate_mode, int rotation, double scale,
                              const double* q, const double* k, const double* v,
                              const double* g, double beta, double w, const double* theta,
                              double* S, double* o)
{
    /* 1-2: X = S D_t, in place. */
    if (!rotation) {
        for (int d = 0; d < dk; ++d) {
            double alpha = exp(oracle_log_decay(g[d], gate_mode));
            for (int i = 0; i < dv; ++i) S[(size_t)i * dk + d] *= alpha;
        }
    } else {
        for (int j = 0; j < dk / 2; ++j) {
            double alpha = exp(oracle_log_decay(g[j], gate_mode));
            double c = cos(theta[j]), s = sin(theta[j]);
            for (int i = 0; i < dv; ++i) {
                double x = S[(size_t)i * dk + 2 * j];
                double y = S[(size_t)i * dk + 2 * j + 1];
                S[(size_t)i * dk + 2 * j] = alpha * (c * x - s * y);
                S[(size_t)i * dk + 2 * j + 1] = alpha * (s * x + c * y);
            }
        }
    }
    /* 3-5: per value row, erase along k, write v, read out with q. */
    for (int i = 0; i < dv; ++i) {
        double* row = S + (size_t)i * dk;
        double xk = 0.0;
        for (int d = 0; d < dk; ++d) xk += row[d] * k[d];
        double e = w * v[i] - beta * xk;
        for (int d = 0; d < dk; ++d) row[d] += e * k[d];
        double oq = 0.0;
        for (int d = 0; d < dk; ++d) oq += row[d] * (scale * q[d]);
        o[i] = oq;
    }
}

/*
 * Whole-sequence forward, token by token.  w may be NULL (w = beta); S0 may be
 * NULL (zero state); S_T may be NULL (final state not wanted).  Heads run in
 * parallel with OpenMP.
 */
void oracle_gdr_fwd(int B, int T, int H, int dk, int dv, int gate_mode, int rotation,
                    double scale, const double* q, const double* k, const double* v,
                    const double* g, const double* beta, const double* w, const double* theta,
                    const double* S0, double* o, double* S_T)
{
    const int ng = rotation ? dk / 2 : dk;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        if (S0) memcpy(S, S0 + (size_t)bh * dv * dk, sizeof(double) * (size_t)dv * dk);
        else memset(S, 0, sizeof(double) * (size_t)dv * dk);
        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            oracle_token_step(dk, dv, gate_mode, rotation, scale,
                              q + tok * dk, k + tok * dk, v + tok * dv,
                              g + tok * ng, beta[tok], w ? w[tok] : beta[tok],
                              rotation ? theta + tok * (dk / 2) : NULL,
                              S, o + tok * dv);
        }
        if (S_T) memcpy(S_T + (size_t)bh * dv * dk, S, sizeof(double) * (size_t)dv * dk);
        free(S);
    }
}

/*
 * One recurrent decode step for N independent sequences: S [N,H,dv,dk] is
 * updated in place; q, k [N,H,dk]; v, o [N,H,dv]; g [N,H,dk] (or dk/2);
 * beta, w [N,H] (w may be NULL: w = beta); theta [N,H,dk/2].  It is the same
 * token step as the forward.
 */
void oracle_gdr_decode_step(int N, int H, int dk, int dv, int gate_mode, int rotation,
                            double scale, const double* q, const double* k, const double* v,
                            const double* g, const double* beta, const double* w,
                            const double* theta, double* S, double* o)
{
    const int ng = rotation ? dk / 2 : dk;
#pragma omp parallel for schedule(static)
    for (int nh = 0; nh < N * H; ++nh) {
        oracle_token_step(dk, dv, gate_mode, rotation, scale,
                          q + (size_t)nh * dk, k + (size_t)nh * dk, v + (size_t)nh * dv,
                          g + (size_t)nh * ng, beta[nh], w ? w[nh] : beta[nh],
                          rotation ? theta + (size_t)nh * (dk / 2) : NULL,
                          S + (size_t)nh * dv * dk, o + (size_t)nh * dv);
    }
}

/* Number of OpenMP threads the oracle's parallel loops use. */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
