/*
 * oracle/adjoint_fp64.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain fp64 CPU oracle of the gradient of the gated delta rule (the layer on
 * the IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
 * DeltaNet"; commentary blog, section 10) for the loss L = sum_t dO_t . o_t,
 * by reverse-mode differentiation of the token recurrence
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t.
 *
 * Written per token with u = S_{t-1} k_t, delta = beta_t (v_t - alpha_t u),
 * S_t = alpha_t S_{t-1} + delta k_t^T, and G = dL/dS_t:
 *
 *     G      += dO_t q_t^T                    (o_t = S_t q_t)
 *     dq_t    = S_t^T dO_t
 *     ddelta  = G k_t
 *     dv_t    = beta_t ddelta
 *     dbeta_t = ddelta . (v_t - alpha_t u)
 *     dalpha_t= <G, S_{t-1}> - beta_t ddelta . u
 *     dk_t    = G^T delta - alpha_t beta_t S_{t-1}^T ddelta
 *     G      <- alpha_t G - alpha_t beta_t ddelta k_t^T     (= dL/dS_{t-1})
 *
 * and dstate_in = G after the first token.  dstate_out (NULL = zeros) is
 * dL/dS of each sequence's final state, from a loss term outside the outputs
 * (a later part of the sequence, split off at that state): G starts from it
 * at the last token.  The forward states come from a first fp64 pass that
 * keeps every C-th state; each C-token span is then recomputed (C states)
 * before its backward sweep.
 *
 * Layouts (fp64, row-major): q, k, dq, dk [T, H, d_k]; v, dO, dv [T, H, d_v];
 * alpha, beta, dalpha, dbeta [T, H]; state_in, dstate_out, dstate_in
 * [N, H, d_v, d_k] (state_in NULL = zeros).  cu_seqlens [N+1] int32.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static void step_fwd(double* S, const double* k, const double* v, double a, double b, int dk, int dv)
{
    for (int i = 0; i < dv; ++i) {
        double u = 0.0;
        for (int j = 0; j < dk; ++j) u += S[(int64_t)i * dk + j] * k[j];
        const double d = b * (v[i] - a * u);
        for (int j = 0; j < dk; ++j) S[(int64_t)i * dk + j] = a * S[(int64_t)i * dk + j] + d * k[j];
    }
}

int oracle_adjoint_fp64(const double* q, const double* k, const double* v, const double* alpha,
                        const double* beta, const double* state_in, const double* dstate_out, const double* dO,
                        const int32_t* cu_seqlens, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C,
                        double* dq, double* dkk, double* dvv, double* dalpha, double* dbeta, double* dstate_in)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return 1;
    for (int32_t n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    const int64_t SZ = (int64_t)dv * dk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            const int64_t t0 = cu_seqlens[n];
            const int32_t L = cu_seqlens[n + 1] - cu_seqlens[n];
            const int32_t nspan = (L + C - 1) / C;
            /* checkpoints: the state at 0, C, 2C, ... */
            double* ck = (double*)malloc(sizeof(double) * (size_t)SZ * (size_t)(nspan + 1));
            double* hist = (double*)malloc(sizeof(double) * (size_t)SZ * (size_t)(C + 1));
            double* G = (double*)calloc((size_t)SZ, sizeof(double));
            double* dd = (double*)malloc(sizeof(double) * (size_t)dv);
            double* uu = (double*)malloc(sizeof(double) * (size_t)dv);
            double* de = (double*)malloc(sizeof(double) * (size_t)dv);
            if (!ck || !hist || !G || !dd || !uu || !de) {
                free(ck); free(hist); free(G); free(dd); free(uu); free(de);
                bad = 1;
                continue;
            }
            if (dstate_out) memcpy(G, dstate_out + ((int64_t)n * H + h) * SZ, sizeof(double) * (size_t)SZ);
            double* S = ck;
            if (state_in) memcpy(S, state_in + ((int64_t)n * H + h) * SZ, sizeof(double) * (size_t)SZ);
            else memset(S, 0, sizeof(double) * (size_t)SZ);
            for (int32_t c = 0; c < nspan; ++c) {
                memcpy(ck + (int64_t)(c + 1) * SZ, ck + (int64_t)c * SZ, sizeof(double) * (size_t)SZ);
                const int32_t len = (c + 1) * C <= L ? C : L - c * C;
                for (int32_t t = 0; t < len; ++t) {
                    const int64_t row = (t0 + (int64_t)c * C + t) * H + h;
                    step_fwd(ck + (int64_t)(c + 1) * SZ, k + row * dk, v + row * dv, alpha[row], beta[row], dk, dv);
                }
            }
            /* backward, span by span */
            for (int32_t c = nspan - 1; c >= 0; --c) {
                const int32_t len = (c + 1) * C <= L ? C : L - c * C;
                memcpy(hist, ck + (int64_t)c * SZ, sizeof(double) * (size_t)SZ);
                for (int32_t t = 0; t < len; ++t) {
                    const int64_t row = (t0 + (int64_t)c * C + t) * H + h;
                    memcpy(hist + (int64_t)(t + 1) * SZ, hist + (int64_t)t * SZ, sizeof(double) * (size_t)SZ);
                    step_fwd(hist + (int64_t)(t + 1) * SZ, k + row * dk, v + row * dv, alpha[row], beta[row], dk, dv);
                }
                for (int32_t t = len - 1; t >= 0; --t) {
                    const int64_t row = (t0 + (int64_t)c * C + t) * H + h;
                    const double* Sp = hist + (int64_t)t * SZ;       /* S_{t-1} */
                    const double* St = hist + (int64_t)(t + 1) * SZ; /* S_t */
                    const double* kt = k + row * dk;
                    const double* qt = q + row * dk;
                    const double* vt = v + row * dv;
                    const double* dOt = dO + row * dv;
                    const double a = alpha[row], b = beta[row];
                    for (int i = 0; i < dv; ++i)
                        for (int j = 0; j < dk; ++j) G[(int64_t)i * dk + j] += dOt[i] * qt[j];
                    for (int j = 0; j < dk; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < dv; ++i) s += St[(int64_t)i * dk + j] * dOt[i];
                        dq[row * dk + j] = s;
                    }
                    double db = 0.0, da = 0.0;
                    for (int i = 0; i < dv; ++i) {
                        double u = 0.0, g = 0.0, gs = 0.0;
                        for (int j = 0; j < dk; ++j) {
                            u += Sp[(int64_t)i * dk + j] * kt[j];
                            g += G[(int64_t)i * dk + j] * kt[j];
                            gs += G[(int64_t)i * dk + j] * Sp[(int64_t)i * dk + j];
                        }
                        uu[i] = u;
                        dd[i] = g;
                        de[i] = b * (vt[i] - a * u);
                        dvv[row * dv + i] = b * g;
                        db += g * (vt[i] - a * u);
                        da += gs - b * g * u;
                    }
                    dbeta[row] = db;
                    dalpha[row] = da;
                    for (int j = 0; j < dk; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < dv; ++i)
                            s += G[(int64_t)i * dk + j] * de[i] - a * b * Sp[(int64_t)i * dk + j] * dd[i];
                        dkk[row * dk + j] = s;
                    }
                    for (int i = 0; i < dv; ++i)
                        for (int j = 0; j < dk; ++j)
                            G[(int64_t)i * dk + j] = a * G[(int64_t)i * dk + j] - a * b * dd[i] * kt[j];
                }
            }
            if (dstate_in) memcpy(dstate_in + ((int64_t)n * H + h) * SZ, G, sizeof(double) * (size_t)SZ);
            free(ck); free(hist); free(G); free(dd); free(uu); free(de);
        }
    }
    return bad ? 2 : 0;
}
