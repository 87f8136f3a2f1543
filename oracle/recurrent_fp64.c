/*
 * oracle/recurrent_fp64.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain fp64 CPU oracle of the gated delta rule, evaluated token by token.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
 * load this code; the product path never does.
 *
 * What it computes (Gated DeltaNet as named on the IsoExec summary page,
 * section "Chunkwise-Parallel Recurrent (CPR) Gated DeltaNet", and on the
 * IsoExec commentary blog, section 10 "Gated DeltaNet"):
 *
 *     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * with S a d_v x d_k matrix (row i = one value channel), per sequence and
 * per head.  In exact arithmetic the chunkwise-parallel recurrent (CPR)
 * evaluation reaches exactly this result, so this recurrence is the
 * oracle for every output and every chunk-boundary state.
 *
 * The product S (I - beta k k^T) is evaluated as S - beta (S k) k^T
 * (distributivity), which avoids forming the d_k x d_k matrix; the
 * exact-rational oracle (oracle/exact.py) forms that matrix literally.
 *
 * Layouts (all fp64, row-major):
 *   q, k      [T_total, H, d_k]      v, o [T_total, H, d_v]
 *   alpha,beta[T_total, H]
 *   state_in  [N, H, d_v, d_k]       (NULL = zeros)
 *   states    [sum_n (L_n / C + 1), H, d_v, d_k]: the state at positions
 *             0, C, 2C, ... of every sequence (sequence-local positions)
 *   final     [N, H, d_v, d_k]: the state after the last token.
 * cu_seqlens [N+1] int32, non-decreasing, cu_seqlens[0] = 0.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

int oracle_recurrent_fp64(const double* q, const double* k, const double* v,
                          const double* alpha, const double* beta,
                          const double* state_in, const int32_t* cu_seqlens,
                          int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C,
                          double* o, double* states, double* final_state)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return 1;
    /* first chunk-state slot of every sequence */
    int64_t* soff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N + 1));
    if (!soff) return 2;
    soff[0] = 0;
    for (int32_t n = 0; n < N; ++n) {
        int32_t L = cu_seqlens[n + 1] - cu_seqlens[n];
        if (L < 0) { free(soff); return 1; }
        soff[n + 1] = soff[n] + L / C + 1;
    }
    const int64_t SZ = (int64_t)dv * dk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            double* S  = (double*)malloc(sizeof(double) * (size_t)SZ);
            double* Sk = (double*)malloc(sizeof(double) * (size_t)dv);
            if (!S || !Sk) { free(S); free(Sk); bad = 1; continue; }
            if (state_in) memcpy(S, state_in + ((int64_t)n * H + h) * SZ, sizeof(double) * (size_t)SZ);
            else memset(S, 0, sizeof(double) * (size_t)SZ);
            int64_t slot = soff[n];
            if (states) memcpy(states + (slot * H + h) * SZ, S, sizeof(double) * (size_t)SZ);
            const int32_t t0 = cu_seqlens[n], L = cu_seqlens[n + 1] - t0;
            for (int32_t p = 0; p < L; ++p) {
                const int64_t tok = (int64_t)(t0 + p) * H + h;
                const double* kt = k + tok * dk;
                const double* qt = q + tok * dk;
                const double* vt = v + tok * dv;
                const double a = alpha[tok], b = beta[tok];
                /* (S k) */
                for (int32_t i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * kt[j];
                    Sk[i] = acc;
                }
                /* S <- alpha (S - beta (S k) k^T) + beta v k^T */
                for (int32_t i = 0; i < dv; ++i)
                    for (int32_t j = 0; j < dk; ++j) {
                        double* s = &S[(int64_t)i * dk + j];
                        *s = a * (*s - b * Sk[i] * kt[j]) + b * vt[i] * kt[j];
                    }
                /* o = S q */
                double* ot = o + tok * dv;
                for (int32_t i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * qt[j];
                    ot[i] = acc;
                }
                if ((p + 1) % C == 0) {
                    ++slot;
                    if (states) memcpy(states + (slot * H + h) * SZ, S, sizeof(double) * (size_t)SZ);
                }
            }
            if (final_state) memcpy(final_state + ((int64_t)n * H + h) * SZ, S, sizeof(double) * (size_t)SZ);
            free(S); free(Sk);
        }
    }
    free(soff);
    return bad ? 2 : 0;
}
