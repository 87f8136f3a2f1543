/*
 * oracle/schedule_fp32.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Scalar CPU model, in IEEE fp32, of the arithmetic schedule that the CUDA
 * kernels are required to execute bit for bit.  It is written from the
 * schedule stated below, not from the kernels, and it shares no code with
 * them.  Only tests/,
 * __graft_entry__.smoke() and bench.py's cpu_baseline leg may load it.
 *
 * Every floating-point operation below is one IEEE-754 binary32 operation
 * rounded to nearest-even: '*', '+', '-' on floats (compiled with
 * -ffp-contract=off, SSE arithmetic, no excess precision) and fmaf() from
 * libm (a correctly rounded fused multiply-add).  Subnormals are kept.
 *
 * Sources of the method: the gated delta rule named on the IsoExec summary
 * page (section "Chunkwise-Parallel Recurrent (CPR) Gated DeltaNet"); CPR
 * itself from the same section (recurrence as the primary computation,
 * evaluated in parallel across chunks, hidden state re-synchronised every
 * C tokens in decode); the fixed reduction tree over contiguous K leaves
 * with FP32 accumulation from the same page, section "Achieving
 * Parallelism Invariance", and from the commentary blog, section 8.
 *
 * Schedule (NL = 8 leaves, L = d_k / 8):
 *   tree(x, y): leaf l = x[lL]*y[lL], then fma(x[lL+m], y[lL+m], .) for
 *               m = 1..L-1; result ((p0+p1)+(p2+p3)) + ((p4+p5)+(p6+p7)).
 *   P_tok on a running state kept as c * Rt (a scale c and a matrix Rt;
 *               c = 1 and Rt = the boundary state at a chunk's start), one
 *               token (k, v, q, a, b):
 *               kq = tree(k, q); cn = a * c;
 *               for every row i: dk = tree(Rt_i, k), dq = tree(Rt_i, q)
 *               (over Rt before the token), d = b * (v_i - cn * dk);
 *               if cn >= 2^-64:  dt = d * (1 / cn) (the reciprocal rounded),
 *                                Rt_ij = fma(dt, k_j, Rt_ij),
 *                                o_i = cn * fma(dt, kq, dq);   c = cn
 *               else (a fold):   Rt_ij = fma(d, k_j, cn * Rt_ij),
 *                                o_i = fma(d, kq, cn * dq);    c = 1.
 *   P_chunk(S; k_1..C, v_1..C, a_1..C, b_1..C):
 *               D[s][s] = 1, D[t][s] = D[t-1][s] * a_t          (t > s)
 *               c[t][s] = D[t][s] * tree(k_s, k_t)              (s < t)
 *               u0_t[i] = b_t * chain_{s<t} fma(-c[t][s], u0_s[i], .)
 *                         starting from v_t[i]
 *               w_t[j]  = b_t * chain_{s<t} fma(-c[t][s], w_s[j], .)
 *                         starting from D[t][0] * k_t[j]
 *               e_t[i]  = D[C][t] * (u0_t[i] - tree(S_i, w_t))
 *               S'_ij   = chain_{t=1..C} fma(e_t[i], k_t[j], .)
 *                         starting from D[C][0] * S_ij
 *   Composition: B_0 = state_in, B_{n+1} = P_chunk(B_n, chunk n); the
 *   outputs of chunk n come from P_tok steps started at (c = 1, Rt = B_n).
 *   Decode runs P_tok on a running state (c, Rt) and, once C tokens are
 *   buffered, sets S_b = P_chunk(S_b, buffer), Rt = S_b, c = 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NL 8

static float tree32(const float* x, const float* y, int dk)
{
    const int L = dk / NL;
    float p[NL];
    for (int l = 0; l < NL; ++l) {
        float acc = x[l * L] * y[l * L];
        for (int m = 1; m < L; ++m) acc = fmaf(x[l * L + m], y[l * L + m], acc);
        p[l] = acc;
    }
    return ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
}

/* The scale below which a decay is folded into the matrix (2^-64). */
#define FOLD_TAU 0x1p-64f

/* One P_tok step on a running state c * Rt (Rt d_v x d_k and *c updated in
 * place); writes o[d_v]. */
static void p_tok(float* R, float* c, const float* k, const float* v, const float* q,
                  float a, float b, int dk, int dv, float* o)
{
    const float kq = tree32(k, q, dk);
    const float cn = a * *c;
    const int fold = !(cn >= FOLD_TAU);
    const float rc = fold ? 1.0f : 1.0f / cn;
    for (int i = 0; i < dv; ++i) {
        float* Ri = R + (int64_t)i * dk;
        const float dkv = tree32(Ri, k, dk);
        const float dqv = tree32(Ri, q, dk);
        const float cu = cn * dkv;
        const float r = v[i] - cu;
        const float d = b * r;
        if (!fold) {
            const float dt = d * rc;
            const float t = fmaf(dt, kq, dqv);
            o[i] = cn * t;
            for (int j = 0; j < dk; ++j) Ri[j] = fmaf(dt, k[j], Ri[j]);
        } else {
            const float cdq = cn * dqv;
            o[i] = fmaf(d, kq, cdq);
            for (int j = 0; j < dk; ++j) {
                const float cR = cn * Ri[j];
                Ri[j] = fmaf(d, k[j], cR);
            }
        }
    }
    *c = fold ? 1.0f : cn;
}

/*
 * P_chunk on a d_v x d_k boundary state S (in place).  kc/vc point at the
 * first of C tokens, consecutive tokens kstride/vstride floats apart;
 * ac/bc likewise with gstride.
 */
static int p_chunk(float* S, const float* kc, int64_t kstride, const float* vc, int64_t vstride,
                   const float* ac, const float* bc, int64_t gstride, int dk, int dv, int C)
{
    const int C1 = C + 1;
    float* D  = (float*)malloc(sizeof(float) * (size_t)C1 * C1);
    float* c  = (float*)malloc(sizeof(float) * (size_t)C1 * C1);
    float* u0 = (float*)malloc(sizeof(float) * (size_t)C1 * dv);
    float* w  = (float*)malloc(sizeof(float) * (size_t)C1 * dk);
    float* e  = (float*)malloc(sizeof(float) * (size_t)C1 * dv);
    if (!D || !c || !u0 || !w || !e) { free(D); free(c); free(u0); free(w); free(e); return 2; }
    /* tokens are 1-indexed inside the chunk: token t lives at kc + (t-1)*kstride */
#define KT(t) (kc + (int64_t)((t) - 1) * kstride)
#define VT(t) (vc + (int64_t)((t) - 1) * vstride)
#define AT(t) (ac[(int64_t)((t) - 1) * gstride])
#define BT(t) (bc[(int64_t)((t) - 1) * gstride])
    for (int s = 0; s <= C; ++s) {
        D[s * C1 + s] = 1.0f;
        for (int t = s + 1; t <= C; ++t) D[t * C1 + s] = D[(t - 1) * C1 + s] * AT(t);
    }
    for (int t = 2; t <= C; ++t)
        for (int s = 1; s < t; ++s) {
            const float G = tree32(KT(s), KT(t), dk);
            c[t * C1 + s] = D[t * C1 + s] * G;
        }
    for (int t = 1; t <= C; ++t) {
        const float bt = BT(t);
        for (int i = 0; i < dv; ++i) {
            float acc = VT(t)[i];
            for (int s = 1; s < t; ++s) acc = fmaf(-c[t * C1 + s], u0[s * dv + i], acc);
            u0[t * dv + i] = bt * acc;
        }
        for (int j = 0; j < dk; ++j) {
            float acc = D[t * C1 + 0] * KT(t)[j];
            for (int s = 1; s < t; ++s) acc = fmaf(-c[t * C1 + s], w[s * dk + j], acc);
            w[t * dk + j] = bt * acc;
        }
    }
    for (int t = 1; t <= C; ++t)
        for (int i = 0; i < dv; ++i) {
            const float sw = tree32(S + (int64_t)i * dk, w + t * dk, dk);
            const float delta = u0[t * dv + i] - sw;
            e[t * dv + i] = D[C * C1 + t] * delta;
        }
    const float DC0 = D[C * C1 + 0];
    for (int i = 0; i < dv; ++i)
        for (int j = 0; j < dk; ++j) {
            float acc = DC0 * S[(int64_t)i * dk + j];
            for (int t = 1; t <= C; ++t) acc = fmaf(e[t * dv + i], KT(t)[j], acc);
            S[(int64_t)i * dk + j] = acc;
        }
#undef KT
#undef VT
#undef AT
#undef BT
    free(D); free(c); free(u0); free(w); free(e);
    return 0;
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs). */
static uint16_t f32_to_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void sched_f32_to_bf16(const float* x, uint16_t* y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) y[i] = f32_to_bf16_bits(x[i]);
}

/*
 * CPR forward (prefill / trainer forward) under the schedule.
 * Layouts as the fp64 oracle, in fp32.  Also fills the decode cache for a
 * continuation when the cache pointers are non-NULL: S_b, R [N,H,dv,dk],
 * kbuf [N,H,C,dk], vbuf [N,H,C,dv], abuf/bbuf [N,H,C], pos [N,H], and
 * Rs_out [N,H] the running state's scale (the running state is Rs * R).
 */
int sched_forward(const float* q, const float* k, const float* v,
                  const float* alpha, const float* beta, const float* state_in,
                  const int32_t* cu_seqlens, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C,
                  float* o, float* states,
                  float* S_b, float* R_out, float* kbuf, float* vbuf, float* abuf, float* bbuf,
                  int32_t* pos, float* Rs_out)
{
    if (N < 0 || H <= 0 || dk <= 0 || dk % NL || dv <= 0 || C <= 0) return 1;
    int64_t* soff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N + 1));
    if (!soff) return 2;
    soff[0] = 0;
    for (int32_t n = 0; n < N; ++n) {
        const int32_t L = cu_seqlens[n + 1] - cu_seqlens[n];
        if (L < 0) { free(soff); return 1; }
        soff[n + 1] = soff[n] + L / C + 1;
    }
    const int64_t SZ = (int64_t)dv * dk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            float* B = (float*)malloc(sizeof(float) * (size_t)SZ);
            float* R = (float*)malloc(sizeof(float) * (size_t)SZ);
            if (!B || !R) { free(B); free(R); bad = 1; continue; }
            if (state_in) memcpy(B, state_in + ((int64_t)n * H + h) * SZ, sizeof(float) * (size_t)SZ);
            else memset(B, 0, sizeof(float) * (size_t)SZ);
            int64_t slot = soff[n];
            memcpy(states + (slot * H + h) * SZ, B, sizeof(float) * (size_t)SZ);
            const int32_t t0 = cu_seqlens[n], L = cu_seqlens[n + 1] - t0;
            memcpy(R, B, sizeof(float) * (size_t)SZ);
            float rs = 1.0f;
            for (int32_t c0 = 0; c0 < L; c0 += C) {
                const int32_t len = (L - c0 < C) ? (L - c0) : C;
                memcpy(R, B, sizeof(float) * (size_t)SZ);
                rs = 1.0f;
                for (int32_t t = 0; t < len; ++t) {
                    const int64_t tok = (int64_t)(t0 + c0 + t) * H + h;
                    p_tok(R, &rs, k + tok * dk, v + tok * dv, q + tok * dk, alpha[tok], beta[tok],
                          dk, dv, o + tok * dv);
                }
                if (len == C) {
                    const int64_t tok = (int64_t)(t0 + c0) * H + h;
                    if (p_chunk(B, k + tok * dk, (int64_t)H * dk, v + tok * dv, (int64_t)H * dv,
                                alpha + tok, beta + tok, H, dk, dv, C)) { bad = 1; break; }
                    ++slot;
                    memcpy(states + (slot * H + h) * SZ, B, sizeof(float) * (size_t)SZ);
                }
            }
            const int32_t p = L % C;
            const int64_t nh = (int64_t)n * H + h;
            if (S_b) memcpy(S_b + nh * SZ, B, sizeof(float) * (size_t)SZ);
            if (R_out) memcpy(R_out + nh * SZ, p ? R : B, sizeof(float) * (size_t)SZ);
            if (Rs_out) Rs_out[nh] = p ? rs : 1.0f;
            if (pos) pos[nh] = p;
            for (int32_t s = 0; s < p; ++s) {
                const int64_t tok = (int64_t)(t0 + L - p + s) * H + h;
                if (kbuf) memcpy(kbuf + (nh * C + s) * dk, k + tok * dk, sizeof(float) * (size_t)dk);
                if (vbuf) memcpy(vbuf + (nh * C + s) * dv, v + tok * dv, sizeof(float) * (size_t)dv);
                if (abuf) abuf[nh * C + s] = alpha[tok];
                if (bbuf) bbuf[nh * C + s] = beta[tok];
            }
            free(B); free(R);
        }
    }
    free(soff);
    return bad ? 2 : 0;
}

/*
 * One decode step for N sequences under the schedule (cache updated in
 * place).  q,k [N,H,dk], v [N,H,dv], alpha/beta [N,H]; o [N,H,dv].
 */
int sched_decode_step(const float* q, const float* k, const float* v,
                      const float* alpha, const float* beta,
                      float* S_b, float* R, float* kbuf, float* vbuf, float* abuf, float* bbuf,
                      int32_t* pos, float* Rs, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C, float* o)
{
    if (N < 0 || H <= 0 || dk <= 0 || dk % NL || dv <= 0 || C <= 0) return 1;
    const int64_t SZ = (int64_t)dv * dk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            const int64_t nh = (int64_t)n * H + h;
            int32_t p = pos[nh];
            if (p < 0 || p >= C) { bad = 1; continue; }
            p_tok(R + nh * SZ, Rs + nh, k + nh * dk, v + nh * dv, q + nh * dk, alpha[nh], beta[nh],
                  dk, dv, o + nh * dv);
            memcpy(kbuf + (nh * C + p) * dk, k + nh * dk, sizeof(float) * (size_t)dk);
            memcpy(vbuf + (nh * C + p) * dv, v + nh * dv, sizeof(float) * (size_t)dv);
            abuf[nh * C + p] = alpha[nh];
            bbuf[nh * C + p] = beta[nh];
            ++p;
            if (p == C) {
                if (p_chunk(S_b + nh * SZ, kbuf + nh * C * dk, dk, vbuf + nh * C * dv, dv,
                            abuf + nh * C, bbuf + nh * C, 1, dk, dv, C)) { bad = 1; continue; }
                memcpy(R + nh * SZ, S_b + nh * SZ, sizeof(float) * (size_t)SZ);
                Rs[nh] = 1.0f;
                p = 0;
            }
            pos[nh] = p;
        }
    }
    return bad ? 2 : 0;
}

/*
 * P_tok over every chunk, started from GIVEN boundary states (layout of the
 * forward's chunk_states).  o [T,H,dv] fp32 before the output cast; R_final
 * [N,H,dv,dk] and Rs_final [N,H]: the running state (Rs * R) after each
 * sequence's last token (the boundary state itself, scale 1, when
 * L % C == 0).  This isolates the per-token schedule from how the boundary
 * states were produced.
 */
int sched_tok_from_states(const float* q, const float* k, const float* v,
                          const float* alpha, const float* beta, const float* states,
                          const int32_t* cu_seqlens, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C,
                          float* o, float* R_final, float* Rs_final)
{
    if (N < 0 || H <= 0 || dk <= 0 || dk % NL || dv <= 0 || C <= 0) return 1;
    int64_t* soff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N + 1));
    if (!soff) return 2;
    soff[0] = 0;
    for (int32_t n = 0; n < N; ++n) {
        const int32_t L = cu_seqlens[n + 1] - cu_seqlens[n];
        if (L < 0) { free(soff); return 1; }
        soff[n + 1] = soff[n] + L / C + 1;
    }
    const int64_t SZ = (int64_t)dv * dk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t n = 0; n < N; ++n) {
        for (int32_t h = 0; h < H; ++h) {
            float* R = (float*)malloc(sizeof(float) * (size_t)SZ);
            if (!R) { bad = 1; continue; }
            const int32_t t0 = cu_seqlens[n], L = cu_seqlens[n + 1] - t0;
            memcpy(R, states + (soff[n] * H + h) * SZ, sizeof(float) * (size_t)SZ);
            float rs = 1.0f;
            for (int32_t c0 = 0; c0 < L; c0 += C) {
                memcpy(R, states + ((soff[n] + c0 / C) * H + h) * SZ, sizeof(float) * (size_t)SZ);
                rs = 1.0f;
                const int32_t len = (L - c0 < C) ? (L - c0) : C;
                for (int32_t t = 0; t < len; ++t) {
                    const int64_t tok = (int64_t)(t0 + c0 + t) * H + h;
                    p_tok(R, &rs, k + tok * dk, v + tok * dv, q + tok * dk, alpha[tok], beta[tok], dk, dv,
                          o + tok * dv);
                }
            }
            const int64_t nh = (int64_t)n * H + h;
            if (R_final) {
                if (L % C == 0)
                    memcpy(R_final + nh * SZ, states + ((soff[n] + L / C) * H + h) * SZ, sizeof(float) * (size_t)SZ);
                else
                    memcpy(R_final + nh * SZ, R, sizeof(float) * (size_t)SZ);
            }
            if (Rs_final) Rs_final[nh] = (L % C == 0) ? 1.0f : rs;
            free(R);
        }
    }
    free(soff);
    return bad ? 2 : 0;
}
