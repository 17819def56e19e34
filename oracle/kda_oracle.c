/*
 * kda_oracle.c -- plain, slow, fp64 CPU oracle of the Kimi Delta Attention (KDA) operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this library.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (one (sequence, head) slice at a time, token by token):
 *
 *   KDA is Gated DeltaNet with the scalar per-head gate replaced by a per-channel (feature-dimension)
 *   gate ("Kimi K3 구조 분석" page, key messages; llm-wiki "Kimi K3" chapter, §1 "GatedDeltaNet과 KDA의
 *   차이").  The state S is a fixed-size dk x dv matrix updated once per token and read by
 *   multiplying the query into it (llm-wiki chapter, §1).  Written out, the gated delta rule with a
 *   channel-wise decay on the key dimension is
 *
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,     o_t = S_t^T q_t,
 *
 *   and the per-step log-decay is floored at ln(0.0067): every step keeps at least 0.67 % of what
 *   it held (orkas.ai "Kimi K3 architecture" post, section "GPU 코드 경로 하나를 없앤 하한").
 *
 *   The loop below takes the steps in that order, with no blocking or reordering:
 *       lambda = max(log_alpha_t, ln 0.0067)        (fmax: a NaN log-decay becomes the floor)
 *       S     <- Diag(exp(lambda)) S
 *       p      = S^T k_t
 *       u      = beta_t (v_t - p)
 *       S     <- S + k_t u^T                         (together: (I - beta k k^T) Diag(alpha) S + beta k v^T)
 *       o_t    = S^T q_t
 *
 * Optional outputs: the state after chosen token counts ("marks"; used for the 512-token prefix-
 * reuse checkpoints of the serving section of the orkas.ai post, and for segment boundaries), the
 * final state, and the cumulative transition prod_t (I - beta_t k_t k_t^T) Diag(alpha_t), i.e. the
 * same per-step map applied to an identity dk x dk matrix with v = 0 (the "cumulative transition"
 * of the sequence-split paragraph of the same serving section).
 *
 * segment compose: X_0 = initial state, X_{s+1} = M_s X_s + Z_s, where (M_s, Z_s) are a segment's
 * cumulative transition and zero-start final state (orkas.ai post, serving section, sequence split).
 *
 * Inputs are single-precision arrays holding the exact values given to the GPU (bf16 values are
 * exactly representable in fp32); all arithmetic is in double.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

double oracle_decay_floor(void) { return log(0.0067); }

/*
 * One (sequence, head) slice.  q, k: [T, dk]; v: [T, dv]; log_alpha: [T, dk]; beta: [T]; all
 * contiguous.  s0: [dk, dv] row-major or NULL (= zero).  o: [T, dv] or NULL.  s_final: [dk, dv] or
 * NULL.  marks: n_marks strictly increasing token counts in [1, T]; mark_states receives the state
 * after marks[m] tokens at [m, dk, dv].  transition: [dk, dk] or NULL.
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
int oracle_kda_seq(long T, int dk, int dv,
                   const float* q, const float* k, const float* v,
                   const float* log_alpha, const float* beta,
                   const double* s0,
                   double* o, double* s_final,
                   long n_marks, const long* marks, double* mark_states,
                   double* transition)
{
    if (T < 0 || dk <= 0 || dv <= 0) return -1;
    if (n_marks > 0 && (!marks || !mark_states)) return -1;
    const double lfloor = log(0.0067);
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* a = (double*)malloc(sizeof(double) * dk);
    double* p = (double*)malloc(sizeof(double) * (dv > dk ? dv : dk));
    double* M = transition ? (double*)calloc((size_t)dk * dk, sizeof(double)) : NULL;
    if (!S || !a || !p || (transition && !M)) { free(S); free(a); free(p); free(M); return -1; }
    if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);
    if (M) for (int i = 0; i < dk; ++i) M[(size_t)i * dk + i] = 1.0;
    long next_mark = 0;

    for (long t = 0; t < T; ++t) {
        const float* qt = q + t * dk;
        const float* kt = k + t * dk;
        const float* vt = v + t * dv;
        const float* lt = log_alpha + t * dk;
        const double bt = (double)beta[t];
        for (int i = 0; i < dk; ++i) a[i] = exp(fmax((double)lt[i], lfloor));

        /* S <- Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a[i];
        /* p = S^T k */
        for (int j = 0; j < dv; ++j) p[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            for (int j = 0; j < dv; ++j) p[j] += S[(size_t)i * dv + j] * ki;
        }
        /* u = beta (v - p);  S <- S + k u^T */
        for (int j = 0; j < dv; ++j) p[j] = bt * ((double)vt[j] - p[j]);
        for (int i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += ki * p[j];
        }
        /* o_t = S^T q */
        if (o) {
            double* ot = o + t * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = (double)qt[i];
                for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)i * dv + j] * qi;
            }
        }
        /* the same step map applied to the transition, with v = 0 */
        if (M) {
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dk; ++j) M[(size_t)i * dk + j] *= a[i];
            for (int j = 0; j < dk; ++j) p[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double ki = (double)kt[i];
                for (int j = 0; j < dk; ++j) p[j] += M[(size_t)i * dk + j] * ki;
            }
            for (int j = 0; j < dk; ++j) p[j] = -bt * p[j];
            for (int i = 0; i < dk; ++i) {
                const double ki = (double)kt[i];
                for (int j = 0; j < dk; ++j) M[(size_t)i * dk + j] += ki * p[j];
            }
        }
        while (next_mark < n_marks && marks[next_mark] == t + 1) {
            memcpy(mark_states + (size_t)next_mark * dk * dv, S, sizeof(double) * (size_t)dk * dv);
            ++next_mark;
        }
    }
    /* a mark at 0 tokens (or any mark not reached) gets the state as it stands */
    while (next_mark < n_marks) {
        if (marks[next_mark] == 0 && s0)
            memcpy(mark_states + (size_t)next_mark * dk * dv, s0, sizeof(double) * (size_t)dk * dv);
        else if (marks[next_mark] == 0)
            memset(mark_states + (size_t)next_mark * dk * dv, 0, sizeof(double) * (size_t)dk * dv);
        else { free(S); free(a); free(p); free(M); return -1; }
        ++next_mark;
    }
    if (s_final) memcpy(s_final, S, sizeof(double) * (size_t)dk * dv);
    if (M) memcpy(transition, M, sizeof(double) * (size_t)dk * dk);
    free(S); free(a); free(p); free(M);
    return 0;
}

/*
 * Segment composition for one (sequence, head): X_0 = x0 (or zero when NULL);
 * starts[s] = X_s; X_{s+1} = M_s X_s + Z_s; end = X_nseg.
 * M: [nseg, dk, dk]; Z: [nseg, dk, dv]; starts: [nseg, dk, dv] or NULL; end: [dk, dv] or NULL.
 */
int oracle_segment_compose(int nseg, int dk, int dv,
                           const double* M, const double* Z, const double* x0,
                           double* starts, double* end)
{
    if (nseg < 0 || dk <= 0 || dv <= 0) return -1;
    const size_t nS = (size_t)dk * dv;
    double* X = (double*)calloc(nS, sizeof(double));
    double* Y = (double*)malloc(sizeof(double) * nS);
    if (!X || !Y) { free(X); free(Y); return -1; }
    if (x0) memcpy(X, x0, sizeof(double) * nS);
    for (int s = 0; s < nseg; ++s) {
        if (starts) memcpy(starts + (size_t)s * nS, X, sizeof(double) * nS);
        const double* Ms = M + (size_t)s * dk * dk;
        const double* Zs = Z + (size_t)s * nS;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = Zs[(size_t)i * dv + j];
                for (int m = 0; m < dk; ++m) acc += Ms[(size_t)i * dk + m] * X[(size_t)m * dv + j];
                Y[(size_t)i * dv + j] = acc;
            }
        memcpy(X, Y, sizeof(double) * nS);
    }
    if (end) memcpy(end, X, sizeof(double) * nS);
    free(X); free(Y);
    return 0;
}

/*
 * MXFP8 inputs.  The til.kil9.dev "Kimi K3 기술 보고서" post (deployment paragraph) says the released
 * model was trained quantisation-aware with MXFP8 activations, so q, k and v may arrive in that form.
 * The format is the OCP Microscaling Formats (MX) v1.0 one: blocks of 32 consecutive elements share one
 * E8M0 scale X, each element is an FP8 E4M3 number P_i, and the element's value is X * P_i.  Here the
 * blocks run along the head dimension of each (token, head) row.
 *
 * E4M3: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent field 0 is subnormal,
 * 2^-6 * m / 8; otherwise 2^(e - 7) * (1 + m / 8); exponent 15 with mantissa 7 is NaN (there are no
 * infinities, and the largest finite magnitude is 448).
 * E8M0: 8 exponent bits, no sign and no mantissa: 2^(e - 127); e = 255 is NaN.
 */
double oracle_e4m3_value(unsigned char b)
{
    const int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

double oracle_e8m0_value(unsigned char e)
{
    if (e == 255) return NAN;
    return ldexp(1.0, (int)e - 127);
}

/*
 * Decodes n rows of d MXFP8 elements: codes [n, d], scales [n, d / block] -> out [n, d] in double.
 * Returns 0, or -1 on a bad argument (block must divide d).
 */
int oracle_mxfp8_decode(long n, int d, int block, const unsigned char* codes, const unsigned char* scales,
                        double* out)
{
    if (n < 0 || d <= 0 || block <= 0 || d % block != 0) return -1;
    const int nb = d / block;
    for (long r = 0; r < n; ++r)
        for (int i = 0; i < d; ++i)
            out[r * d + i] = oracle_e8m0_value(scales[r * nb + i / block]) * oracle_e4m3_value(codes[r * d + i]);
    return 0;
}
