/*
 * CPU oracle for the BinaryAttention forward pass.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check
 * and the benchmark's CPU-baseline / reference arm load this library. The GPU
 * path never calls it and shares no code with it: no headers, no helpers, no
 * tables. It is plain, slow and written to be checked against the pages by eye.
 *
 * Sources (cited by page title and section):
 *   [ES] "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 *        Transformers", Spanish technical summary ("Resumen técnico"),
 *        §2 Metodología.
 *   [KO] the same title, Korean technical summary ("기술 요약"),
 *        §2 방법론 나 (core components) and 다 (hardware-aware implementation).
 *
 * What is computed, for every (b, h, i) query row of an [B, H, N, d] problem:
 *   1. sigma(x) = +1 if x >= 0 else -1                  ([ES] §2, scaled binary
 *      representations: s_i = mu_q * sign(q_i), t_j = mu_k * sign(k_j)).
 *      x >= 0 is evaluated on the stored value, so +0.0 and -0.0 both give +1.
 *   2. alpha(token) = (1/d) * sum_c |x_c| over the d real channels: the scale
 *      mu of [ES] §2, read as the per-token mean absolute value ([KO] §2 나-1
 *      names a token-axis mean used as the scaling factor).
 *   3. S_ij = sum_c sigma(q_ic) * sigma(k_jc): an explicit +-1 dot product
 *      (what XNOR + popcount evaluate, [ES] §2 and [KO] §2 나-1).
 *   4. logit_ij = softmax_scale * alpha_q_i * alpha_k_j * S_ij + bias[h, i, j]
 *      (learnable additive bias b_ij, [ES] §2 "Mejora mediante Sesgo";
 *      [KO] §2 나-2). The bias is not multiplied by softmax_scale; a NULL bias
 *      means zero. The bias is shared by every batch index b.
 *   5. P_ij = exp(logit_ij - max_j logit_ij) / sum_j exp(...) over all N keys
 *      (ordinary softmax attention; no mask).
 *   6. O_i = sum_j P_ij * V_j, dense, fp64 ([ES] §2 implementation follows
 *      FlashAttention2, whose tiling gives exactly this result).
 *
 * All arithmetic is IEEE double. bf16 inputs are widened exactly (the 16 bits
 * become the top half of a float). Rows are processed in parallel with OpenMP;
 * each row's arithmetic is sequential in the order written above.
 *
 * Besides O, oracle_forward_spread(_rows) returns, for every output element,
 * E_ic = sum_j P_ij * |V_jc - O_ic|: how far the values a row averages lie
 * from their average. Rounding each P_ij to an 8-bit significand (relative
 * 2^-9), with the row sum taken from the same rounded values, moves O_ic by at
 * most about 2^-8 * E_ic; the GPU parity tests use it as that element's bound
 * where it exceeds the fixed one. It is a plain definition, not a method step.
 *
 * The 8-bit P.V variant ([ES] §2 "Cuantización Híbrida": attention
 * coefficients, range [0, 1], in a static unsigned 8-bit code; values in a
 * per-channel 8-bit code; [KO] §2 나-3; [ES] §2 "Implementación en Hardware":
 * mma.s32.u8.s8.s32) is oracle_forward_int8(_rows), read as:
 *   7. per (b, h, channel c): s_c = max_j |V_jc| / 127 and
 *      vq_jc = rint(V_jc / s_c) (round half to even, clamped to [-127, 127]),
 *      both in fp32, the precision in which the GPU takes these integer
 *      decisions; s_c = 0 gives vq = 0;
 *   8. u_ij = rint(255 * exp(logit_ij - m_i)) with m_i = max_j logit_ij, so
 *      every u is in [0, 255] and the row max gets 255;
 *   9. O_ic = s_c * (sum_j u_ij vq_jc) / (sum_j u_ij), the row sum taken from
 *      the same 8-bit weights.
 *
 * The position-sensitive bias ([ES] §2 "Mejora mediante Sesgo", which names
 * dense, position-sensitive and context-aware forms; [KO] §2 나-2) is read as a
 * relative-position table, expanded to the dense bias by
 * oracle_expand_relpos_bias:
 *  10. tokens n_cls .. N - 1 are the patches of a gh x gw grid in row-major
 *      order (patch p at row p / gw, column p % gw); n_cls (0 or 1) class
 *      tokens come first. For two patches, bias[h, i, j] =
 *      table[h, (y_i - y_j + gh - 1) * (2 gw - 1) + (x_i - x_j + gw - 1)];
 *      with R0 = (2 gh - 1)(2 gw - 1), a class query and a patch key take
 *      table[h, R0], a patch query and a class key table[h, R0 + 1], class
 *      with class table[h, R0 + 2]. The table is bf16 [H, R0 + 3 n_cls].
 *
 * The backward (oracle_backward) gives the gradients of a loss that the
 * forward fixes exactly, for an upstream gradient dO = dLoss/dO (bf16
 * [B, H, N, d]). With s_i = alpha_q_i * sigma(q_i) and t_j = alpha_k_j *
 * sigma(k_j), the scaled binary representations of [ES] §2, the logit of
 * step 4 is softmax_scale * <s_i, t_j> + bias[h, i, j], and:
 *  11. dV_j = sum_i P_ij * dO_i;
 *  12. dP_ij = <dO_i, V_j> and D_i = sum_j P_ij * dP_ij;
 *  13. dlogit_ij = P_ij * (dP_ij - D_i), the softmax's Jacobian applied to dP;
 *  14. ds_i = softmax_scale * sum_j dlogit_ij * t_j and
 *      dt_j = softmax_scale * sum_i dlogit_ij * s_i;
 *  15. dbias[h, i, j] = sum_b dlogit_bhij (one bias serves every b).
 * Training ([ES] §2 "Entrenamiento y Optimización": quantisation-aware
 * training with self-distillation; [KO] §2 다) also needs the gradient through
 * sigma and the mean to q and k; the pages give no estimator for it, so the
 * backward stops at s and t. Under the straight-through reading, dq = ds.
 *
 * Parity pins for each function live in the CPU test suite (exhaustive sign
 * predicate, packbits layout, Hamming identity, closed forms, invariants and an
 * independent numpy formulation on small cases).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* Exact widening of one stored element to double. */
static double load_elem(const void *x, int dtype, size_t idx)
{
    if (dtype == ORACLE_BF16) {
        uint32_t u = ((uint32_t)((const uint16_t *)x)[idx]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)x)[idx];
}

/* Step 1: the sign used by the method. x >= 0 maps to +1 (so -0.0 -> +1). */
static double sign_pm1(double x)
{
    return x >= 0.0 ? 1.0 : -1.0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Signs and scales of every token of one [T, d] tensor (T = B*H*N):
 * sig[t*d + c] = sigma(x[t, c]) as +-1.0 and alpha[t] = mean_c |x[t, c]|.
 */
static void signs_and_scales(const void *x, int dtype, size_t T, long d,
                             double *sig, double *alpha)
{
    long t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < (long)T; t++) {
        double sum_abs = 0.0;
        for (long c = 0; c < d; c++) {
            double v = load_elem(x, dtype, (size_t)t * d + c);
            if (sig)
                sig[(size_t)t * d + c] = sign_pm1(v);
            sum_abs += fabs(v);
        }
        alpha[t] = sum_abs / (double)d;
    }
}

/*
 * a1 + a2: sign bits and per-token scale.
 * bits[t*W + w], W = ceil(d/32): bit (c % 32) of word (c / 32) is 1 exactly
 * when sigma(x[t, c]) = +1. Bits for channels c >= d are 0. Built one bit at a
 * time with shifts from the +-1 value.
 */
int oracle_pack(const void *x, int dtype, long B, long H, long N, long d,
                uint32_t *bits, double *alpha)
{
    if (!x || !bits || !alpha || d < 1 || B < 0 || H < 0 || N < 0)
        return 1;
    const long W = (d + 31) / 32;
    const size_t T = (size_t)B * H * N;
    signs_and_scales(x, dtype, T, d, NULL, alpha);
    long t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < (long)T; t++) {
        for (long w = 0; w < W; w++)
            bits[(size_t)t * W + w] = 0u;
        for (long c = 0; c < d; c++) {
            double s = sign_pm1(load_elem(x, dtype, (size_t)t * d + c));
            if (s > 0.0)
                bits[(size_t)t * W + c / 32] |= (uint32_t)1u << (c % 32);
        }
    }
    return 0;
}

/* Shared preparation for the row functions below: signs and scales of Q and K. */
typedef struct {
    long B, H, N, d;
    double *sq, *sk; /* [B*H*N*d] +-1 */
    double *aq, *ak; /* [B*H*N]      */
} prep_t;

static int prep_init(prep_t *p, const void *q, const void *k, int qk_dtype,
                     long B, long H, long N, long d)
{
    size_t T = (size_t)B * H * N;
    p->B = B; p->H = H; p->N = N; p->d = d;
    p->sq = (double *)malloc(sizeof(double) * (T * d + 1));
    p->sk = (double *)malloc(sizeof(double) * (T * d + 1));
    p->aq = (double *)malloc(sizeof(double) * (T + 1));
    p->ak = (double *)malloc(sizeof(double) * (T + 1));
    if (!p->sq || !p->sk || !p->aq || !p->ak)
        return 1;
    signs_and_scales(q, qk_dtype, T, d, p->sq, p->aq);
    signs_and_scales(k, qk_dtype, T, d, p->sk, p->ak);
    return 0;
}

static void prep_free(prep_t *p)
{
    free(p->sq); free(p->sk); free(p->aq); free(p->ak);
}

/* Step 3 for one pair: explicit +-1 dot product over the d real channels. */
static double score_pm1(const prep_t *p, size_t qtok, size_t ktok)
{
    double s = 0.0;
    for (long c = 0; c < p->d; c++)
        s += p->sq[qtok * p->d + c] * p->sk[ktok * p->d + c];
    return s;
}

static int check_rows(long nrows, const int64_t *rows, long B, long H, long N)
{
    for (long r = 0; r < nrows; r++)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * H * N)
            return 1;
    return 0;
}

/*
 * a3: integer scores for selected query rows. rows[r] = (b*H + h)*N + i.
 * S_rows[r*N + j] = S_ij as int32 (each value is an exact integer in [-d, d]).
 */
int oracle_scores_rows(const void *q, const void *k, int qk_dtype,
                       long B, long H, long N, long d,
                       long nrows, const int64_t *rows, int32_t *S_rows)
{
    if (!q || !k || !rows || !S_rows || d < 1 || N < 1)
        return 1;
    if (check_rows(nrows, rows, B, H, N))
        return 2;
    prep_t p;
    if (prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        prep_free(&p);
        return 3;
    }
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; r++) {
        size_t qtok = (size_t)rows[r];
        size_t bh = qtok / (size_t)N;
        for (long j = 0; j < N; j++) {
            double s = score_pm1(&p, qtok, bh * (size_t)N + (size_t)j);
            S_rows[(size_t)r * N + j] = (int32_t)s;
        }
    }
    prep_free(&p);
    return 0;
}

/* Steps 3-5 up to the normalisation: P[j] = exp(logit_j - max_j logit_j). */
static void expdiff_row(const prep_t *p, size_t qtok, const uint16_t *bias,
                        double softmax_scale, double *P)
{
    const long N = p->N, H = p->H;
    size_t bh = qtok / (size_t)N;
    long i = (long)(qtok % (size_t)N);
    long h = (long)(bh % (size_t)H);
    double aq = p->aq[qtok];
    double m = -INFINITY;
    for (long j = 0; j < N; j++) {
        size_t ktok = bh * (size_t)N + (size_t)j;
        double s = score_pm1(p, qtok, ktok);
        double logit = softmax_scale * aq * p->ak[ktok] * s;
        if (bias)
            logit += load_elem(bias, ORACLE_BF16, ((size_t)h * N + i) * N + j);
        P[j] = logit;
        if (logit > m)
            m = logit;
    }
    for (long j = 0; j < N; j++)
        P[j] = exp(P[j] - m);
}

/* Steps 3-5 for one query row: attention probabilities P[j], j < N. */
static void probs_row(const prep_t *p, size_t qtok, const uint16_t *bias,
                      double softmax_scale, double *P)
{
    expdiff_row(p, qtok, bias, softmax_scale, P);
    double z = 0.0;
    for (long j = 0; j < p->N; j++)
        z += P[j];
    for (long j = 0; j < p->N; j++)
        P[j] /= z;
}

/*
 * a5: softmax probabilities for selected rows: P_rows[r*N + j] (fp64).
 * bias: bf16 [H, N, N] or NULL.
 */
int oracle_probs_rows(const void *q, const void *k, int qk_dtype,
                      const uint16_t *bias, double softmax_scale,
                      long B, long H, long N, long d,
                      long nrows, const int64_t *rows, double *P_rows)
{
    if (!q || !k || !rows || !P_rows || d < 1 || N < 1)
        return 1;
    if (check_rows(nrows, rows, B, H, N))
        return 2;
    prep_t p;
    if (prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        prep_free(&p);
        return 3;
    }
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; r++)
        probs_row(&p, (size_t)rows[r], bias, softmax_scale, P_rows + (size_t)r * N);
    prep_free(&p);
    return 0;
}

/*
 * Steps 1-6: attention output for selected rows, O_rows[r*d + c] (fp64,
 * unrounded). V is bf16 [B, H, N, d]; bias is bf16 [H, N, N] or NULL.
 */
int oracle_forward_rows(const void *q, const void *k, int qk_dtype,
                        const uint16_t *bias, const uint16_t *v,
                        double softmax_scale, long B, long H, long N, long d,
                        long nrows, const int64_t *rows, double *O_rows)
{
    if (!q || !k || !v || !rows || !O_rows || d < 1 || N < 1)
        return 1;
    if (check_rows(nrows, rows, B, H, N))
        return 2;
    prep_t p;
    if (prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        prep_free(&p);
        return 3;
    }
    int err = 0;
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; r++) {
        double *P = (double *)malloc(sizeof(double) * (size_t)N);
        if (!P) {
#pragma omp atomic write
            err = 3;
            continue;
        }
        size_t qtok = (size_t)rows[r];
        size_t bh = qtok / (size_t)N;
        probs_row(&p, qtok, bias, softmax_scale, P);
        for (long c = 0; c < d; c++) {
            double o = 0.0;
            for (long j = 0; j < N; j++)
                o += P[j] * load_elem(v, ORACLE_BF16, (bh * (size_t)N + (size_t)j) * d + c);
            O_rows[(size_t)r * d + c] = o;
        }
        free(P);
    }
    prep_free(&p);
    return err;
}

/* All rows: O[B, H, N, d] in fp64. */
int oracle_forward(const void *q, const void *k, int qk_dtype,
                   const uint16_t *bias, const uint16_t *v, double softmax_scale,
                   long B, long H, long N, long d, double *O)
{
    size_t T = (size_t)B * H * N;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (T + 1));
    if (!rows)
        return 3;
    for (size_t t = 0; t < T; t++)
        rows[t] = (int64_t)t;
    int rc = oracle_forward_rows(q, k, qk_dtype, bias, v, softmax_scale,
                                 B, H, N, d, (long)T, rows, O);
    free(rows);
    return rc;
}

/*
 * O rows as oracle_forward_rows, plus the spread E_rows[r*d + c] =
 * sum_j P_ij * |V_jc - O_ic| of each output element (fp64). O comes from
 * oracle_forward_rows; the probabilities are evaluated a second time for E.
 */
int oracle_forward_spread_rows(const void *q, const void *k, int qk_dtype,
                               const uint16_t *bias, const uint16_t *v,
                               double softmax_scale, long B, long H, long N, long d,
                               long nrows, const int64_t *rows, double *O_rows, double *E_rows)
{
    if (!E_rows)
        return 1;
    int rc = oracle_forward_rows(q, k, qk_dtype, bias, v, softmax_scale, B, H, N, d, nrows, rows, O_rows);
    if (rc)
        return rc;
    prep_t p;
    if (prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        prep_free(&p);
        return 3;
    }
    int err = 0;
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; r++) {
        double *P = (double *)malloc(sizeof(double) * (size_t)N);
        if (!P) {
#pragma omp atomic write
            err = 3;
            continue;
        }
        size_t qtok = (size_t)rows[r];
        size_t vtok0 = qtok / (size_t)N * (size_t)N;  /* key 0 of this (b, h) */
        probs_row(&p, qtok, bias, softmax_scale, P);
        for (long c = 0; c < d; c++) {
            const double oc = O_rows[(size_t)r * d + c];
            double e = 0.0;
            for (long j = 0; j < N; j++)
                e += P[j] * fabs(load_elem(v, ORACLE_BF16, (vtok0 + (size_t)j) * d + c) - oc);
            E_rows[(size_t)r * d + c] = e;
        }
        free(P);
    }
    prep_free(&p);
    return err;
}

/* All rows: O and E [B, H, N, d] in fp64. */
int oracle_forward_spread(const void *q, const void *k, int qk_dtype,
                          const uint16_t *bias, const uint16_t *v, double softmax_scale,
                          long B, long H, long N, long d, double *O, double *E)
{
    size_t T = (size_t)B * H * N;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (T + 1));
    if (!rows)
        return 3;
    for (size_t t = 0; t < T; t++)
        rows[t] = (int64_t)t;
    int rc = oracle_forward_spread_rows(q, k, qk_dtype, bias, v, softmax_scale,
                                        B, H, N, d, (long)T, rows, O, E);
    free(rows);
    return rc;
}

/*
 * Step 7: per-channel 8-bit code of V (bf16 [B, H, N, d]): vq int8 [B, H, N, d]
 * and s fp32 [B, H, d], in fp32 arithmetic.
 */
int oracle_quantize_v(const uint16_t *v, long B, long H, long N, long d, int8_t *vq, float *s)
{
    if (!v || !vq || !s || d < 1 || N < 1)
        return 1;
    long bh;
#pragma omp parallel for schedule(static)
    for (bh = 0; bh < B * H; bh++) {
        for (long c = 0; c < d; c++) {
            float mx = 0.0f;
            for (long j = 0; j < N; j++) {
                float a = fabsf((float)load_elem(v, ORACLE_BF16, ((size_t)bh * N + j) * d + c));
                if (a > mx)
                    mx = a;
            }
            const float sc = mx / 127.0f;
            s[(size_t)bh * d + c] = sc;
            for (long j = 0; j < N; j++) {
                const size_t idx = ((size_t)bh * N + j) * d + c;
                float q = 0.0f;
                if (sc > 0.0f) {
                    q = nearbyintf((float)load_elem(v, ORACLE_BF16, idx) / sc);
                    if (q > 127.0f)
                        q = 127.0f;
                    if (q < -127.0f)
                        q = -127.0f;
                }
                vq[idx] = (int8_t)q;
            }
        }
    }
    return 0;
}

/*
 * Steps 1-5 and 7-9: the 8-bit P.V forward for selected rows, O_rows[r*d + c]
 * (fp64, unrounded). V is bf16 [B, H, N, d]; bias is bf16 [H, N, N] or NULL.
 */
int oracle_forward_int8_rows(const void *q, const void *k, int qk_dtype,
                             const uint16_t *bias, const uint16_t *v,
                             double softmax_scale, long B, long H, long N, long d,
                             long nrows, const int64_t *rows, double *O_rows)
{
    if (!q || !k || !v || !rows || !O_rows || d < 1 || N < 1)
        return 1;
    if (check_rows(nrows, rows, B, H, N))
        return 2;
    int8_t *vq = (int8_t *)malloc((size_t)B * H * N * d);
    float *s = (float *)malloc(sizeof(float) * (size_t)B * H * d);
    prep_t p;
    if (!vq || !s || prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        free(vq);
        free(s);
        if (vq && s)
            prep_free(&p);
        return 3;
    }
    oracle_quantize_v(v, B, H, N, d, vq, s);
    int err = 0;
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; r++) {
        double *U = (double *)malloc(sizeof(double) * (size_t)N);
        if (!U) {
#pragma omp atomic write
            err = 3;
            continue;
        }
        size_t qtok = (size_t)rows[r];
        size_t bh = qtok / (size_t)N;
        expdiff_row(&p, qtok, bias, softmax_scale, U);
        double usum = 0.0;
        for (long j = 0; j < N; j++) {
            U[j] = nearbyint(255.0 * U[j]);
            usum += U[j];
        }
        for (long c = 0; c < d; c++) {
            double acc = 0.0;
            for (long j = 0; j < N; j++)
                acc += U[j] * (double)vq[(bh * (size_t)N + (size_t)j) * d + c];
            O_rows[(size_t)r * d + c] = (double)s[bh * (size_t)d + c] * acc / usum;
        }
        free(U);
    }
    prep_free(&p);
    free(vq);
    free(s);
    return err;
}

/* All rows of the 8-bit P.V forward: O [B, H, N, d] in fp64. */
int oracle_forward_int8(const void *q, const void *k, int qk_dtype,
                        const uint16_t *bias, const uint16_t *v, double softmax_scale,
                        long B, long H, long N, long d, double *O)
{
    size_t T = (size_t)B * H * N;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (T + 1));
    if (!rows)
        return 3;
    for (size_t t = 0; t < T; t++)
        rows[t] = (int64_t)t;
    int rc = oracle_forward_int8_rows(q, k, qk_dtype, bias, v, softmax_scale, B, H, N, d, (long)T, rows, O);
    free(rows);
    return rc;
}

/* Step 10: the dense bias [H, N, N] (bf16 bits) of a relative-position table. */
int oracle_expand_relpos_bias(const uint16_t *table, long H, long gh, long gw, long n_cls, uint16_t *bias)
{
    if (!table || !bias || H < 1 || gh < 1 || gw < 1 || n_cls < 0 || n_cls > 1)
        return 1;
    const long N = n_cls + gh * gw;
    const long R0 = (2 * gh - 1) * (2 * gw - 1);
    const long R = R0 + 3 * n_cls;
    for (long h = 0; h < H; h++) {
        for (long i = 0; i < N; i++) {
            uint16_t *brow = bias + ((size_t)h * N + (size_t)i) * (size_t)N;
            for (long j = 0; j < N; j++) {
                long idx;
                if (i < n_cls && j < n_cls)
                    idx = R0 + 2;
                else if (i < n_cls)
                    idx = R0;
                else if (j < n_cls)
                    idx = R0 + 1;
                else {
                    const long pi = i - n_cls, pj = j - n_cls;
                    const long dy = pi / gw - pj / gw, dx = pi % gw - pj % gw;
                    idx = (dy + gh - 1) * (2 * gw - 1) + (dx + gw - 1);
                }
                brow[j] = table[(size_t)h * R + idx];
            }
        }
    }
    return 0;
}

/*
 * Steps 11-15: gradients of the forward for an upstream gradient dO (bf16
 * [B, H, N, d]), all fp64: dV, ds, dt [B, H, N, d] and, when dbias is not
 * NULL, dbias [H, N, N] summed over b. bias is bf16 [H, N, N] or NULL (zero).
 * Every (b, h) is computed with its full N x N matrices P and dlogit; the
 * batch entries of one head run in order, so dbias sums them in order b.
 */
int oracle_backward(const void *q, const void *k, int qk_dtype, const uint16_t *bias,
                    const uint16_t *v, const uint16_t *dO, double softmax_scale,
                    long B, long H, long N, long d,
                    double *dV, double *ds, double *dt, double *dbias)
{
    if (!q || !k || !v || !dO || !dV || !ds || !dt || d < 1 || N < 1 || B < 1 || H < 1)
        return 1;
    prep_t p;
    if (prep_init(&p, q, k, qk_dtype, B, H, N, d)) {
        prep_free(&p);
        return 3;
    }
    int err = 0;
    long h;
#pragma omp parallel for schedule(dynamic, 1)
    for (h = 0; h < H; h++) {
        double *P = (double *)malloc(sizeof(double) * (size_t)N * N);
        double *dL = (double *)malloc(sizeof(double) * (size_t)N * N);
        if (!P || !dL) {
            free(P); free(dL);
#pragma omp atomic write
            err = 4;
            continue;
        }
        if (dbias)
            for (size_t e = 0; e < (size_t)N * N; e++)
                dbias[(size_t)h * N * N + e] = 0.0;
        for (long b = 0; b < B; b++) {
            const size_t tok0 = ((size_t)b * H + (size_t)h) * (size_t)N; /* token of (b, h, 0) */
            /* steps 3-5: the probabilities of every row */
            for (long i = 0; i < N; i++)
                probs_row(&p, tok0 + (size_t)i, bias, softmax_scale, P + (size_t)i * N);
            /* steps 12-13 */
            for (long i = 0; i < N; i++) {
                double Di = 0.0;
                for (long j = 0; j < N; j++) {
                    double dP = 0.0;
                    for (long c = 0; c < d; c++)
                        dP += load_elem(dO, ORACLE_BF16, (tok0 + i) * d + c) *
                              load_elem(v, ORACLE_BF16, (tok0 + j) * d + c);
                    dL[(size_t)i * N + j] = dP;
                    Di += P[(size_t)i * N + j] * dP;
                }
                for (long j = 0; j < N; j++)
                    dL[(size_t)i * N + j] = P[(size_t)i * N + j] * (dL[(size_t)i * N + j] - Di);
            }
            /* step 11 */
            for (long j = 0; j < N; j++)
                for (long c = 0; c < d; c++) {
                    double acc = 0.0;
                    for (long i = 0; i < N; i++)
                        acc += P[(size_t)i * N + j] * load_elem(dO, ORACLE_BF16, (tok0 + i) * d + c);
                    dV[(tok0 + j) * d + c] = acc;
                }
            /* step 14: t_j = alpha_k_j sigma(k_j), s_i = alpha_q_i sigma(q_i) */
            for (long i = 0; i < N; i++)
                for (long c = 0; c < d; c++) {
                    double acc = 0.0;
                    for (long j = 0; j < N; j++)
                        acc += dL[(size_t)i * N + j] * p.ak[tok0 + j] * p.sk[(tok0 + j) * d + c];
                    ds[(tok0 + i) * d + c] = softmax_scale * acc;
                }
            for (long j = 0; j < N; j++)
                for (long c = 0; c < d; c++) {
                    double acc = 0.0;
                    for (long i = 0; i < N; i++)
                        acc += dL[(size_t)i * N + j] * p.aq[tok0 + i] * p.sq[(tok0 + i) * d + c];
                    dt[(tok0 + j) * d + c] = softmax_scale * acc;
                }
            /* step 15 */
            if (dbias)
                for (size_t e = 0; e < (size_t)N * N; e++)
                    dbias[(size_t)h * N * N + e] += dL[e];
        }
        free(P);
        free(dL);
    }
    prep_free(&p);
    return err;
}
