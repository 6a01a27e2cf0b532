/*
 * streamkl_oracle.c -- plain fp64 CPU oracle for the StreamKL attention KL divergence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (per batch b, query head h, query row i):
 *   s_t[j] = scale * <Q_t[b,h,i,:], K_t[b,hk,j,:]>     t in {1,2}, hk = h / (Hq/Hkv)
 *   valid keys: j < NK, and j <= i when causal
 *   P_t = softmax over the valid keys of s_t
 *   KL_i = sum_j P1[j] * (log P1[j] - log P2[j])
 * This is the row-wise attention KL of "StreamKL: Fast and Memory-Efficient KL
 * Divergence for Boosting Attention Distillation" (abstract), and of the StreamKL
 * technical summary (gist.science, Portuguese), section "Definição do Problema".
 * Grouped heads follow the GQA definition of the KV-cache lecture notes (hackmd,
 * "3. 架構層級的記憶體妥協：從 MHA、MQA 到 GQA").
 *
 * The oracle is the definition written out, two passes per row, in double:
 *   LSE_t = M_t + log sum_j exp(s_t[j] - M_t),  M_t = max_j s_t[j]
 *   KL    = sum_j exp(s1[j]-LSE1) * ((s1[j]-LSE1) - (s2[j]-LSE2))
 * Using log-probabilities through logit differences and the LSEs, never log(P), is the
 * stable form the summary asks for ("3. Otimizações de Kernel de GPU", "Estabilidade
 * Numérica").
 *
 * A second forward, oracle_fwd_streaming, follows the pages' online formulation step by
 * step (summary, "1. Formulação Online (Passagem Forward)": five running scalars m1, l1,
 * m2, l2, acc per row and L = acc/l1 + LSE2 - LSE1), with the running sums multiplied by
 * exp(m_old - m_new) whenever a maximum grows (the correction of the FlashAttention
 * lecture notes, hackmd, "4. Flash Attention 的核心數學重構：動態修正與單趟掃描").
 * Tests compare the two; they must agree to rounding.
 *
 * Backward (summary, "2. Estratégia de Recomputação (Passagem Backward)"): the gradient
 * of sum_i g_i * KL_i with one distribution held fixed.  With d log p_k / d s_j =
 * delta_kj - p_j:
 *   setting 1 (P1 fixed, gradients of Q2, K2):   dS2[i,j] = g_i * (P2[i,j] - P1[i,j])
 *   setting 2 (P2 fixed, gradients of Q1, K1):   dS1[i,j] = g_i * P1[i,j] * (r_ij - KL_i),
 *                                                r_ij = (s1-LSE1) - (s2-LSE2)
 *   dQ_t[i] = scale * sum_j dS_t[i,j] * K_t[j]
 *   dK_t[j] = scale * sum over (heads of the KV group, rows i) of dS_t[i,j] * Q_t[i]
 * With K1 and K2 the same tensor, the fixed distribution is detached as a whole, so the
 * returned dK is the gradient through the free distribution only.
 *
 * All arrays are dense row-major: Q [B,Hq,NQ,d], K [B,Hkv,NK,d], per-row [B,Hq,NQ].
 * Functions return 0 on success, -1 on a bad argument, -2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, NQ, NK, d, causal;
    double scale;
} shape_t;

static int shape_ok(const shape_t* s) {
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->NQ < 1 || s->NK < 1 || s->d < 1) return 0;
    if (s->Hq % s->Hkv != 0) return 0;
    if (s->causal && s->NQ != s->NK) return 0;
    return 1;
}

static const double* q_row(const double* Q, const shape_t* s, int b, int h, int i) {
    return Q + (((size_t)b * s->Hq + h) * s->NQ + i) * (size_t)s->d;
}
static const double* k_base(const double* K, const shape_t* s, int b, int hk) {
    return K + ((size_t)b * s->Hkv + hk) * (size_t)s->NK * s->d;
}
static int n_valid(const shape_t* s, int i) {
    if (s->causal && i + 1 < s->NK) return i + 1;
    return s->NK;
}

/* s[j] = scale * <q, K[j]> for the first n keys. */
static void scores(const double* q, const double* K, int n, int d, double scale, double* out) {
    for (int j = 0; j < n; ++j) {
        const double* k = K + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[c] * k[c];
        out[j] = scale * acc;
    }
}

static double log_sum_exp(const double* s, int n) {
    double M = -INFINITY;
    for (int j = 0; j < n; ++j) if (s[j] > M) M = s[j];
    if (M == -INFINITY) return -INFINITY;
    double sum = 0.0;
    for (int j = 0; j < n; ++j) sum += exp(s[j] - M);
    return M + log(sum);
}

/* Two-pass definition for one row: fills s1, s2 (length n) and returns KL, LSE1, LSE2. */
static void row_forward(const double* q1, const double* K1, const double* q2, const double* K2,
                        int n, int d, double scale, double* s1, double* s2,
                        double* kl, double* lse1, double* lse2) {
    scores(q1, K1, n, d, scale, s1);
    scores(q2, K2, n, d, scale, s2);
    double L1 = log_sum_exp(s1, n);
    double L2 = log_sum_exp(s2, n);
    double acc = 0.0;
    for (int j = 0; j < n; ++j) {
        double lp1 = s1[j] - L1;
        double lp2 = s2[j] - L2;
        acc += exp(lp1) * (lp1 - lp2);
    }
    *kl = acc;
    *lse1 = L1;
    *lse2 = L2;
}

/* Forward for a list of flat row indices r in [0, B*Hq*NQ). */
int oracle_fwd_rows(const double* q1, const double* k1, const double* q2, const double* k2,
                    int B, int Hq, int Hkv, int NQ, int NK, int d, double scale, int causal,
                    const int64_t* rows, int64_t nrows,
                    double* kl, double* lse1, double* lse2) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || nrows < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * NQ;
    for (int64_t t = 0; t < nrows; ++t) if (rows[t] < 0 || rows[t] >= total) return -1;
    int fail = 0;
#pragma omp parallel
    {
        double* s1 = (double*)malloc(sizeof(double) * (size_t)NK);
        double* s2 = (double*)malloc(sizeof(double) * (size_t)NK);
        if (!s1 || !s2) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < nrows; ++t) {
                int64_t r = rows[t];
                int i = (int)(r % NQ);
                int h = (int)((r / NQ) % Hq);
                int b = (int)(r / ((int64_t)NQ * Hq));
                int hk = h / group;
                row_forward(q_row(q1, &s, b, h, i), k_base(k1, &s, b, hk),
                            q_row(q2, &s, b, h, i), k_base(k2, &s, b, hk),
                            n_valid(&s, i), d, scale, s1, s2, &kl[t], &lse1[t], &lse2[t]);
            }
        }
        free(s1);
        free(s2);
    }
    return fail ? -2 : 0;
}

/* Forward for every row; outputs [B,Hq,NQ]. */
int oracle_fwd(const double* q1, const double* k1, const double* q2, const double* k2,
               int B, int Hq, int Hkv, int NQ, int NK, int d, double scale, int causal,
               double* kl, double* lse1, double* lse2) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s)) return -1;
    int64_t total = (int64_t)B * Hq * NQ;
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)total);
    if (!rows) return -2;
    for (int64_t r = 0; r < total; ++r) rows[r] = r;
    int rc = oracle_fwd_rows(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, rows, total,
                             kl, lse1, lse2);
    free(rows);
    return rc;
}

/*
 * The pages' online formulation, run literally: keys are visited in tiles of `tile` keys;
 * per row the five scalars (m1, l1, m2, l2, acc) are updated once per tile, the old sums
 * rescaled by exp(m_old - m_new) when a maximum grows, and the row's value is
 * L = acc/l1 + LSE2 - LSE1 with LSE_t = m_t + log l_t.
 */
int oracle_fwd_streaming(const double* q1, const double* k1, const double* q2, const double* k2,
                         int B, int Hq, int Hkv, int NQ, int NK, int d, double scale, int causal,
                         int tile, double* kl, double* lse1, double* lse2) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || tile < 1) return -1;
    const int group = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * NQ;
    int fail = 0;
#pragma omp parallel
    {
        double* s1 = (double*)malloc(sizeof(double) * (size_t)tile);
        double* s2 = (double*)malloc(sizeof(double) * (size_t)tile);
        if (!s1 || !s2) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < total; ++r) {
                int i = (int)(r % NQ);
                int h = (int)((r / NQ) % Hq);
                int b = (int)(r / ((int64_t)NQ * Hq));
                int hk = h / group;
                const double* q1r = q_row(q1, &s, b, h, i);
                const double* q2r = q_row(q2, &s, b, h, i);
                const double* K1 = k_base(k1, &s, b, hk);
                const double* K2 = k_base(k2, &s, b, hk);
                int n = n_valid(&s, i);
                double m1 = -INFINITY, l1 = 0.0, m2 = -INFINITY, l2 = 0.0, acc = 0.0;
                for (int j0 = 0; j0 < n; j0 += tile) {
                    int w = n - j0 < tile ? n - j0 : tile;
                    scores(q1r, K1 + (size_t)j0 * d, w, d, scale, s1);
                    scores(q2r, K2 + (size_t)j0 * d, w, d, scale, s2);
                    double t1 = -INFINITY, t2 = -INFINITY;
                    for (int j = 0; j < w; ++j) {
                        if (s1[j] > t1) t1 = s1[j];
                        if (s2[j] > t2) t2 = s2[j];
                    }
                    double m1n = m1 > t1 ? m1 : t1;
                    double m2n = m2 > t2 ? m2 : t2;
                    double a1 = (m1 == -INFINITY) ? 0.0 : exp(m1 - m1n);
                    double a2 = (m2 == -INFINITY) ? 0.0 : exp(m2 - m2n);
                    l1 *= a1;
                    acc *= a1;
                    l2 *= a2;
                    for (int j = 0; j < w; ++j) {
                        double e1 = exp(s1[j] - m1n);
                        l1 += e1;
                        acc += e1 * (s1[j] - s2[j]);
                        l2 += exp(s2[j] - m2n);
                    }
                    m1 = m1n;
                    m2 = m2n;
                }
                double L1 = m1 + log(l1);
                double L2 = m2 + log(l2);
                kl[r] = acc / l1 + L2 - L1;
                lse1[r] = L1;
                lse2[r] = L2;
            }
        }
        free(s1);
        free(s2);
    }
    return fail ? -2 : 0;
}

/* dS for one row into ds[0..n): setting 1 or 2, from the row's scores and statistics. */
static void row_ds(int mode, const double* s1, const double* s2, int n, double L1, double L2,
                   double kl, double g, double* ds) {
    for (int j = 0; j < n; ++j) {
        double lp1 = s1[j] - L1;
        double lp2 = s2[j] - L2;
        double p1 = exp(lp1);
        if (mode == 1) {
            ds[j] = g * (exp(lp2) - p1);
        } else {
            ds[j] = g * p1 * ((lp1 - lp2) - kl);
        }
    }
}

/*
 * Full backward.  mode 1: outputs dq = dQ2 [B,Hq,NQ,d], dk = dK2 [B,Hkv,NK,d].
 * mode 2: dq = dQ1, dk = dK1.  g = dkl [B,Hq,NQ].  Row statistics (LSE, KL) are
 * recomputed here from the definition; nothing is taken from a caller.
 */
int oracle_bwd(int mode, const double* q1, const double* k1, const double* q2, const double* k2,
               const double* dkl, int B, int Hq, int Hkv, int NQ, int NK, int d, double scale,
               int causal, double* dq, double* dk) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || (mode != 1 && mode != 2)) return -1;
    const int group = Hq / Hkv;
    const double* Qf = (mode == 1) ? q2 : q1;   /* the free distribution's inputs */
    const double* Kf = (mode == 1) ? k2 : k1;
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * NK * d);
    int fail = 0;
    /* one task per (b, KV head): dK of that head is written by this task only */
#pragma omp parallel
    {
        double* s1 = (double*)malloc(sizeof(double) * (size_t)NK);
        double* s2 = (double*)malloc(sizeof(double) * (size_t)NK);
        double* ds = (double*)malloc(sizeof(double) * (size_t)NK);
        if (!s1 || !s2 || !ds) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int u = 0; u < B * Hkv; ++u) {
                int b = u / Hkv, hk = u % Hkv;
                const double* K1 = k_base(k1, &s, b, hk);
                const double* K2 = k_base(k2, &s, b, hk);
                const double* KF = k_base(Kf, &s, b, hk);
                double* dkh = dk + ((size_t)b * Hkv + hk) * (size_t)NK * d;
                for (int h = hk * group; h < (hk + 1) * group; ++h) {
                    for (int i = 0; i < NQ; ++i) {
                        int n = n_valid(&s, i);
                        double kl, L1, L2;
                        row_forward(q_row(q1, &s, b, h, i), K1, q_row(q2, &s, b, h, i), K2, n, d,
                                    scale, s1, s2, &kl, &L1, &L2);
                        double g = dkl[((size_t)b * Hq + h) * NQ + i];
                        row_ds(mode, s1, s2, n, L1, L2, kl, g, ds);
                        const double* qf = q_row(Qf, &s, b, h, i);
                        double* dqr = dq + (((size_t)b * Hq + h) * NQ + i) * (size_t)d;
                        for (int c = 0; c < d; ++c) dqr[c] = 0.0;
                        for (int j = 0; j < n; ++j) {
                            const double* kr = KF + (size_t)j * d;
                            double* dkr = dkh + (size_t)j * d;
                            double w = scale * ds[j];
                            for (int c = 0; c < d; ++c) {
                                dqr[c] += w * kr[c];
                                dkr[c] += w * qf[c];
                            }
                        }
                    }
                }
            }
        }
        free(s1);
        free(s2);
        free(ds);
    }
    return fail ? -2 : 0;
}

/*
 * dQ for a list of flat rows (each dQ row depends only on its own row): dq_rows [nrows, d].
 */
int oracle_bwd_dq_rows(int mode, const double* q1, const double* k1, const double* q2,
                       const double* k2, const double* dkl, int B, int Hq, int Hkv, int NQ, int NK,
                       int d, double scale, int causal, const int64_t* rows, int64_t nrows,
                       double* dq_rows) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || (mode != 1 && mode != 2) || nrows < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * NQ;
    for (int64_t t = 0; t < nrows; ++t) if (rows[t] < 0 || rows[t] >= total) return -1;
    const double* Qf = (mode == 1) ? q2 : q1;
    const double* Kf = (mode == 1) ? k2 : k1;
    (void)Qf;
    int fail = 0;
#pragma omp parallel
    {
        double* s1 = (double*)malloc(sizeof(double) * (size_t)NK);
        double* s2 = (double*)malloc(sizeof(double) * (size_t)NK);
        double* ds = (double*)malloc(sizeof(double) * (size_t)NK);
        if (!s1 || !s2 || !ds) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < nrows; ++t) {
                int64_t r = rows[t];
                int i = (int)(r % NQ);
                int h = (int)((r / NQ) % Hq);
                int b = (int)(r / ((int64_t)NQ * Hq));
                int hk = h / group;
                int n = n_valid(&s, i);
                double kl, L1, L2;
                row_forward(q_row(q1, &s, b, h, i), k_base(k1, &s, b, hk), q_row(q2, &s, b, h, i),
                            k_base(k2, &s, b, hk), n, d, scale, s1, s2, &kl, &L1, &L2);
                row_ds(mode, s1, s2, n, L1, L2, kl, dkl[r], ds);
                const double* KF = k_base(Kf, &s, b, hk);
                double* out = dq_rows + (size_t)t * d;
                for (int c = 0; c < d; ++c) out[c] = 0.0;
                for (int j = 0; j < n; ++j) {
                    double w = scale * ds[j];
                    const double* kr = KF + (size_t)j * d;
                    for (int c = 0; c < d; ++c) out[c] += w * kr[c];
                }
            }
        }
        free(s1);
        free(s2);
        free(ds);
    }
    return fail ? -2 : 0;
}

/*
 * dK for a list of (b, KV head, key) triples given as flat key indices into [B*Hkv*NK]:
 * dk_keys [nkeys, d].  Every query row of the KV group that sees the key contributes, so
 * the row statistics of the whole group are recomputed here (one forward per row).
 */
int oracle_bwd_dk_keys(int mode, const double* q1, const double* k1, const double* q2,
                       const double* k2, const double* dkl, int B, int Hq, int Hkv, int NQ, int NK,
                       int d, double scale, int causal, const int64_t* keys, int64_t nkeys,
                       double* dk_keys) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || (mode != 1 && mode != 2) || nkeys < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t totalk = (int64_t)B * Hkv * NK;
    for (int64_t t = 0; t < nkeys; ++t) if (keys[t] < 0 || keys[t] >= totalk) return -1;
    const double* Qf = (mode == 1) ? q2 : q1;
    memset(dk_keys, 0, sizeof(double) * (size_t)nkeys * d);
    /* row statistics for every row of every (b, KV head) that owns a requested key */
    const int64_t nrow_all = (int64_t)B * Hq * NQ;
    double* KL = (double*)malloc(sizeof(double) * (size_t)nrow_all);
    double* L1 = (double*)malloc(sizeof(double) * (size_t)nrow_all);
    double* L2 = (double*)malloc(sizeof(double) * (size_t)nrow_all);
    char* need = (char*)calloc((size_t)B * Hkv, 1);
    if (!KL || !L1 || !L2 || !need) {
        free(KL); free(L1); free(L2); free(need);
        return -2;
    }
    for (int64_t t = 0; t < nkeys; ++t) need[keys[t] / NK] = 1;
    int64_t nsel = 0;
    for (int u = 0; u < B * Hkv; ++u) if (need[u]) nsel += (int64_t)group * NQ;
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nsel > 0 ? nsel : 1));
    double *kl_s = (double*)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
    double *l1_s = (double*)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
    double *l2_s = (double*)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
    int rc = 0;
    if (!rows || !kl_s || !l1_s || !l2_s) rc = -2;
    if (rc == 0) {
        int64_t p = 0;
        for (int u = 0; u < B * Hkv; ++u) {
            if (!need[u]) continue;
            int b = u / Hkv, hk = u % Hkv;
            for (int h = hk * group; h < (hk + 1) * group; ++h)
                for (int i = 0; i < NQ; ++i) rows[p++] = ((int64_t)b * Hq + h) * NQ + i;
        }
        rc = oracle_fwd_rows(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, rows, nsel,
                             kl_s, l1_s, l2_s);
        for (int64_t t = 0; rc == 0 && t < nsel; ++t) {
            KL[rows[t]] = kl_s[t];
            L1[rows[t]] = l1_s[t];
            L2[rows[t]] = l2_s[t];
        }
    }
    if (rc == 0) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t t = 0; t < nkeys; ++t) {
            int64_t kk = keys[t];
            int j = (int)(kk % NK);
            int hk = (int)((kk / NK) % Hkv);
            int b = (int)(kk / ((int64_t)NK * Hkv));
            const double* k1r = k_base(k1, &s, b, hk) + (size_t)j * d;
            const double* k2r = k_base(k2, &s, b, hk) + (size_t)j * d;
            double* out = dk_keys + (size_t)t * d;
            for (int h = hk * group; h < (hk + 1) * group; ++h) {
                for (int i = (causal ? j : 0); i < NQ; ++i) {
                    int64_t r = ((int64_t)b * Hq + h) * NQ + i;
                    double a1 = 0.0, a2 = 0.0;
                    const double* q1r = q_row(q1, &s, b, h, i);
                    const double* q2r = q_row(q2, &s, b, h, i);
                    for (int c = 0; c < d; ++c) {
                        a1 += q1r[c] * k1r[c];
                        a2 += q2r[c] * k2r[c];
                    }
                    double ds1;
                    double lp1 = scale * a1 - L1[r];
                    double lp2 = scale * a2 - L2[r];
                    double p1 = exp(lp1);
                    if (mode == 1) ds1 = dkl[r] * (exp(lp2) - p1);
                    else ds1 = dkl[r] * p1 * ((lp1 - lp2) - KL[r]);
                    const double* qf = q_row(Qf, &s, b, h, i);
                    double w = scale * ds1;
                    for (int c = 0; c < d; ++c) out[c] += w * qf[c];
                }
            }
        }
    }
    free(rows); free(kl_s); free(l1_s); free(l2_s);
    free(KL); free(L1); free(L2); free(need);
    return rc;
}

/*
 * dK for flat key indices like oracle_bwd_dk_keys, but with the row statistics (KL, LSE1,
 * LSE2 of every row, [B*Hq*NQ]) taken as inputs instead of recomputed.  For sizes where
 * recomputing every row's statistics is out of reach; the caller states where the
 * statistics came from.
 */
int oracle_bwd_dk_keys_stats(int mode, const double* q1, const double* k1, const double* q2,
                             const double* k2, const double* dkl, const double* KL,
                             const double* L1, const double* L2, int B, int Hq, int Hkv, int NQ,
                             int NK, int d, double scale, int causal, const int64_t* keys,
                             int64_t nkeys, double* dk_keys) {
    shape_t s = {B, Hq, Hkv, NQ, NK, d, causal, scale};
    if (!shape_ok(&s) || (mode != 1 && mode != 2) || nkeys < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t totalk = (int64_t)B * Hkv * NK;
    for (int64_t t = 0; t < nkeys; ++t) if (keys[t] < 0 || keys[t] >= totalk) return -1;
    const double* Qf = (mode == 1) ? q2 : q1;
    memset(dk_keys, 0, sizeof(double) * (size_t)nkeys * d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < nkeys; ++t) {
        int64_t kk = keys[t];
        int j = (int)(kk % NK);
        int hk = (int)((kk / NK) % Hkv);
        int b = (int)(kk / ((int64_t)NK * Hkv));
        const double* k1r = k_base(k1, &s, b, hk) + (size_t)j * d;
        const double* k2r = k_base(k2, &s, b, hk) + (size_t)j * d;
        double* out = dk_keys + (size_t)t * d;
        for (int h = hk * group; h < (hk + 1) * group; ++h) {
            for (int i = (causal ? j : 0); i < NQ; ++i) {
                int64_t r = ((int64_t)b * Hq + h) * NQ + i;
                const double* q1r = q_row(q1, &s, b, h, i);
                const double* q2r = q_row(q2, &s, b, h, i);
                double a1 = 0.0, a2 = 0.0;
                for (int c = 0; c < d; ++c) {
                    a1 += q1r[c] * k1r[c];
                    a2 += q2r[c] * k2r[c];
                }
                double lp1 = scale * a1 - L1[r];
                double lp2 = scale * a2 - L2[r];
                double p1 = exp(lp1);
                double ds = (mode == 1) ? dkl[r] * (exp(lp2) - p1)
                                        : dkl[r] * p1 * ((lp1 - lp2) - KL[r]);
                const double* qf = q_row(Qf, &s, b, h, i);
                double w = scale * ds;
                for (int c = 0; c < d; ++c) out[c] += w * qf[c];
            }
        }
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
