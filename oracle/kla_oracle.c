/*
 * Oracle for Kaczmarz Linear Attention (KLA) -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64, token-by-token evaluation of the recurrence.  Only the
 * test-suite, the smoke check and the CPU-baseline leg of the benchmark may
 * load this library; the product path never does.  It shares no code, header
 * or constant with the CUDA library.
 *
 * What it computes (h = S^T stored [dk][dv] per head):
 *
 *   beta_t = eta_t / (||k_t||_2^2 + eps)
 *       Kaczmarz Linear Attention (tomesphere summary of arXiv 2605.08587),
 *       Abstract: the key-norm-normalised step size.
 *   S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   alpha_t = exp(g_t)
 *       Gated DeltaNet recurrence ("Deep Dive into KDA", section 2.2), of which
 *       KLA is the one-scalar modification (same Abstract).  The page prints
 *       the erase factor on the left of S; with S mapping keys to values
 *       (S is dv x dk) only the right-hand placement type-checks, and for a
 *       scalar gate the two placements of alpha agree.
 *   o_t = S_t q_t   (the updated state is read)
 *
 * In h-form, per token:  r = h^T k;  u = beta (v - alpha r);
 *                        h = alpha h + k u^T;  o = h^T q.
 * which is the line above transposed: S^T = alpha (I - beta k k^T) S_{t-1}^T
 * + beta k v^T  and  alpha (I - beta k k^T) h + beta k v^T
 *  = alpha h + k (beta v - alpha beta k^T h)^T.
 *
 * Per-channel gate (KDA, "Deep Dive into KDA", section 2.3; the KLA Abstract
 * lists a preconditioned KDA among its variants):
 *   S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t v_t k_t^T,
 *   a_t = exp(g_t) with g_t one log-gate per key channel.
 * The page's orientation is garbled the same way as the GDN line; with S
 * mapping keys to values the diagonal acts on the key side, and the page's
 * order is kept: decay first, then the erase reads the decayed state.  In
 * h-form, per token:  h <- Diag(a) h  (row i scaled by a_i);  r = h^T k;
 *                     u = beta (v - r);  h <- h + k u^T;  o = h^T q.
 *
 * Gradients (reverse mode through the token loop of the GDN form, for a
 * loss L with dL/do = do and dL/dh_T = dhT; the pages print no backward
 * algorithm, so this is the chain rule applied to the lines above, each
 * step of it named where it is taken).  The states h_t are kept for every
 * token; walking t down from T - 1 with H = dL/dh_t:
 *   H += q_t do_t^T;  dq_t = h_t do_t                      (o_t = h_t^T q_t)
 *   du = H^T k_t;  dk_t += H u_t;  da = <H, h_{t-1}>;  H' = alpha H
 *                                                      (h_t = alpha h_{t-1} + k u^T)
 *   dv_t = beta du;  dbeta = du . (v - alpha r);  da -= beta du . r;
 *   dr = -alpha beta du                              (u = beta (v - alpha r))
 *   H' += k dr^T;  dk_t += h_{t-1} dr                (r = h_{t-1}^T k)
 *   dg_t = da alpha                                  (alpha = exp(g))
 * and H <- H'; dh0 = H at the end.  KLA adds the step size
 * beta = eta / (n2 + eps), n2 = ||k||^2: deta = dbeta / (n2 + eps) and
 * dk += -2 dbeta eta / (n2 + eps)^2 k.
 *
 * Layouts (row-major, contiguous):
 *   q, k : [B][T][H][dk]     v, o : [B][T][H][dv]
 *   g, eta, beta : [B][T][H]  (per-channel gate: g is [B][T][H][dk])
 *   h0, hT : [B][H][dk][dv]  (h0 may be NULL = zeros; hT may be NULL)
 * Heads (b, h) are independent; OpenMP runs them in parallel.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* beta_t = eta_t / (||k_t||^2 + eps), one value per (b, t, h). */
void kla_oracle_beta(const double *k, const double *eta, double eps,
                     double *beta, int B, int T, int H, int dk)
{
    long n = (long)B * T * H;
    for (long p = 0; p < n; ++p) {
        const double *kp = k + p * dk;
        double n2 = 0.0;
        for (int i = 0; i < dk; ++i) n2 += kp[i] * kp[i];
        beta[p] = eta[p] / (n2 + eps);
    }
}

/* The gated delta rule with beta supplied per token (GDN form). */
void kla_oracle_gated_delta(const double *q, const double *k, const double *v,
                            const double *g, const double *beta,
                            const double *h0, double *o, double *hT,
                            int B, int T, int H, int dk, int dv)
{
    int nheads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < nheads; ++bh) {
        int b = bh / H, hh = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (h0)
            memcpy(S, h0 + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = 0; t < T; ++t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *kt = k + tok * dk;
            const double *qt = q + tok * dk;
            const double *vt = v + tok * dv;
            double alpha = exp(g[tok]);
            double bt = beta[tok];
            /* r = h^T k  (= S_{t-1} k_t) */
            for (int j = 0; j < dv; ++j) r[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) r[j] += Si[j] * kt[i];
            }
            /* u = beta (v - alpha r) */
            for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - alpha * r[j]);
            /* h = alpha h + k u^T */
            for (int i = 0; i < dk; ++i) {
                double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) Si[j] = alpha * Si[j] + kt[i] * u[j];
            }
            /* o = h^T q with the updated state */
            double *ot = o + tok * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += Si[j] * qt[i];
            }
        }
        if (hT) memcpy(hT + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(r);
        free(u);
    }
}

/* KLA forward: beta from the key norm, then the gated delta rule. */
void kla_oracle_forward(const double *q, const double *k, const double *v,
                        const double *g, const double *eta, double eps,
                        const double *h0, double *o, double *hT,
                        int B, int T, int H, int dk, int dv)
{
    size_t n = (size_t)B * T * H;
    double *beta = (double *)malloc(sizeof(double) * (n ? n : 1));
    kla_oracle_beta(k, eta, eps, beta, B, T, H, dk);
    kla_oracle_gated_delta(q, k, v, g, beta, h0, o, hT, B, T, H, dk, dv);
    free(beta);
}

/* The delta rule with a per-channel gate (KDA form), beta given per token. */
void kla_oracle_kda(const double *q, const double *k, const double *v,
                    const double *g, const double *beta,
                    const double *h0, double *o, double *hT,
                    int B, int T, int H, int dk, int dv)
{
    int nheads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < nheads; ++bh) {
        int b = bh / H, hh = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (h0)
            memcpy(S, h0 + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = 0; t < T; ++t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *kt = k + tok * dk;
            const double *qt = q + tok * dk;
            const double *vt = v + tok * dv;
            const double *gt = g + tok * dk;
            double bt = beta[tok];
            /* Diag(a_t) S_{t-1}: row i of h (key channel i) times exp(g_i) */
            for (int i = 0; i < dk; ++i) {
                double a = exp(gt[i]);
                double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) Si[j] *= a;
            }
            /* u = beta (v - h^T k), from the decayed state */
            for (int j = 0; j < dv; ++j) u[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) u[j] += Si[j] * kt[i];
            }
            for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - u[j]);
            /* h += k u^T; o = h^T q with the updated state */
            for (int i = 0; i < dk; ++i) {
                double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) Si[j] += kt[i] * u[j];
            }
            double *ot = o + tok * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += Si[j] * qt[i];
            }
        }
        if (hT) memcpy(hT + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(u);
    }
}

/* Gradients of the GDN form (beta given) for dL/do = dout and dL/dh_T =
 * dhT (NULL = 0): writes dq, dk [B][T][H][dk], dv [B][T][H][dv],
 * dg, dbeta [B][T][H] and dh0 [B][H][dk][dv] (NULL = not returned). */
void kla_oracle_gated_delta_backward(const double *q, const double *k, const double *v,
                                     const double *g, const double *beta, const double *h0,
                                     const double *dout, const double *dhT,
                                     double *dq, double *dk, double *dv, double *dg,
                                     double *dbeta, double *dh0,
                                     int B, int T, int H, int dk_, int dv_)
{
    const int dK = dk_, dV = dv_;
    int nheads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < nheads; ++bh) {
        int b = bh / H, hh = bh % H;
        size_t SZ = (size_t)dK * dV;
        /* hs[t + 1] = h_t, hs[0] = h0 */
        double *hs = (double *)malloc(sizeof(double) * SZ * (size_t)(T + 1));
        double *Hm = (double *)malloc(sizeof(double) * SZ);
        double *Hn = (double *)malloc(sizeof(double) * SZ);
        double *r = (double *)malloc(sizeof(double) * (size_t)dV);
        double *u = (double *)malloc(sizeof(double) * (size_t)dV);
        double *du = (double *)malloc(sizeof(double) * (size_t)dV);
        double *dr = (double *)malloc(sizeof(double) * (size_t)dV);
        if (h0)
            memcpy(hs, h0 + (size_t)bh * SZ, sizeof(double) * SZ);
        else
            memset(hs, 0, sizeof(double) * SZ);
        /* forward, keeping every state */
        for (int t = 0; t < T; ++t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *kt = k + tok * dK, *vt = v + tok * dV;
            const double *hp = hs + (size_t)t * SZ;
            double *hc = hs + (size_t)(t + 1) * SZ;
            double alpha = exp(g[tok]), bt = beta[tok];
            for (int j = 0; j < dV; ++j) r[j] = 0.0;
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j) r[j] += hp[(size_t)i * dV + j] * kt[i];
            for (int j = 0; j < dV; ++j) u[j] = bt * (vt[j] - alpha * r[j]);
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j)
                    hc[(size_t)i * dV + j] = alpha * hp[(size_t)i * dV + j] + kt[i] * u[j];
        }
        /* reverse */
        if (dhT)
            memcpy(Hm, dhT + (size_t)bh * SZ, sizeof(double) * SZ);
        else
            memset(Hm, 0, sizeof(double) * SZ);
        for (int t = T - 1; t >= 0; --t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *qt = q + tok * dK, *kt = k + tok * dK, *vt = v + tok * dV;
            const double *dot = dout + tok * dV;
            const double *hp = hs + (size_t)t * SZ, *hc = hs + (size_t)(t + 1) * SZ;
            double *dqt = dq + tok * dK, *dkt = dk + tok * dK, *dvt = dv + tok * dV;
            double alpha = exp(g[tok]), bt = beta[tok];
            /* o_t = h_t^T q_t */
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dV; ++j) {
                    Hm[(size_t)i * dV + j] += qt[i] * dot[j];
                    acc += hc[(size_t)i * dV + j] * dot[j];
                }
                dqt[i] = acc;
            }
            /* recompute r, u of this step */
            for (int j = 0; j < dV; ++j) r[j] = 0.0;
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j) r[j] += hp[(size_t)i * dV + j] * kt[i];
            for (int j = 0; j < dV; ++j) u[j] = bt * (vt[j] - alpha * r[j]);
            /* h_t = alpha h_{t-1} + k u^T */
            double da = 0.0;
            for (int j = 0; j < dV; ++j) du[j] = 0.0;
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dV; ++j) {
                    du[j] += Hm[(size_t)i * dV + j] * kt[i];
                    acc += Hm[(size_t)i * dV + j] * u[j];
                    da += Hm[(size_t)i * dV + j] * hp[(size_t)i * dV + j];
                    Hn[(size_t)i * dV + j] = alpha * Hm[(size_t)i * dV + j];
                }
                dkt[i] = acc;
            }
            /* u = beta (v - alpha r) */
            double db = 0.0;
            for (int j = 0; j < dV; ++j) {
                dvt[j] = bt * du[j];
                db += du[j] * (vt[j] - alpha * r[j]);
                da -= bt * du[j] * r[j];
                dr[j] = -alpha * bt * du[j];
            }
            /* r = h_{t-1}^T k */
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dV; ++j) {
                    Hn[(size_t)i * dV + j] += kt[i] * dr[j];
                    acc += hp[(size_t)i * dV + j] * dr[j];
                }
                dkt[i] += acc;
            }
            dg[tok] = da * alpha;
            dbeta[tok] = db;
            double *tmp = Hm; Hm = Hn; Hn = tmp;
        }
        if (dh0) memcpy(dh0 + (size_t)bh * SZ, Hm, sizeof(double) * SZ);
        free(hs); free(Hm); free(Hn); free(r); free(u); free(du); free(dr);
    }
}

/* Gradients of the per-channel-gate form (beta given) for dL/do = dout and
 * dL/dh_T = dhT (NULL = 0): dq, dk, dg [B][T][H][dk], dv [B][T][H][dv],
 * dbeta [B][T][H], dh0 [B][H][dk][dv] (NULL = not returned).  Reverse mode
 * through the token loop of kla_oracle_kda, with H = dL/dh_t and
 * hd = Diag(a_t) h_{t-1} the decayed state:
 *   H += q_t do_t^T;  dq_t = h_t do_t                      (o_t = h_t^T q_t)
 *   du = H^T k;  dk_t += H u;  Hd = H                       (h_t = hd + k u^T)
 *   dv_t = beta du;  dbeta = du . (v - r);  dr = -beta du   (u = beta (v - r))
 *   Hd += k dr^T;  dk_t += hd dr                            (r = hd^T k)
 *   dg_{t,i} = sum_j Hd_ij hd_ij;  H' = Diag(a_t) Hd          (hd = Diag(a) h)
 */
void kla_oracle_kda_backward(const double *q, const double *k, const double *v,
                             const double *g, const double *beta, const double *h0,
                             const double *dout, const double *dhT, double *dq, double *dk,
                             double *dv, double *dg, double *dbeta, double *dh0, int B, int T,
                             int H, int dk_, int dv_)
{
    const int dK = dk_, dV = dv_;
    int nheads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < nheads; ++bh) {
        int b = bh / H, hh = bh % H;
        size_t SZ = (size_t)dK * dV;
        /* hs[t + 1] = h_t, hs[0] = h0 */
        double *hs = (double *)malloc(sizeof(double) * SZ * (size_t)(T + 1));
        double *Hm = (double *)malloc(sizeof(double) * SZ);
        double *hd = (double *)malloc(sizeof(double) * SZ);
        double *r = (double *)malloc(sizeof(double) * (size_t)dV);
        double *u = (double *)malloc(sizeof(double) * (size_t)dV);
        double *du = (double *)malloc(sizeof(double) * (size_t)dV);
        if (h0)
            memcpy(hs, h0 + (size_t)bh * SZ, sizeof(double) * SZ);
        else
            memset(hs, 0, sizeof(double) * SZ);
        /* forward, keeping every state (the steps of kla_oracle_kda) */
        for (int t = 0; t < T; ++t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *kt = k + tok * dK, *vt = v + tok * dV, *gt = g + tok * dK;
            const double *hp = hs + (size_t)t * SZ;
            double *hc = hs + (size_t)(t + 1) * SZ;
            for (int i = 0; i < dK; ++i) {
                double a = exp(gt[i]);
                for (int j = 0; j < dV; ++j) hc[(size_t)i * dV + j] = a * hp[(size_t)i * dV + j];
            }
            for (int j = 0; j < dV; ++j) r[j] = 0.0;
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j) r[j] += hc[(size_t)i * dV + j] * kt[i];
            for (int j = 0; j < dV; ++j) u[j] = beta[tok] * (vt[j] - r[j]);
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j) hc[(size_t)i * dV + j] += kt[i] * u[j];
        }
        /* reverse */
        if (dhT)
            memcpy(Hm, dhT + (size_t)bh * SZ, sizeof(double) * SZ);
        else
            memset(Hm, 0, sizeof(double) * SZ);
        for (int t = T - 1; t >= 0; --t) {
            size_t tok = ((size_t)b * T + t) * H + hh;
            const double *qt = q + tok * dK, *kt = k + tok * dK, *vt = v + tok * dV;
            const double *gt = g + tok * dK, *dot = dout + tok * dV;
            const double *hp = hs + (size_t)t * SZ, *hc = hs + (size_t)(t + 1) * SZ;
            double *dqt = dq + tok * dK, *dkt = dk + tok * dK, *dvt = dv + tok * dV;
            double *dgt = dg + tok * dK;
            double bt = beta[tok];
            /* o_t = h_t^T q_t */
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dV; ++j) {
                    Hm[(size_t)i * dV + j] += qt[i] * dot[j];
                    acc += hc[(size_t)i * dV + j] * dot[j];
                }
                dqt[i] = acc;
            }
            /* recompute hd = Diag(a) h_{t-1}, r, u of this step */
            for (int i = 0; i < dK; ++i) {
                double a = exp(gt[i]);
                for (int j = 0; j < dV; ++j) hd[(size_t)i * dV + j] = a * hp[(size_t)i * dV + j];
            }
            for (int j = 0; j < dV; ++j) r[j] = 0.0;
            for (int i = 0; i < dK; ++i)
                for (int j = 0; j < dV; ++j) r[j] += hd[(size_t)i * dV + j] * kt[i];
            for (int j = 0; j < dV; ++j) u[j] = bt * (vt[j] - r[j]);
            /* h_t = hd + k u^T */
            for (int j = 0; j < dV; ++j) du[j] = 0.0;
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dV; ++j) {
                    du[j] += Hm[(size_t)i * dV + j] * kt[i];
                    acc += Hm[(size_t)i * dV + j] * u[j];
                }
                dkt[i] = acc;
            }
            /* u = beta (v - r) */
            double db = 0.0;
            for (int j = 0; j < dV; ++j) {
                dvt[j] = bt * du[j];
                db += du[j] * (vt[j] - r[j]);
            }
            dbeta[tok] = db;
            /* r = hd^T k:  Hd = H + k dr^T,  dk += hd dr;  then hd = Diag(a) h */
            for (int i = 0; i < dK; ++i) {
                double acc = 0.0, ga = 0.0, a = exp(gt[i]);
                for (int j = 0; j < dV; ++j) {
                    double drj = -bt * du[j];
                    double Hd = Hm[(size_t)i * dV + j] + kt[i] * drj;
                    acc += hd[(size_t)i * dV + j] * drj;
                    ga += Hd * hd[(size_t)i * dV + j];
                    Hm[(size_t)i * dV + j] = a * Hd;
                }
                dkt[i] += acc;
                dgt[i] = ga;
            }
        }
        if (dh0) memcpy(dh0 + (size_t)bh * SZ, Hm, sizeof(double) * SZ);
        free(hs); free(Hm); free(hd); free(r); free(u); free(du);
    }
}

/* Gradients of KLA (beta = eta / (||k||^2 + eps)): the GDN gradients, then
 * the step size's chain rule into deta and dk. */
void kla_oracle_backward(const double *q, const double *k, const double *v, const double *g,
                         const double *eta, double eps, const double *h0,
                         const double *dout, const double *dhT,
                         double *dq, double *dk, double *dv, double *dg, double *deta,
                         double *dh0, int B, int T, int H, int dk_, int dv_)
{
    size_t n = (size_t)B * T * H;
    double *beta = (double *)malloc(sizeof(double) * (n ? n : 1));
    double *dbeta = (double *)malloc(sizeof(double) * (n ? n : 1));
    kla_oracle_beta(k, eta, eps, beta, B, T, H, dk_);
    kla_oracle_gated_delta_backward(q, k, v, g, beta, h0, dout, dhT, dq, dk, dv, dg, dbeta,
                                    dh0, B, T, H, dk_, dv_);
    for (size_t p = 0; p < n; ++p) {
        const double *kp = k + p * dk_;
        double n2 = 0.0;
        for (int i = 0; i < dk_; ++i) n2 += kp[i] * kp[i];
        double den = n2 + eps;
        deta[p] = dbeta[p] / den;
        double c = -2.0 * dbeta[p] * eta[p] / (den * den);
        for (int i = 0; i < dk_; ++i) dk[p * dk_ + i] += c * kp[i];
    }
    free(beta);
    free(dbeta);
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int kla_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
