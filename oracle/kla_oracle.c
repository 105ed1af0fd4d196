/*
 * kla_oracle.c -- plain fp64 CPU reference for Kaczmarz Linear Attention (KLA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA library is
 * checked against.  Only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark may load it.  It shares no code, header or
 * constant with the CUDA path, and the CUDA path never calls it.
 *
 * Source: "Kaczmarz Linear Attention" (arXiv 2605.08587).
 *   - kla_oracle_forward / kla_oracle_decode_step: the tokenwise update of
 *     Algorithm 1 (left panel) with the coefficient of Eq. (3):
 *         beta_t = eta_t / (||k_t||^2 + eps),  alpha_t = exp(g_t)
 *         Sbar   = alpha_t S_{t-1}
 *         e_t    = v_t - Sbar^T k_t
 *         S_t    = Sbar + beta_t k_t e_t^T
 *         o_t    = S_t^T q_t            (section 2 readout; q is used as given)
 *     g_t is the log-decay (the author's blog, "From Gated DeltaNet to
 *     Kaczmarz", section 2, writes alpha_t = exp(g_t)).
 *     If ||k_t||^2 + eps == 0 the write is skipped (beta_t = 0); the paper is
 *     silent on that case.
 *     With direct != 0 every function takes the write strength as given,
 *     beta_t = eta_t: the Gated DeltaNet update that the paper starts from
 *     (section 3.3 contrasts its beta with the Kaczmarz step; the blog "From
 *     Gated DeltaNet to Kaczmarz" writes the same recurrence with a learned
 *     beta); eps is then unused.
 *   - kla_oracle_backward: reverse-mode differentiation of the same token
 *     recurrence.  The paper gives no backward; this one is derived by hand
 *     from the forward above (chain rule, one token at a time, newest first)
 *     and is pinned only by finite differences.
 *   - kla_oracle_chunk_forward: the chunkwise form of section 4,
 *     Proposition 3 (Eq. 7) and Proposition 4 (Eqs. 8, 9), solved by forward
 *     substitution as Appendix B.2 states.  It exists only so that the tests
 *     can check the tokenwise oracle against an independent formulation.
 *
 * Layouts (all row-major, contiguous, fp64):
 *   q, k : [B, T, H, Dk]     v, o : [B, T, H, Dv]
 *   eta, g : [B, T, H]       S0, S_T, S : [B, H, Dk, Dv]
 * No blocking, fusion or reordering beyond the formulas above: one (b, h)
 * pair per OpenMP iteration, one token at a time.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define IDX_TOK(b, t, h, i, T, H, D) ((((size_t)(b) * (T) + (t)) * (H) + (h)) * (D) + (i))
#define IDX_GATE(b, t, h, T, H) (((size_t)(b) * (T) + (t)) * (H) + (h))
#define IDX_STATE(b, h, H, Dk, Dv) (((size_t)(b) * (H) + (h)) * (size_t)(Dk) * (Dv))

/* Eq. (3): beta = eta / (||k||^2 + eps); zero when the denominator is zero.
 * direct: beta = eta (the Gated DeltaNet write strength). */
static double kaczmarz_beta(double eta, double knorm2, double eps, int direct) {
    if (direct) return eta;
    double den = knorm2 + eps;
    return den != 0.0 ? eta / den : 0.0;
}

/* One tokenwise step of Algorithm 1 (left panel), in place on S (Dk x Dv).
 * e (length Dv) is scratch.  Writes o (length Dv) when o != NULL. */
static void token_step(double *S, const double *q, const double *k, const double *v, double eta,
                       double g, double eps, int direct, int Dk, int Dv, double *e, double *o) {
    double alpha = exp(g);
    double n = 0.0;
    for (int i = 0; i < Dk; ++i) n += k[i] * k[i];
    double beta = kaczmarz_beta(eta, n, eps, direct);
    /* Sbar = alpha S */
    for (size_t x = 0; x < (size_t)Dk * Dv; ++x) S[x] *= alpha;
    /* e = v - Sbar^T k */
    for (int j = 0; j < Dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < Dk; ++i) s += S[(size_t)i * Dv + j] * k[i];
        e[j] = v[j] - s;
    }
    /* S = Sbar + beta k e^T */
    for (int i = 0; i < Dk; ++i)
        for (int j = 0; j < Dv; ++j) S[(size_t)i * Dv + j] += beta * k[i] * e[j];
    /* o = S^T q */
    if (o) {
        for (int j = 0; j < Dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < Dk; ++i) s += S[(size_t)i * Dv + j] * q[i];
            o[j] = s;
        }
    }
}

/* Gather token t of head (b, h) into contiguous vectors. */
static void gather_token(const double *src, int b, int t, int h, int T, int H, int D, double *dst) {
    memcpy(dst, src + IDX_TOK(b, t, h, 0, T, H, D), sizeof(double) * (size_t)D);
}

int kla_oracle_forward(int B, int T, int H, int Dk, int Dv, const double *q, const double *k,
                       const double *v, const double *eta, const double *g, double eps, int direct,
                       const double *S0, double *o, double *S_T) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    int npairs = B * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < npairs; ++p) {
        int b = p / H, h = p % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)Dk * Dv);
        double *qt = (double *)malloc(sizeof(double) * (size_t)Dk);
        double *kt = (double *)malloc(sizeof(double) * (size_t)Dk);
        double *vt = (double *)malloc(sizeof(double) * (size_t)Dv);
        double *e = (double *)malloc(sizeof(double) * (size_t)Dv);
        double *ot = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!S || !qt || !kt || !vt || !e || !ot) {
#pragma omp atomic write
            bad = 1;
        } else {
            if (S0)
                memcpy(S, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * (size_t)Dk * Dv);
            else
                memset(S, 0, sizeof(double) * (size_t)Dk * Dv);
            for (int t = 0; t < T; ++t) {
                gather_token(q, b, t, h, T, H, Dk, qt);
                gather_token(k, b, t, h, T, H, Dk, kt);
                gather_token(v, b, t, h, T, H, Dv, vt);
                size_t gi = IDX_GATE(b, t, h, T, H);
                token_step(S, qt, kt, vt, eta[gi], g[gi], eps, direct, Dk, Dv, e, ot);
                if (o) memcpy(o + IDX_TOK(b, t, h, 0, T, H, Dv), ot, sizeof(double) * (size_t)Dv);
            }
            if (S_T) memcpy(S_T + IDX_STATE(b, h, H, Dk, Dv), S, sizeof(double) * (size_t)Dk * Dv);
        }
        free(S); free(qt); free(kt); free(vt); free(e); free(ot);
    }
    return bad ? 2 : 0;
}

/* One decode step: Algorithm 1 (left panel) once per (b, h), S updated in place.
 * q, k: [B, H, Dk]; v, o: [B, H, Dv]; eta, g: [B, H]; S: [B, H, Dk, Dv]. */
int kla_oracle_decode_step(int B, int H, int Dk, int Dv, const double *q, const double *k,
                           const double *v, const double *eta, const double *g, double eps, int direct,
                           double *S, double *o) {
    if (B < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    int npairs = B * H;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int p = 0; p < npairs; ++p) {
        double *e = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!e) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        token_step(S + (size_t)p * Dk * Dv, q + (size_t)p * Dk, k + (size_t)p * Dk,
                   v + (size_t)p * Dv, eta[p], g[p], eps, direct, Dk, Dv, e, o ? o + (size_t)p * Dv : NULL);
        free(e);
    }
    return bad ? 2 : 0;
}

/*
 * Backward of the token recurrence.  With G the gradient of the loss with
 * respect to S_t (seeded by dS_T, zero when dS_T is NULL), newest token first:
 *   G     += q do^T                       (o_t = S_t^T q_t)
 *   dq     = S_t do
 *   de     = beta G^T k                    (S_t = Sbar + beta k e^T)
 *   dbeta  = k^T G e
 *   dv     = de                            (e = v - Sbar^T k)
 *   dn     = -dbeta * beta / (n + eps)     (n = ||k||^2)
 *   deta   = dbeta / (n + eps)
 *   (direct: beta = eta, so dn = 0 and deta = dbeta)
 *   dk     = beta G e - Sbar de + 2 k dn
 *   dSbar  = G - k de^T
 *   dg     = alpha <dSbar, S_{t-1}>_F      (Sbar = exp(g) S_{t-1})
 *   G      = alpha dSbar                   (gradient w.r.t. S_{t-1})
 * and dS0 = G at the end.  When n + eps == 0 the write is skipped, so
 * dbeta does not reach eta or n.
 * States S_{t-1} are recomputed from checkpoints taken every `ckpt` tokens.
 */
int kla_oracle_backward(int B, int T, int H, int Dk, int Dv, const double *q, const double *k,
                        const double *v, const double *eta, const double *g, double eps, int direct,
                        const double *S0, const double *dO, const double *dS_T, double *dq,
                        double *dk, double *dv, double *deta, double *dg, double *dS0,
                        int ckpt) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    if (ckpt <= 0) ckpt = 64;
    int npairs = B * H;
    int bad = 0;
    size_t SS = (size_t)Dk * Dv;
    int nck = T > 0 ? (T + ckpt - 1) / ckpt : 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < npairs; ++p) {
        int b = p / H, h = p % H;
        double *ck = (double *)malloc(sizeof(double) * SS * (size_t)(nck + 1));
        double *blk = (double *)malloc(sizeof(double) * SS * (size_t)(ckpt + 1));
        double *G = (double *)malloc(sizeof(double) * SS);
        double *dSb = (double *)malloc(sizeof(double) * SS);
        double *vec = (double *)malloc(sizeof(double) * (size_t)(5 * Dk + 4 * Dv));
        if (!ck || !blk || !G || !dSb || !vec) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *qt = vec, *kt = qt + Dk, *vt = kt + Dk, *e = vt + Dv, *dot = e + Dv;
            double *de = dot + Dv, *dkt = de + Dv, *dqt = dkt + Dk;
            double *Sbde = dqt + Dk;
            /* forward pass keeping checkpoints of S at the start of each block */
            double *S = blk;
            if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (int c = 0; c < nck; ++c) {
                memcpy(ck + (size_t)c * SS, S, sizeof(double) * SS);
                int t1 = (c + 1) * ckpt < T ? (c + 1) * ckpt : T;
                for (int t = c * ckpt; t < t1; ++t) {
                    gather_token(q, b, t, h, T, H, Dk, qt);
                    gather_token(k, b, t, h, T, H, Dk, kt);
                    gather_token(v, b, t, h, T, H, Dv, vt);
                    size_t gi = IDX_GATE(b, t, h, T, H);
                    token_step(S, qt, kt, vt, eta[gi], g[gi], eps, direct, Dk, Dv, e, NULL);
                }
            }
            if (dS_T) memcpy(G, dS_T + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(G, 0, sizeof(double) * SS);
            for (int c = nck - 1; c >= 0; --c) {
                int t0 = c * ckpt;
                int t1 = (c + 1) * ckpt < T ? (c + 1) * ckpt : T;
                /* recompute S_{t0} .. S_{t1} into blk[0 .. t1-t0] */
                memcpy(blk, ck + (size_t)c * SS, sizeof(double) * SS);
                for (int t = t0; t < t1; ++t) {
                    double *Sn = blk + (size_t)(t - t0 + 1) * SS;
                    memcpy(Sn, blk + (size_t)(t - t0) * SS, sizeof(double) * SS);
                    gather_token(q, b, t, h, T, H, Dk, qt);
                    gather_token(k, b, t, h, T, H, Dk, kt);
                    gather_token(v, b, t, h, T, H, Dv, vt);
                    size_t gi = IDX_GATE(b, t, h, T, H);
                    token_step(Sn, qt, kt, vt, eta[gi], g[gi], eps, direct, Dk, Dv, e, NULL);
                }
                for (int t = t1 - 1; t >= t0; --t) {
                    const double *Sprev = blk + (size_t)(t - t0) * SS;
                    const double *Scur = blk + (size_t)(t - t0 + 1) * SS;
                    gather_token(q, b, t, h, T, H, Dk, qt);
                    gather_token(k, b, t, h, T, H, Dk, kt);
                    gather_token(v, b, t, h, T, H, Dv, vt);
                    gather_token(dO, b, t, h, T, H, Dv, dot);
                    size_t gi = IDX_GATE(b, t, h, T, H);
                    double alpha = exp(g[gi]);
                    double n = 0.0;
                    for (int i = 0; i < Dk; ++i) n += kt[i] * kt[i];
                    double den = n + eps;
                    double beta = kaczmarz_beta(eta[gi], n, eps, direct);
                    /* e = v - Sbar^T k, Sbar = alpha S_{t-1} */
                    for (int j = 0; j < Dv; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < Dk; ++i) s += alpha * Sprev[(size_t)i * Dv + j] * kt[i];
                        e[j] = vt[j] - s;
                    }
                    /* G += q do^T */
                    for (int i = 0; i < Dk; ++i)
                        for (int j = 0; j < Dv; ++j) G[(size_t)i * Dv + j] += qt[i] * dot[j];
                    /* dq = S_t do */
                    for (int i = 0; i < Dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < Dv; ++j) s += Scur[(size_t)i * Dv + j] * dot[j];
                        dqt[i] = s;
                    }
                    /* de = beta G^T k ; dbeta = k^T G e */
                    double dbeta = 0.0;
                    for (int j = 0; j < Dv; ++j) {
                        double s = 0.0;
                        for (int i = 0; i < Dk; ++i) s += G[(size_t)i * Dv + j] * kt[i];
                        de[j] = beta * s;
                        dbeta += s * e[j];
                    }
                    double dn = 0.0, detat = 0.0;
                    if (direct) {
                        detat = dbeta;
                    } else if (den != 0.0) {
                        dn = -dbeta * beta / den;
                        detat = dbeta / den;
                    }
                    /* Sbar de */
                    for (int i = 0; i < Dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < Dv; ++j) s += alpha * Sprev[(size_t)i * Dv + j] * de[j];
                        Sbde[i] = s;
                    }
                    /* dk = beta G e - Sbar de + 2 k dn */
                    for (int i = 0; i < Dk; ++i) {
                        double s = 0.0;
                        for (int j = 0; j < Dv; ++j) s += G[(size_t)i * Dv + j] * e[j];
                        dkt[i] = beta * s - Sbde[i] + 2.0 * kt[i] * dn;
                    }
                    /* dSbar = G - k de^T ; dg = alpha <dSbar, S_{t-1}> ; G = alpha dSbar */
                    double dgt = 0.0;
                    for (int i = 0; i < Dk; ++i)
                        for (int j = 0; j < Dv; ++j) {
                            size_t x = (size_t)i * Dv + j;
                            double d = G[x] - kt[i] * de[j];
                            dgt += d * Sprev[x];
                            dSb[x] = d;
                        }
                    dgt *= alpha;
                    for (size_t x = 0; x < SS; ++x) G[x] = alpha * dSb[x];
                    memcpy(dq + IDX_TOK(b, t, h, 0, T, H, Dk), dqt, sizeof(double) * (size_t)Dk);
                    memcpy(dk + IDX_TOK(b, t, h, 0, T, H, Dk), dkt, sizeof(double) * (size_t)Dk);
                    memcpy(dv + IDX_TOK(b, t, h, 0, T, H, Dv), de, sizeof(double) * (size_t)Dv);
                    deta[gi] = detat;
                    dg[gi] = dgt;
                }
            }
            memcpy(dS0 + IDX_STATE(b, h, H, Dk, Dv), G, sizeof(double) * SS);
        }
        free(ck); free(blk); free(G); free(dSb); free(vec);
    }
    return bad ? 2 : 0;
}

/*
 * Chunkwise form (section 4, Propositions 3 and 4; Appendix B.2, B.3).
 * Per chunk of length C (the last chunk may be shorter), with local index
 * i = 1..C, incoming state S (Dk x Dv):
 *   gamma_i = prod_{r<=i} alpha_r,  beta_i = eta_i / (||k_i||^2 + eps)
 *   A_ij    = gamma_i / gamma_j for j <= i (0 otherwise); A^- its strict part
 *   (I + B (A^- o K K^T)) U = B (V - D_gamma K S)          (Eq. 7)
 *   O     = D_gamma Q S + (A o Q K^T) U                     (Eq. 8)
 *   S_out = gamma_C S + K^T Diag(gamma_C / gamma_1 .. 1) U   (Eq. 9)
 * The unit-lower-triangular system is solved by forward substitution.
 */
int kla_oracle_chunk_forward(int B, int T, int H, int Dk, int Dv, const double *q,
                             const double *k, const double *v, const double *eta,
                             const double *g, double eps, int direct, const double *S0, int C, double *o,
                             double *S_T) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0 || C <= 0) return 1;
    int npairs = B * H;
    int bad = 0;
    size_t SS = (size_t)Dk * Dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < npairs; ++p) {
        int b = p / H, h = p % H;
        double *S = (double *)malloc(sizeof(double) * SS);
        double *Sn = (double *)malloc(sizeof(double) * SS);
        double *K = (double *)malloc(sizeof(double) * (size_t)C * Dk);
        double *Q = (double *)malloc(sizeof(double) * (size_t)C * Dk);
        double *V = (double *)malloc(sizeof(double) * (size_t)C * Dv);
        double *U = (double *)malloc(sizeof(double) * (size_t)C * Dv);
        double *Mx = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *gam = (double *)malloc(sizeof(double) * (size_t)C);
        double *bet = (double *)malloc(sizeof(double) * (size_t)C);
        if (!S || !Sn || !K || !Q || !V || !U || !Mx || !gam || !bet) {
#pragma omp atomic write
            bad = 1;
        } else {
            if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (int t0 = 0; t0 < T; t0 += C) {
                int n = T - t0 < C ? T - t0 : C;
                for (int i = 0; i < n; ++i) {
                    gather_token(q, b, t0 + i, h, T, H, Dk, Q + (size_t)i * Dk);
                    gather_token(k, b, t0 + i, h, T, H, Dk, K + (size_t)i * Dk);
                    gather_token(v, b, t0 + i, h, T, H, Dv, V + (size_t)i * Dv);
                }
                /* gamma and beta (Algorithm 1, right panel, first loop) */
                double gprev = 1.0;
                for (int i = 0; i < n; ++i) {
                    size_t gi = IDX_GATE(b, t0 + i, h, T, H);
                    gam[i] = exp(g[gi]) * gprev;
                    gprev = gam[i];
                    double kn = 0.0;
                    for (int x = 0; x < Dk; ++x) kn += K[(size_t)i * Dk + x] * K[(size_t)i * Dk + x];
                    bet[i] = kaczmarz_beta(eta[gi], kn, eps, direct);
                }
                /* strictly lower L = B (A^- o K K^T), stored in Mx */
                for (int i = 0; i < n; ++i)
                    for (int j = 0; j < n; ++j) {
                        double val = 0.0;
                        if (j < i) {
                            double kk = 0.0;
                            for (int x = 0; x < Dk; ++x) kk += K[(size_t)i * Dk + x] * K[(size_t)j * Dk + x];
                            val = bet[i] * (gam[i] / gam[j]) * kk;
                        }
                        Mx[(size_t)i * C + j] = val;
                    }
                /* right-hand side B (V - D_gamma K S), into U */
                for (int i = 0; i < n; ++i)
                    for (int c2 = 0; c2 < Dv; ++c2) {
                        double ks = 0.0;
                        for (int x = 0; x < Dk; ++x) ks += K[(size_t)i * Dk + x] * S[(size_t)x * Dv + c2];
                        U[(size_t)i * Dv + c2] = bet[i] * (V[(size_t)i * Dv + c2] - gam[i] * ks);
                    }
                /* forward substitution: u_i = rhs_i - sum_{j<i} L_ij u_j */
                for (int i = 0; i < n; ++i)
                    for (int j = 0; j < i; ++j) {
                        double l = Mx[(size_t)i * C + j];
                        for (int c2 = 0; c2 < Dv; ++c2) U[(size_t)i * Dv + c2] -= l * U[(size_t)j * Dv + c2];
                    }
                /* O = D_gamma Q S + (A o Q K^T) U */
                for (int i = 0; i < n; ++i) {
                    double *orow = o ? o + IDX_TOK(b, t0 + i, h, 0, T, H, Dv) : NULL;
                    if (!orow) break;
                    for (int c2 = 0; c2 < Dv; ++c2) {
                        double qs = 0.0;
                        for (int x = 0; x < Dk; ++x) qs += Q[(size_t)i * Dk + x] * S[(size_t)x * Dv + c2];
                        orow[c2] = gam[i] * qs;
                    }
                    for (int j = 0; j <= i; ++j) {
                        double qk = 0.0;
                        for (int x = 0; x < Dk; ++x) qk += Q[(size_t)i * Dk + x] * K[(size_t)j * Dk + x];
                        double a = (gam[i] / gam[j]) * qk;
                        for (int c2 = 0; c2 < Dv; ++c2) orow[c2] += a * U[(size_t)j * Dv + c2];
                    }
                }
                /* S_out = gamma_C S + K^T Diag(gamma_C / gamma_j) U */
                double gC = gam[n - 1];
                for (int x = 0; x < Dk; ++x)
                    for (int c2 = 0; c2 < Dv; ++c2) {
                        double s = gC * S[(size_t)x * Dv + c2];
                        for (int j = 0; j < n; ++j) s += K[(size_t)j * Dk + x] * (gC / gam[j]) * U[(size_t)j * Dv + c2];
                        Sn[(size_t)x * Dv + c2] = s;
                    }
                memcpy(S, Sn, sizeof(double) * SS);
            }
            if (S_T) memcpy(S_T + IDX_STATE(b, h, H, Dk, Dv), S, sizeof(double) * SS);
        }
        free(S); free(Sn); free(K); free(Q); free(V); free(U); free(Mx); free(gam); free(bet);
    }
    return bad ? 2 : 0;
}

/*
 * Diagonal gating ("Kaczmarz Linear Attention", Appendix A.5 and B.5): the decay is the
 * per-key-channel operator D_t = Diag(alpha_t), alpha_t = exp(g_t) with g_t in R^{Dk}:
 *     Sdec = Diag(alpha_t) S_{t-1}
 *     e_t  = v_t - Sdec^T k_t
 *     S_t  = Sdec + beta_t k_t e_t^T      (beta_t unchanged: A.5's decay-agnostic remark)
 *     o_t  = S_t^T q_t
 * g is laid out [B, T, H, Dk].  Not yet a row of the CUDA library: these functions exist so that
 * its diagonal-gated kernels can be checked against them.
 */
static void diag_token_step(double *S, const double *q, const double *k, const double *v, double eta,
                            const double *gvec, double eps, int direct, int Dk, int Dv, double *resid,
                            double *out) {
    double knorm2 = 0.0;
    for (int r = 0; r < Dk; ++r) knorm2 += k[r] * k[r];
    const double bt = kaczmarz_beta(eta, knorm2, eps, direct);
    for (int r = 0; r < Dk; ++r) {
        const double ar = exp(gvec[r]);
        for (int c = 0; c < Dv; ++c) S[(size_t)r * Dv + c] *= ar;
    }
    for (int c = 0; c < Dv; ++c) {
        double acc = 0.0;
        for (int r = 0; r < Dk; ++r) acc += k[r] * S[(size_t)r * Dv + c];
        resid[c] = v[c] - acc;
    }
    for (int r = 0; r < Dk; ++r) {
        const double w = bt * k[r];
        for (int c = 0; c < Dv; ++c) S[(size_t)r * Dv + c] += w * resid[c];
    }
    if (out) {
        for (int c = 0; c < Dv; ++c) {
            double acc = 0.0;
            for (int r = 0; r < Dk; ++r) acc += q[r] * S[(size_t)r * Dv + c];
            out[c] = acc;
        }
    }
}

int kla_oracle_forward_diag(int B, int T, int H, int Dk, int Dv, const double *q, const double *k,
                            const double *v, const double *eta, const double *g, double eps, int direct,
                            const double *S0, double *o, double *ST) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    int bad = 0;
    const size_t SS = (size_t)Dk * Dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < B * H; ++p) {
        const int b = p / H, h = p % H;
        double *S = (double *)malloc(sizeof(double) * SS);
        double *tmp = (double *)malloc(sizeof(double) * (size_t)(3 * Dk + 3 * Dv));
        if (!S || !tmp) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *qv = tmp, *kv = qv + Dk, *gv = kv + Dk, *vv = gv + Dk, *res = vv + Dv, *ov = res + Dv;
            if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (int t = 0; t < T; ++t) {
                gather_token(q, b, t, h, T, H, Dk, qv);
                gather_token(k, b, t, h, T, H, Dk, kv);
                gather_token(v, b, t, h, T, H, Dv, vv);
                gather_token(g, b, t, h, T, H, Dk, gv);
                diag_token_step(S, qv, kv, vv, eta[IDX_GATE(b, t, h, T, H)], gv, eps, direct, Dk, Dv, res,
                                o ? ov : NULL);
                if (o) memcpy(o + IDX_TOK(b, t, h, 0, T, H, Dv), ov, sizeof(double) * (size_t)Dv);
            }
            if (ST) memcpy(ST + IDX_STATE(b, h, H, Dk, Dv), S, sizeof(double) * SS);
        }
        free(S); free(tmp);
    }
    return bad ? 2 : 0;
}

int kla_oracle_decode_step_diag(int B, int H, int Dk, int Dv, const double *q, const double *k,
                                const double *v, const double *eta, const double *g, double eps, int direct,
                                double *S, double *o) {
    if (B < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int p = 0; p < B * H; ++p) {
        double *res = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!res) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        diag_token_step(S + (size_t)p * Dk * Dv, q + (size_t)p * Dk, k + (size_t)p * Dk, v + (size_t)p * Dv, eta[p],
                        g + (size_t)p * Dk, eps, direct, Dk, Dv, res, o ? o + (size_t)p * Dv : NULL);
        free(res);
    }
    return bad ? 2 : 0;
}

/*
 * Backward of the diagonal-gated recurrence, newest token first, with Lambda = dL/dS_t:
 *   Lambda += q do^T;  dq = S_t do;  de = beta Lambda^T k;  dbeta = k^T Lambda e;  dv = de
 *   dn, deta as for scalar gating (Kaczmarz or direct beta)
 *   dk = beta Lambda e - Sdec de + 2 k dn
 *   dSdec = Lambda - k de^T
 *   dg[r] = alpha[r] sum_c dSdec[r][c] S_{t-1}[r][c]     (one entry per key channel)
 *   Lambda <- Diag(alpha) dSdec
 * States are recomputed forward from S0 for every token (plain, slow: the sizes the tests use
 * are tiny).
 */
int kla_oracle_backward_diag(int B, int T, int H, int Dk, int Dv, const double *q, const double *k,
                             const double *v, const double *eta, const double *g, double eps, int direct,
                             const double *S0, const double *dO, const double *dS_T, double *dq, double *dk,
                             double *dv, double *deta, double *dg, double *dS0) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return 1;
    int bad = 0;
    const size_t SS = (size_t)Dk * Dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < B * H; ++p) {
        const int b = p / H, h = p % H;
        double *states = (double *)malloc(sizeof(double) * SS * (size_t)(T + 1));
        double *Lam = (double *)malloc(sizeof(double) * SS);
        double *tmp = (double *)malloc(sizeof(double) * (size_t)(5 * Dk + 4 * Dv));
        if (!states || !Lam || !tmp) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *qv = tmp, *kv = qv + Dk, *gv = kv + Dk, *dqv = gv + Dk, *dkv = dqv + Dk;
            double *vv = dkv + Dk, *res = vv + Dv, *dov = res + Dv, *dres = dov + Dv;
            if (S0) memcpy(states, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(states, 0, sizeof(double) * SS);
            for (int t = 0; t < T; ++t) {  /* states[t] = S_t (states[0] = S0) */
                memcpy(states + (size_t)(t + 1) * SS, states + (size_t)t * SS, sizeof(double) * SS);
                gather_token(q, b, t, h, T, H, Dk, qv);
                gather_token(k, b, t, h, T, H, Dk, kv);
                gather_token(v, b, t, h, T, H, Dv, vv);
                gather_token(g, b, t, h, T, H, Dk, gv);
                diag_token_step(states + (size_t)(t + 1) * SS, qv, kv, vv, eta[IDX_GATE(b, t, h, T, H)], gv, eps,
                                direct, Dk, Dv, res, NULL);
            }
            if (dS_T) memcpy(Lam, dS_T + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(Lam, 0, sizeof(double) * SS);
            for (int t = T - 1; t >= 0; --t) {
                const double *Sp = states + (size_t)t * SS, *Sc = states + (size_t)(t + 1) * SS;
                gather_token(q, b, t, h, T, H, Dk, qv);
                gather_token(k, b, t, h, T, H, Dk, kv);
                gather_token(v, b, t, h, T, H, Dv, vv);
                gather_token(g, b, t, h, T, H, Dk, gv);
                gather_token(dO, b, t, h, T, H, Dv, dov);
                const size_t gi = IDX_GATE(b, t, h, T, H);
                double knorm2 = 0.0;
                for (int r = 0; r < Dk; ++r) knorm2 += kv[r] * kv[r];
                const double kden = knorm2 + eps;
                const double bt = kaczmarz_beta(eta[gi], knorm2, eps, direct);
                for (int c = 0; c < Dv; ++c) {  /* residual against the decayed state */
                    double acc = 0.0;
                    for (int r = 0; r < Dk; ++r) acc += kv[r] * exp(gv[r]) * Sp[(size_t)r * Dv + c];
                    res[c] = vv[c] - acc;
                }
                for (int r = 0; r < Dk; ++r)
                    for (int c = 0; c < Dv; ++c) Lam[(size_t)r * Dv + c] += qv[r] * dov[c];
                for (int r = 0; r < Dk; ++r) {
                    double acc = 0.0;
                    for (int c = 0; c < Dv; ++c) acc += Sc[(size_t)r * Dv + c] * dov[c];
                    dqv[r] = acc;
                }
                double dbt = 0.0;
                for (int c = 0; c < Dv; ++c) {
                    double acc = 0.0;
                    for (int r = 0; r < Dk; ++r) acc += Lam[(size_t)r * Dv + c] * kv[r];
                    dres[c] = bt * acc;
                    dbt += acc * res[c];
                }
                double dnorm = 0.0, det = 0.0;
                if (direct) det = dbt;
                else if (kden != 0.0) { dnorm = -dbt * bt / kden; det = dbt / kden; }
                for (int r = 0; r < Dk; ++r) {
                    const double ar = exp(gv[r]);
                    double a1 = 0.0, a2 = 0.0;
                    for (int c = 0; c < Dv; ++c) {
                        a1 += Lam[(size_t)r * Dv + c] * res[c];
                        a2 += ar * Sp[(size_t)r * Dv + c] * dres[c];
                    }
                    dkv[r] = bt * a1 - a2 + 2.0 * kv[r] * dnorm;
                }
                for (int r = 0; r < Dk; ++r) {
                    const double ar = exp(gv[r]);
                    double acc = 0.0;
                    for (int c = 0; c < Dv; ++c) {
                        const size_t x = (size_t)r * Dv + c;
                        const double dsd = Lam[x] - kv[r] * dres[c];
                        acc += dsd * Sp[x];
                        Lam[x] = ar * dsd;
                    }
                    dg[IDX_TOK(b, t, h, r, T, H, Dk)] = ar * acc;
                }
                memcpy(dq + IDX_TOK(b, t, h, 0, T, H, Dk), dqv, sizeof(double) * (size_t)Dk);
                memcpy(dk + IDX_TOK(b, t, h, 0, T, H, Dk), dkv, sizeof(double) * (size_t)Dk);
                memcpy(dv + IDX_TOK(b, t, h, 0, T, H, Dv), dres, sizeof(double) * (size_t)Dv);
                deta[gi] = det;
            }
            memcpy(dS0 + IDX_STATE(b, h, H, Dk, Dv), Lam, sizeof(double) * SS);
        }
        free(states); free(Lam); free(tmp);
    }
    return bad ? 2 : 0;
}

/*
 * Chunk form of the diagonal-gated recurrence (Appendix B.5: the scalar decay products become
 * elementwise).  Per chunk, G_i = sum_{r<=i} g_r per channel; for i > j the decayed Gram is
 * A_ij = sum_c k_i[c] k_j[c] exp(G_i[c] - G_j[c]); then, solving by forward substitution,
 *     u_i = beta_i (v_i - S0^T (exp(G_i) o k_i)) - beta_i sum_{j<i} A_ij u_j
 *     o_i = S0^T (exp(G_i) o q_i) + sum_{j<=i} [sum_c q_i[c] k_j[c] exp(G_i[c] - G_j[c])] u_j
 *     S_end = Diag(exp(G_C)) S0 + sum_j Diag(exp(G_C - G_j)) k_j u_j^T
 * Used only to check the token form above.
 */
int kla_oracle_chunk_forward_diag(int B, int T, int H, int Dk, int Dv, const double *q, const double *k,
                                  const double *v, const double *eta, const double *g, double eps, int direct,
                                  const double *S0, int C, double *o, double *ST) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0 || C <= 0) return 1;
    int bad = 0;
    const size_t SS = (size_t)Dk * Dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < B * H; ++p) {
        const int b = p / H, h = p % H;
        double *S = (double *)malloc(sizeof(double) * SS);
        double *Gc = (double *)malloc(sizeof(double) * (size_t)C * Dk);
        double *uu = (double *)malloc(sizeof(double) * (size_t)C * Dv);
        double *bb = (double *)malloc(sizeof(double) * (size_t)C);
        double *Snew = (double *)malloc(sizeof(double) * SS);
        if (!S || !Gc || !uu || !bb || !Snew) {
#pragma omp atomic write
            bad = 1;
        } else {
            if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, Dk, Dv), sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (int t0 = 0; t0 < T; t0 += C) {
                const int n = T - t0 < C ? T - t0 : C;
                for (int i = 0; i < n; ++i) {
                    const double *ki = k + IDX_TOK(b, t0 + i, h, 0, T, H, Dk);
                    double kn = 0.0;
                    for (int r = 0; r < Dk; ++r) {
                        const double gr = g[IDX_TOK(b, t0 + i, h, r, T, H, Dk)];
                        Gc[(size_t)i * Dk + r] = (i ? Gc[(size_t)(i - 1) * Dk + r] : 0.0) + gr;
                        kn += ki[r] * ki[r];
                    }
                    bb[i] = kaczmarz_beta(eta[IDX_GATE(b, t0 + i, h, T, H)], kn, eps, direct);
                }
                for (int i = 0; i < n; ++i) {
                    const double *ki = k + IDX_TOK(b, t0 + i, h, 0, T, H, Dk);
                    const double *vi = v + IDX_TOK(b, t0 + i, h, 0, T, H, Dv);
                    for (int c = 0; c < Dv; ++c) {
                        double acc = 0.0;
                        for (int r = 0; r < Dk; ++r) acc += exp(Gc[(size_t)i * Dk + r]) * ki[r] * S[(size_t)r * Dv + c];
                        uu[(size_t)i * Dv + c] = bb[i] * (vi[c] - acc);
                    }
                    for (int j = 0; j < i; ++j) {
                        const double *kj = k + IDX_TOK(b, t0 + j, h, 0, T, H, Dk);
                        double aij = 0.0;
                        for (int r = 0; r < Dk; ++r)
                            aij += ki[r] * kj[r] * exp(Gc[(size_t)i * Dk + r] - Gc[(size_t)j * Dk + r]);
                        for (int c = 0; c < Dv; ++c) uu[(size_t)i * Dv + c] -= bb[i] * aij * uu[(size_t)j * Dv + c];
                    }
                }
                if (o) {
                    for (int i = 0; i < n; ++i) {
                        const double *qi = q + IDX_TOK(b, t0 + i, h, 0, T, H, Dk);
                        double *oi = o + IDX_TOK(b, t0 + i, h, 0, T, H, Dv);
                        for (int c = 0; c < Dv; ++c) {
                            double acc = 0.0;
                            for (int r = 0; r < Dk; ++r) acc += exp(Gc[(size_t)i * Dk + r]) * qi[r] * S[(size_t)r * Dv + c];
                            oi[c] = acc;
                        }
                        for (int j = 0; j <= i; ++j) {
                            const double *kj = k + IDX_TOK(b, t0 + j, h, 0, T, H, Dk);
                            double sij = 0.0;
                            for (int r = 0; r < Dk; ++r)
                                sij += qi[r] * kj[r] * exp(Gc[(size_t)i * Dk + r] - Gc[(size_t)j * Dk + r]);
                            for (int c = 0; c < Dv; ++c) oi[c] += sij * uu[(size_t)j * Dv + c];
                        }
                    }
                }
                for (int r = 0; r < Dk; ++r) {
                    const double gl = Gc[(size_t)(n - 1) * Dk + r];
                    for (int c = 0; c < Dv; ++c) {
                        double acc = exp(gl) * S[(size_t)r * Dv + c];
                        for (int j = 0; j < n; ++j) {
                            const double kjr = k[IDX_TOK(b, t0 + j, h, r, T, H, Dk)];
                            acc += exp(gl - Gc[(size_t)j * Dk + r]) * kjr * uu[(size_t)j * Dv + c];
                        }
                        Snew[(size_t)r * Dv + c] = acc;
                    }
                }
                memcpy(S, Snew, sizeof(double) * SS);
            }
            if (ST) memcpy(ST + IDX_STATE(b, h, H, Dk, Dv), S, sizeof(double) * SS);
        }
        free(S); free(Gc); free(uu); free(bb); free(Snew);
    }
    return bad ? 2 : 0;
}
