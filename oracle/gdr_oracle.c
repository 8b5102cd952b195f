/*
 * gdr_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library.  It shares no code, header,
 * table or helper with the CUDA library in gated_delta_rule_91_b200/csrc, and
 * the product path never calls it.
 *
 * Every function runs the recurrence exactly as the pages state it, one token
 * at a time, in double precision, with no chunking, blocking or reordering.
 * Parallelism is only across independent (batch, head) units (OpenMP); the
 * time loop is always sequential.
 *
 * Sources (cited by page title and section):
 *   [GDN-R]  "[논문리뷰] Gated Delta Netoworks: Improving MAMBA2 with Delta Rule
 *            (ICLR, 2025)", meaningful96.github.io/nr/GDN
 *            -- section 1 (problem: inputs q,k,v,alpha,beta; outputs S_t and
 *               o_t = S_t q_t), section 3.3 (delta rule, two written forms),
 *               section 3.4 (gated delta rule), section 3.5 (SGD view).
 *   [GDN-E]  "Gated DeltaNet: Merging Gating and the Delta Rule to Beat Mamba2
 *            on Language and Retrieval", agihunt.info/en/papers/2412.06464,
 *            section "Method" (the gated delta rule).
 *   [GDN2]   "Gated DeltaNet-2: Decoupling Erase and Write in Linear
 *            Attention", agihunt.info/papers/2605.22791, the paragraph on
 *            Gated Delta Rule-2 (decay by alpha_t, read along b_t*k_t, write
 *            the residual of w_t*v_t along k_t).  The printed formula is
 *            missing from the extracted page; the update used here is the
 *            plainest reading of that paragraph's stated order of operations.
 *
 * Layouts (row-major, all double):
 *   q, k        [B, T, H, dk]        v, o, dO     [B, T, H, dv]
 *   log_alpha   [B, T, H]            beta         [B, T, H]
 *   S0, S_T     [B, H, dv, dk]       (S = sum of v k^T, so dv rows, dk cols)
 *   GDN-2:  log_alpha [B,T,H,dk] (per key channel), b [B,T,H,dk], w [B,T,H,dv]
 *
 * Any pointer documented as "may be NULL" is treated as all-zeros (inputs) or
 * skipped (outputs).
 *
 * Parity status: every entry point here is pinned by tests/test_oracle_*.py
 * against identities, closed forms, exact rational arithmetic, a hand-worked
 * example and finite differences; see those files.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of host threads the oracle's parallel loops use. */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static size_t tok_index(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

/*
 * One token of the gated delta rule on one head, in place:
 *     S <- S . alpha (I - beta k k^T) + beta v k^T          ([GDN-R] 3.4)
 * evaluated through the expanded delta form of [GDN-R] 3.3,
 *     S <- alpha S + beta (v - alpha S k) k^T,
 * which is the same matrix (alpha scales S before the read, as S.alpha(I-..)
 * distributes).  Then the readout o = S q uses the UPDATED state ([GDN-R] 1:
 * o_t = S_t q_t).  `r` is caller scratch of length dv.  `o` may be NULL.
 */
static void gdr_token(int dk, int dv, double *S, const double *q,
                      const double *k, const double *v, double alpha,
                      double beta, double *r, double *o, size_t o_stride) {
    for (int i = 0; i < dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * k[j];
        r[i] = acc;                              /* r = S_{t-1} k_t */
    }
    for (int i = 0; i < dv; ++i) {
        double u = beta * (v[i] - alpha * r[i]); /* delta, scaled by beta */
        double *row = S + (size_t)i * dk;
        for (int j = 0; j < dk; ++j) row[j] = alpha * row[j] + u * k[j];
    }
    if (o) {
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * q[j];
            o[i * o_stride] = acc;
        }
    }
}

/*
 * Forward: for every (b,h), S = S0 (or 0), then for t = 0..T-1 apply one
 * token of the gated delta rule and read o_t = S_t q_t.  Writes o and, if
 * S_T != NULL, the final state.
 */
void oracle_gdr_fwd(int B, int T, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *log_alpha, const double *beta,
                    const double *S0, double *o, double *S_T) {
    long units = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < units; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        size_t ssz = (size_t)dv * dk;
        double *S = (double *)malloc(ssz * sizeof(double));
        double *r = (double *)malloc((size_t)dv * sizeof(double));
        if (S0) memcpy(S, S0 + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(S, 0, ssz * sizeof(double));
        for (int t = 0; t < T; ++t) {
            size_t ti = tok_index(b, t, h, T, H);
            gdr_token(dk, dv, S, q + ti * dk, k + ti * dk, v + ti * dv,
                      exp(log_alpha[ti]), beta[ti], r, o ? o + ti * dv : NULL, 1);
        }
        if (S_T) memcpy(S_T + (size_t)bh * ssz, S, ssz * sizeof(double));
        free(S);
        free(r);
    }
}

/*
 * Single-token decode: one token of the same recurrence on every (b,h),
 * state S [B,H,dv,dk] updated in place, o [B,H,dv] = S_t q_t.
 * Inputs q,k [B,H,dk], v [B,H,dv], log_alpha, beta [B,H].
 */
void oracle_gdr_step(int B, int H, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *log_alpha, const double *beta,
                     double *S, double *o) {
    long units = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < units; ++bh) {
        double *r = (double *)malloc((size_t)dv * sizeof(double));
        gdr_token(dk, dv, S + (size_t)bh * dv * dk, q + (size_t)bh * dk,
                  k + (size_t)bh * dk, v + (size_t)bh * dv,
                  exp(log_alpha[bh]), beta[bh], r, o + (size_t)bh * dv, 1);
        free(r);
    }
}

/*
 * Reverse mode of oracle_gdr_fwd (the pages give no backward; this is the
 * chain rule applied to the per-token update above, by hand).
 *
 * Per token, with P = S_{t-1}, a = alpha_t, r = P k, e = v - a r, u = beta e:
 *   S_t = a P + u k^T,     o_t = S_t q.
 * Given G = dL/dS_t (from later tokens and dS_T) the step is
 *   G   += do_t q^T                       (readout)
 *   dq_t = S_t^T do_t
 *   gk   = G k
 *   dv_t = beta gk
 *   dbeta_t = e . gk
 *   dk_t = beta G^T e - a beta P^T gk
 *   da   = <G, P>_F - beta r . gk ;   dlog_alpha_t = a da
 *   G   <- a G - a beta gk k^T            (= dL/dS_{t-1})
 * and dS0 is the final G.
 *
 * States are checkpointed every CK tokens and recomputed inside each block
 * (plain recomputation with the same forward arithmetic), so memory stays at
 * (T/CK + CK) states per head.
 * dO is required; dS_T may be NULL (zero).  All outputs are written fully.
 */
#define ORACLE_CK 64
void oracle_gdr_bwd(int B, int T, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *log_alpha, const double *beta,
                    const double *S0, const double *dO, const double *dS_T,
                    double *dq, double *dk_out, double *dv_out,
                    double *dlog_alpha, double *dbeta, double *dS0) {
    long units = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < units; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        size_t ssz = (size_t)dv * dk;
        int nblk = (T + ORACLE_CK - 1) / ORACLE_CK;
        double *ckpt = (double *)malloc((size_t)(nblk > 0 ? nblk : 1) * ssz * sizeof(double));
        double *Sb = (double *)malloc((size_t)(ORACLE_CK + 1) * ssz * sizeof(double));
        double *G = (double *)malloc(ssz * sizeof(double));
        double *r = (double *)malloc((size_t)dv * sizeof(double));
        double *e = (double *)malloc((size_t)dv * sizeof(double));
        double *gk = (double *)malloc((size_t)dv * sizeof(double));

        /* forward pass, keeping the state that enters each block */
        double *S = Sb; /* reuse slot 0 as the running state */
        if (S0) memcpy(S, S0 + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(S, 0, ssz * sizeof(double));
        for (int t = 0; t < T; ++t) {
            if (t % ORACLE_CK == 0)
                memcpy(ckpt + (size_t)(t / ORACLE_CK) * ssz, S, ssz * sizeof(double));
            size_t ti = tok_index(b, t, h, T, H);
            gdr_token(dk, dv, S, q + ti * dk, k + ti * dk, v + ti * dv,
                      exp(log_alpha[ti]), beta[ti], r, NULL, 1);
        }

        if (dS_T) memcpy(G, dS_T + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(G, 0, ssz * sizeof(double));

        for (int blk = nblk - 1; blk >= 0; --blk) {
            int t0 = blk * ORACLE_CK;
            int t1 = t0 + ORACLE_CK < T ? t0 + ORACLE_CK : T;
            memcpy(Sb, ckpt + (size_t)blk * ssz, ssz * sizeof(double));
            for (int t = t0; t < t1; ++t) {
                size_t ti = tok_index(b, t, h, T, H);
                double *nxt = Sb + (size_t)(t - t0 + 1) * ssz;
                memcpy(nxt, Sb + (size_t)(t - t0) * ssz, ssz * sizeof(double));
                gdr_token(dk, dv, nxt, q + ti * dk, k + ti * dk, v + ti * dv,
                          exp(log_alpha[ti]), beta[ti], r, NULL, 1);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                size_t ti = tok_index(b, t, h, T, H);
                const double *P = Sb + (size_t)(t - t0) * ssz;
                const double *St = Sb + (size_t)(t - t0 + 1) * ssz;
                const double *qt = q + ti * dk, *kt = k + ti * dk, *vt = v + ti * dv;
                const double *dot = dO + ti * dv;
                double a = exp(log_alpha[ti]), bt = beta[ti];

                /* readout: G += do q^T ; dq = S_t^T do */
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += dot[i] * qt[j];
                for (int j = 0; j < dk; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dv; ++i) acc += St[(size_t)i * dk + j] * dot[i];
                    dq[ti * dk + j] = acc;
                }
                /* r = P k, e = v - a r, gk = G k */
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0, acc2 = 0.0;
                    for (int j = 0; j < dk; ++j) {
                        acc += P[(size_t)i * dk + j] * kt[j];
                        acc2 += G[(size_t)i * dk + j] * kt[j];
                    }
                    r[i] = acc;
                    e[i] = vt[i] - a * acc;
                    gk[i] = acc2;
                }
                double db = 0.0, rgk = 0.0, gp = 0.0;
                for (int i = 0; i < dv; ++i) {
                    dv_out[ti * dv + i] = bt * gk[i];
                    db += e[i] * gk[i];
                    rgk += r[i] * gk[i];
                }
                for (size_t x = 0; x < ssz; ++x) gp += G[x] * P[x];
                dbeta[ti] = db;
                dlog_alpha[ti] = a * (gp - bt * rgk);
                for (int j = 0; j < dk; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dv; ++i)
                        acc += bt * G[(size_t)i * dk + j] * e[i]
                             - a * bt * P[(size_t)i * dk + j] * gk[i];
                    dk_out[ti * dk + j] = acc;
                }
                /* G <- a G - a beta gk k^T */
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j)
                        G[(size_t)i * dk + j] = a * G[(size_t)i * dk + j] - a * bt * gk[i] * kt[j];
            }
        }
        if (dS0) memcpy(dS0 + (size_t)bh * ssz, G, ssz * sizeof(double));
        free(ckpt); free(Sb); free(G); free(r); free(e); free(gk);
    }
}

/*
 * Gated Delta Rule-2 forward ([GDN2]): per token, in this order,
 *   S'  = S_{t-1} Diag(alpha_t)              (decay each key channel j by alpha_t[j])
 *   r   = S' (b_t * k_t)                      (read the old value along b_t*k_t)
 *   S_t = S' - (r - w_t * v_t) k_t^T          (write the residual along k_t)
 *   o_t = S_t q_t
 * alpha_t = exp(log_alpha_t) per key channel, b_t per key channel, w_t per
 * value channel ('*' is the element-wise product).
 */
void oracle_gdr2_fwd(int B, int T, int H, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *log_alpha, const double *bgate,
                     const double *wgate, const double *S0,
                     double *o, double *S_T) {
    long units = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < units; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        size_t ssz = (size_t)dv * dk;
        double *S = (double *)malloc(ssz * sizeof(double));
        double *bk = (double *)malloc((size_t)dk * sizeof(double));
        double *al = (double *)malloc((size_t)dk * sizeof(double));
        if (S0) memcpy(S, S0 + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(S, 0, ssz * sizeof(double));
        for (int t = 0; t < T; ++t) {
            size_t ti = tok_index(b, t, h, T, H);
            const double *qt = q + ti * dk, *kt = k + ti * dk, *vt = v + ti * dv;
            const double *la = log_alpha + ti * dk, *bt = bgate + ti * dk;
            const double *wt = wgate + ti * dv;
            for (int j = 0; j < dk; ++j) { al[j] = exp(la[j]); bk[j] = bt[j] * kt[j]; }
            for (int i = 0; i < dv; ++i) {
                double *row = S + (size_t)i * dk;
                double rd = 0.0;
                for (int j = 0; j < dk; ++j) { row[j] *= al[j]; rd += row[j] * bk[j]; }
                double res = rd - wt[i] * vt[i];
                for (int j = 0; j < dk; ++j) row[j] -= res * kt[j];
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
                o[ti * dv + i] = acc;
            }
        }
        if (S_T) memcpy(S_T + (size_t)bh * ssz, S, ssz * sizeof(double));
        free(S); free(bk); free(al);
    }
}

/* One Gated Delta Rule-2 step on S in place (the update of oracle_gdr2_fwd). */
static void gdr2_token(int dk, int dv, double *S, const double *kt, const double *vt,
                       const double *la, const double *bt, const double *wt) {
    for (int i = 0; i < dv; ++i) {
        double *row = S + (size_t)i * dk;
        double rd = 0.0;
        for (int j = 0; j < dk; ++j) { row[j] *= exp(la[j]); rd += row[j] * bt[j] * kt[j]; }
        double res = rd - wt[i] * vt[i];
        for (int j = 0; j < dk; ++j) row[j] -= res * kt[j];
    }
}

/*
 * Gated Delta Rule-2 backward: reverse mode of the step of oracle_gdr2_fwd
 * (the pages give no backward).  With S = S_{t-1}, P = S Diag(alpha),
 * e = w*v - P(b*k) (so S_t = P + e k^T), and G = dL/dS_t once the readout's
 * do q^T is added:
 *   dq    = S_t^T do                 gk = G k
 *   dv    = w * gk                   dw = v * gk
 *   dk    = G^T e - b * (P^T gk)     db = -k * (P^T gk)
 *   dlog alpha_j = sum_i P_ij (G_ij - gk_i b_j k_j)
 *   dL/dS_{t-1} = (G - gk (b*k)^T) Diag(alpha)
 * The state entering each block of ORACLE_CK tokens is kept from a forward
 * pass and the block's states are recomputed before walking it backwards.
 * Gradient layouts match the inputs; dS_T and dS0 may be NULL.
 */
void oracle_gdr2_bwd(int B, int T, int H, int dk, int dv,
                     const double *q, const double *k, const double *v,
                     const double *log_alpha, const double *bgate, const double *wgate,
                     const double *S0, const double *dO, const double *dS_T,
                     double *dq, double *dk_out, double *dv_out,
                     double *dlog_alpha, double *db_out, double *dw_out, double *dS0) {
    long units = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < units; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        size_t ssz = (size_t)dv * dk;
        int nblk = (T + ORACLE_CK - 1) / ORACLE_CK;
        double *ckpt = (double *)malloc((size_t)(nblk > 0 ? nblk : 1) * ssz * sizeof(double));
        double *Sb = (double *)malloc((size_t)(ORACLE_CK + 1) * ssz * sizeof(double));
        double *G = (double *)malloc(ssz * sizeof(double));
        double *P = (double *)malloc(ssz * sizeof(double));
        double *e = (double *)malloc((size_t)dv * sizeof(double));
        double *gk = (double *)malloc((size_t)dv * sizeof(double));
        double *bk = (double *)malloc((size_t)dk * sizeof(double));
        double *al = (double *)malloc((size_t)dk * sizeof(double));

        double *S = Sb;
        if (S0) memcpy(S, S0 + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(S, 0, ssz * sizeof(double));
        for (int t = 0; t < T; ++t) {
            if (t % ORACLE_CK == 0)
                memcpy(ckpt + (size_t)(t / ORACLE_CK) * ssz, S, ssz * sizeof(double));
            size_t ti = tok_index(b, t, h, T, H);
            gdr2_token(dk, dv, S, k + ti * dk, v + ti * dv, log_alpha + ti * dk, bgate + ti * dk,
                       wgate + ti * dv);
        }

        if (dS_T) memcpy(G, dS_T + (size_t)bh * ssz, ssz * sizeof(double));
        else memset(G, 0, ssz * sizeof(double));

        for (int blk = nblk - 1; blk >= 0; --blk) {
            int t0 = blk * ORACLE_CK;
            int t1 = t0 + ORACLE_CK < T ? t0 + ORACLE_CK : T;
            memcpy(Sb, ckpt + (size_t)blk * ssz, ssz * sizeof(double));
            for (int t = t0; t < t1; ++t) {
                size_t ti = tok_index(b, t, h, T, H);
                double *nxt = Sb + (size_t)(t - t0 + 1) * ssz;
                memcpy(nxt, Sb + (size_t)(t - t0) * ssz, ssz * sizeof(double));
                gdr2_token(dk, dv, nxt, k + ti * dk, v + ti * dv, log_alpha + ti * dk, bgate + ti * dk,
                           wgate + ti * dv);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                size_t ti = tok_index(b, t, h, T, H);
                const double *Sp = Sb + (size_t)(t - t0) * ssz;      /* S_{t-1} */
                const double *St = Sb + (size_t)(t - t0 + 1) * ssz;  /* S_t */
                const double *qt = q + ti * dk, *kt = k + ti * dk, *vt = v + ti * dv;
                const double *la = log_alpha + ti * dk, *bt = bgate + ti * dk, *wt = wgate + ti * dv;
                const double *dot = dO + ti * dv;
                for (int j = 0; j < dk; ++j) { al[j] = exp(la[j]); bk[j] = bt[j] * kt[j]; }
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) P[(size_t)i * dk + j] = Sp[(size_t)i * dk + j] * al[j];

                /* readout: G += do q^T ; dq = S_t^T do */
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += dot[i] * qt[j];
                for (int j = 0; j < dk; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dv; ++i) acc += St[(size_t)i * dk + j] * dot[i];
                    dq[ti * dk + j] = acc;
                }
                /* e = w*v - P(b*k), gk = G k; dv, dw */
                for (int i = 0; i < dv; ++i) {
                    double rd = 0.0, g = 0.0;
                    for (int j = 0; j < dk; ++j) {
                        rd += P[(size_t)i * dk + j] * bk[j];
                        g += G[(size_t)i * dk + j] * kt[j];
                    }
                    e[i] = wt[i] * vt[i] - rd;
                    gk[i] = g;
                    dv_out[ti * dv + i] = wt[i] * g;
                    dw_out[ti * dv + i] = vt[i] * g;
                }
                /* dk, db, dlog alpha (column sums over the value channels) */
                for (int j = 0; j < dk; ++j) {
                    double ge = 0.0, pg = 0.0, da = 0.0;
                    for (int i = 0; i < dv; ++i) {
                        double pij = P[(size_t)i * dk + j], gij = G[(size_t)i * dk + j];
                        ge += gij * e[i];
                        pg += pij * gk[i];
                        da += pij * (gij - gk[i] * bk[j]);
                    }
                    dk_out[ti * dk + j] = ge - bt[j] * pg;
                    db_out[ti * dk + j] = -kt[j] * pg;
                    dlog_alpha[ti * dk + j] = da;
                }
                /* dL/dS_{t-1} = (G - gk (b*k)^T) Diag(alpha) */
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j)
                        G[(size_t)i * dk + j] = (G[(size_t)i * dk + j] - gk[i] * bk[j]) * al[j];
            }
        }
        if (dS0) memcpy(dS0 + (size_t)bh * ssz, G, ssz * sizeof(double));
        free(ckpt); free(Sb); free(G); free(P); free(e); free(gk); free(bk); free(al);
    }
}
