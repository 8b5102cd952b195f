/*
 * block_oracle.c -- plain fp64 CPU oracle for the pre- and post-processing
 * around the gated delta rule in a Gated DeltaNet block.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library.  It shares no code with the
 * CUDA library and the product path never calls it.
 *
 * Sources (cited by page title and section):
 *   [GDN-R]  "[논문리뷰] Gated Delta Netoworks: Improving MAMBA2 with Delta Rule
 *            (ICLR, 2025)", meaningful96.github.io/nr/GDN
 *            -- section 3.8 "Gated DeltaNet Block": q and k go Linear ->
 *               ShortConv -> SiLU -> L2 normalisation, v goes Linear ->
 *               ShortConv -> SiLU; after the recurrence the output is
 *               normalised, gated and projected.  Section 1 repeats the q/k/v
 *               path (short convolution, SiLU, L2 on q and k).
 *   [GDN2]   "Gated DeltaNet-2: Decoupling Erase and Write in Linear
 *            Attention", agihunt.info/papers/2605.22791, the paragraph on the
 *            block design: short convolution with SiLU, L2 normalisation of q
 *            and k, and RMSNorm followed by a SiLU output gate on the
 *            recurrent output.
 *
 * The pages name the steps but fix no widths, weights or epsilons.  Readings
 * used here (the plainest ones the pages support):
 *   * ShortConv is a depthwise causal 1-D convolution along time of width K,
 *     one filter per channel, in the cross-correlation convention of a
 *     framework Conv1d: y[t,c] = bias[c] + sum_{j<K} w[c,j] x[t-K+1+j, c].
 *     Tokens before the first are taken from a carried conv state (the last
 *     K-1 inputs of the previous segment) or are zero.
 *   * SiLU(z) = z / (1 + exp(-z)).
 *   * L2 normalisation acts per (token, head) over the head's d channels:
 *     y / sqrt(sum y^2 + eps).  eps = 0 is the plain definition.
 *   * The output norm is RMSNorm per (token, head) over dv channels with a
 *     per-channel weight shared by all heads, y = o / sqrt(mean o^2 + eps) *
 *     weight, and the output gate multiplies by SiLU(g), g being the gate
 *     projection of the block input, [B, T, H, dv].
 *   * The Linear projections themselves are plain matrix products and are
 *     not part of this file.
 *
 * Layouts (row-major, all double):
 *   x, y          [B, T, H, d]
 *   w             [H*d, K]         bias  [H*d] (may be NULL)
 *   state_in/out  [B, K-1, H*d]    (may be NULL: zeros in / not written)
 *   o, g, y       [B, T, H, dv]    weight [dv]     (g may be NULL: no gate)
 *
 * Parity status: pinned by tests/test_oracle_block_pins.py (numpy convolution
 * of the zero-state case, impulse response, state continuity across a split,
 * unit norm, closed forms of SiLU and RMSNorm; the reverse modes by central
 * differences of the forward functions and by their invariants).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ShortConv -> SiLU -> (L2) for one projected stream ([GDN-R] section 3.8). */
void oracle_short_conv(int B, int T, int H, int d, int K, const double *x,
                       const double *w, const double *bias,
                       const double *state_in, int l2, double eps, double *y,
                       double *state_out) {
    const int C = H * d;
    for (int b = 0; b < B; ++b) {
        const double *xb = x + (size_t)b * T * C;
        const double *sb = state_in ? state_in + (size_t)b * (K - 1) * C : NULL;
        double *yb = y + (size_t)b * T * C;
        for (int t = 0; t < T; ++t) {
            for (int c = 0; c < C; ++c) {
                double acc = bias ? bias[c] : 0.0;
                for (int j = 0; j < K; ++j) {
                    int s = t - (K - 1) + j; /* source token */
                    double xv;
                    if (s >= 0)
                        xv = xb[(size_t)s * C + c];
                    else
                        xv = sb ? sb[(size_t)(K - 1 + s) * C + c] : 0.0;
                    acc += w[(size_t)c * K + j] * xv;
                }
                yb[(size_t)t * C + c] = silu(acc);
            }
            if (l2) {
                for (int h = 0; h < H; ++h) {
                    double *r = yb + (size_t)t * C + (size_t)h * d;
                    double ss = 0.0;
                    for (int i = 0; i < d; ++i) ss += r[i] * r[i];
                    double inv = 1.0 / sqrt(ss + eps);
                    for (int i = 0; i < d; ++i) r[i] *= inv;
                }
            }
        }
        /* the carried state: the last K-1 inputs of (state_in, x) */
        if (state_out) {
            double *ob = state_out + (size_t)b * (K - 1) * C;
            for (int j = 0; j < K - 1; ++j) {
                int s = T - (K - 1) + j;
                for (int c = 0; c < C; ++c) {
                    double xv;
                    if (s >= 0)
                        xv = xb[(size_t)s * C + c];
                    else
                        xv = sb ? sb[(size_t)(K - 1 + s) * C + c] : 0.0;
                    ob[(size_t)j * C + c] = xv;
                }
            }
        }
    }
}

/* RMSNorm of the recurrent output, then the SiLU output gate ([GDN2] block
 * paragraph; [GDN-R] section 3.8). */
void oracle_rmsnorm_gate(int B, int T, int H, int dv, const double *o,
                         const double *g, const double *weight, double eps,
                         double *y) {
    size_t rows = (size_t)B * T * H;
    for (size_t r = 0; r < rows; ++r) {
        const double *orow = o + r * dv;
        double ms = 0.0;
        for (int i = 0; i < dv; ++i) ms += orow[i] * orow[i];
        ms /= dv;
        double inv = 1.0 / sqrt(ms + eps);
        for (int i = 0; i < dv; ++i) {
            double gate = g ? silu(g[r * dv + i]) : 1.0;
            y[r * dv + i] = orow[i] * inv * weight[i] * gate;
        }
    }
}

/* Reverse mode of oracle_rmsnorm_gate (the chain rule of the epilogue's
 * definition above): with r = 1/sqrt(mean o^2 + eps), a = o r, s = SiLU(g)
 * (s = 1 without a gate) and y = a * weight * s,
 *     dg = dy a weight SiLU'(g),   SiLU'(z) = sigma(z) (1 + z (1 - sigma(z)))
 *     da = dy weight s,            do = r (da - a mean(da a))
 *     dweight = sum over rows of dy a s.
 * dg may be NULL (no gate); every output is overwritten. */
void oracle_rmsnorm_gate_bwd(int B, int T, int H, int dv, const double *o,
                             const double *g, const double *weight, double eps,
                             const double *dy, double *dO, double *dg,
                             double *dweight) {
    size_t rows = (size_t)B * T * H;
    for (int i = 0; i < dv; ++i) dweight[i] = 0.0;
    for (size_t r = 0; r < rows; ++r) {
        const double *orow = o + r * dv, *dyr = dy + r * dv;
        double ms = 0.0;
        for (int i = 0; i < dv; ++i) ms += orow[i] * orow[i];
        ms /= dv;
        const double inv = 1.0 / sqrt(ms + eps);
        double dot = 0.0; /* sum_i da_i a_i */
        for (int i = 0; i < dv; ++i) {
            const double a = orow[i] * inv;
            double s = 1.0;
            if (g) {
                const double z = g[r * dv + i];
                const double sig = 1.0 / (1.0 + exp(-z));
                s = z * sig;
                dg[r * dv + i] = dyr[i] * a * weight[i] * sig * (1.0 + z * (1.0 - sig));
            }
            const double da = dyr[i] * weight[i] * s;
            dot += da * a;
            dweight[i] += dyr[i] * a * s;
        }
        dot /= dv;
        for (int i = 0; i < dv; ++i) {
            const double a = orow[i] * inv;
            double s = 1.0;
            if (g) {
                const double z = g[r * dv + i];
                s = z / (1.0 + exp(-z));
            }
            const double da = dyr[i] * weight[i] * s;
            dO[r * dv + i] = inv * (da - a * dot);
        }
    }
}

/* Reverse mode of oracle_short_conv for an incoming dy [B,T,H,d] (and, if
 * not NULL, dstate_out [B,K-1,H*d], the gradient of the returned state).
 * Steps, each the chain rule of one forward step:
 *   z = conv(x), u = SiLU(z), y = u / n with n = sqrt(sum_head u^2 + eps)
 *   du = (dy - y (y . dy)) / n          (l2; du = dy without it)
 *   dz = du sig(z) (1 + z (1 - sig(z)))
 *   dx[s] = sum_j w[j] dz[s + K-1-j]    (+ dstate_out where x[s] was carried)
 *   dw[c,j] = sum_t dz[t,c] x[t-K+1+j, c],  dbias[c] = sum_t dz[t,c]
 * Tokens s < 0 are the carried state: their dx goes to dstate_in.
 * Outputs dx [B,T,H,d], dw [H*d,K] and dbias [H*d] (may be NULL) are
 * overwritten; dstate_in [B,K-1,H*d] is written if not NULL. */
void oracle_short_conv_bwd(int B, int T, int H, int d, int K, const double *x,
                           const double *w, const double *bias,
                           const double *state_in, int l2, double eps,
                           const double *dy, const double *dstate_out,
                           double *dx, double *dw, double *dbias,
                           double *dstate_in) {
    const int C = H * d;
    double *dz = (double *)malloc(sizeof(double) * ((size_t)T * C + 1));
    double *ub = (double *)malloc(sizeof(double) * ((size_t)C + 1));
    double *zb = (double *)malloc(sizeof(double) * ((size_t)C + 1));
    for (int i = 0; i < C * K; ++i) dw[i] = 0.0;
    if (dbias)
        for (int c = 0; c < C; ++c) dbias[c] = 0.0;
    for (int b = 0; b < B; ++b) {
        const double *xb = x + (size_t)b * T * C;
        const double *sb = state_in ? state_in + (size_t)b * (K - 1) * C : NULL;
        const double *dyb = dy + (size_t)b * T * C;
        /* x at token s (s < 0: carried state or zero) */
#define XAT(s, c) ((s) >= 0 ? xb[(size_t)(s) * C + (c)] : (sb ? sb[(size_t)(K - 1 + (s)) * C + (c)] : 0.0))
        for (int t = 0; t < T; ++t) {
            for (int c = 0; c < C; ++c) {
                double acc = bias ? bias[c] : 0.0;
                for (int j = 0; j < K; ++j) acc += w[(size_t)c * K + j] * XAT(t - (K - 1) + j, c);
                zb[c] = acc;
                ub[c] = silu(acc);
            }
            for (int h = 0; h < H; ++h) {
                const double *u = ub + (size_t)h * d, *g = dyb + (size_t)t * C + (size_t)h * d;
                double *dzr = dz + (size_t)t * C + (size_t)h * d;
                double n = 1.0, dot = 0.0;
                if (l2) {
                    double ss = 0.0;
                    for (int i = 0; i < d; ++i) ss += u[i] * u[i];
                    n = sqrt(ss + eps);
                    for (int i = 0; i < d; ++i) dot += (u[i] / n) * g[i];
                }
                for (int i = 0; i < d; ++i) {
                    const double du = l2 ? (g[i] - (u[i] / n) * dot) / n : g[i];
                    const double z = zb[(size_t)h * d + i];
                    const double sig = 1.0 / (1.0 + exp(-z));
                    dzr[i] = du * sig * (1.0 + z * (1.0 - sig));
                }
            }
        }
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < C; ++c) {
                const double g = dz[(size_t)t * C + c];
                for (int j = 0; j < K; ++j) dw[(size_t)c * K + j] += g * XAT(t - (K - 1) + j, c);
                if (dbias) dbias[c] += g;
            }
#undef XAT
        /* dx[s] for s in [-(K-1), T): conv transpose plus the state gradient */
        for (int s = -(K - 1); s < T; ++s) {
            if (s < 0 && !dstate_in) continue;
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int j = 0; j < K; ++j) {
                    const int t = s + (K - 1) - j; /* output token that read x[s] via tap j */
                    if (t >= 0 && t < T) acc += w[(size_t)c * K + j] * dz[(size_t)t * C + c];
                }
                const int m = s - (T - (K - 1)); /* slot of x[s] in the returned state */
                if (dstate_out && m >= 0) acc += dstate_out[((size_t)b * (K - 1) + m) * C + c];
                if (s >= 0)
                    dx[((size_t)b * T + s) * C + c] = acc;
                else
                    dstate_in[((size_t)b * (K - 1) + (K - 1 + s)) * C + c] = acc;
            }
        }
    }
    free(dz);
    free(ub);
    free(zb);
}
