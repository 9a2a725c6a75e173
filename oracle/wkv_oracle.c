/*
 * fp64 CPU oracle for RWKV's WKV time-mixing operator.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg do. It
 * shares no code, header or constant with the CUDA library.
 *
 * It is written to be checked by eye against the pages, not to be fast: no blocking,
 * no stabilisation, no reordering. Everything is double precision; exponents are formed
 * as sums first and exponentiated afterwards.
 *
 * Sources (page title, then section):
 *   [concept]  "RWKV（Receptance Weighted Key Value）概念" (compassingai.com),
 *              section 3.2 "时间混合（Time-mixing）与 WKV 算子": the wkv_t equation and
 *              out_t = sigmoid(receptance_t) * wkv_t.
 *   [notes]    "RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型" (papernotes,
 *              2023_rwkv): "一句话总结" (the recurrence a_t, b_t and the output that uses
 *              a_{t-1}, b_{t-1}), "关键设计 2：WKV 算子" (parallel form and RNN cell),
 *              "关键设计 4：双执行模式" (single-token inference step).
 *
 * Layout: k, v, r, y, dy, dk, dv, dr are (B, T, C) row-major (C fastest); w, u, dw, du
 * are [C]. Time is 0-based here; the pages' t is our t + 1. All functions return 0, or
 * -1 on a NULL required pointer / negative size / allocation failure.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#define AT(b, t, c) ((((int64_t)(b)) * T + (t)) * C + (c))

static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * O1: the parallel (summation) form, O(T^2) per channel.
 * [concept] 3.2 and [notes] "关键设计 2": for 1-based t,
 *   wkv_t = (sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u + k_t} v_t)
 *         / (sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u + k_t})
 *   y_t   = sigmoid(r_t) * wkv_t            (r == NULL: y_t = wkv_t, no gate)
 * Optional initial state (A0, B0) [B*C]: the true numerator and denominator of the past
 * before the first token; it enters token t (0-based) decayed by e^{-t w}, the same
 * weight the recurrence gives it. NULL means no past.
 */
int oracle_wkv_direct(int64_t B, int64_t T, int64_t C, const double *w, const double *u,
                      const double *k, const double *v, const double *r, double *y,
                      const double *A0, const double *B0)
{
    if (B < 0 || T < 0 || C < 0 || !w || !u || !k || !v || !y) return -1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c)
            for (int64_t t = 0; t < T; ++t) {
                double num = 0.0, den = 0.0;
                if (A0 && B0) {
                    double e = exp(-(double)t * w[c]);
                    num += e * A0[b * C + c];
                    den += e * B0[b * C + c];
                }
                for (int64_t i = 0; i < t; ++i) {
                    double e = exp(-(double)(t - 1 - i) * w[c] + k[AT(b, i, c)]);
                    num += e * v[AT(b, i, c)];
                    den += e;
                }
                double e = exp(u[c] + k[AT(b, t, c)]);
                num += e * v[AT(b, t, c)];
                den += e;
                double wkv = num / den;
                y[AT(b, t, c)] = r ? sigm(r[AT(b, t, c)]) * wkv : wkv;
            }
    return 0;
}

/*
 * O2: the recurrent form, unstabilised.
 * [notes] "一句话总结": a_t = e^{-w} a_{t-1} + e^{k_t} v_t, b_t = e^{-w} b_{t-1} + e^{k_t},
 * and the output at t uses the state before the token:
 *   wkv_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}).
 * State in (A0, B0) and out (A1, B1) are the true (unscaled) numerator and denominator,
 * [B*C] each; NULL in means a_0 = b_0 = 0, NULL out means not wanted.
 */
int oracle_wkv_recurrent(int64_t B, int64_t T, int64_t C, const double *w, const double *u,
                         const double *k, const double *v, const double *r, double *y,
                         const double *A0, const double *B0, double *A1, double *B1)
{
    if (B < 0 || T < 0 || C < 0 || !w || !u || !k || !v || !y) return -1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c) {
            double a = (A0 && B0) ? A0[b * C + c] : 0.0;
            double d = (A0 && B0) ? B0[b * C + c] : 0.0;
            double decay = exp(-w[c]);
            for (int64_t t = 0; t < T; ++t) {
                double kt = k[AT(b, t, c)], vt = v[AT(b, t, c)];
                double cur = exp(u[c] + kt);
                double wkv = (a + cur * vt) / (d + cur);
                y[AT(b, t, c)] = r ? sigm(r[AT(b, t, c)]) * wkv : wkv;
                double ek = exp(kt);
                a = decay * a + ek * vt;
                d = decay * d + ek;
            }
            if (A1) A1[b * C + c] = a;
            if (B1) B1[b * C + c] = d;
        }
    return 0;
}

/*
 * Single-token step for N sequences x L layers, state updated in place.
 * [notes] "关键设计 4" (inference keeps only the numerator/denominator state and updates
 * it once per token) with the WKV lines of "一句话总结". Layer l of sequence n uses
 * w[l*C + c], u[l*C + c]. k, v, r, y, A, Bd are [N, L, C]; A, Bd are true (unscaled).
 */
int oracle_wkv_decode(int64_t N, int64_t L, int64_t C, const double *w, const double *u,
                      const double *k, const double *v, const double *r, double *y,
                      double *A, double *Bd)
{
    if (N < 0 || L < 0 || C < 0 || !w || !u || !k || !v || !y || !A || !Bd) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t l = 0; l < L; ++l)
            for (int64_t c = 0; c < C; ++c) {
                int64_t s = (n * L + l) * C + c, p = l * C + c;
                double cur = exp(u[p] + k[s]);
                double wkv = (A[s] + cur * v[s]) / (Bd[s] + cur);
                y[s] = r ? sigm(r[s]) * wkv : wkv;
                double ek = exp(k[s]);
                A[s] = exp(-w[p]) * A[s] + ek * v[s];
                Bd[s] = exp(-w[p]) * Bd[s] + ek;
            }
    return 0;
}

/*
 * O4: gradients of L = sum_t dy_t . y_t with respect to k, v, w, u (and r), analytic.
 * The pages say only that the operator supports ordinary backpropagation; the formulas
 * below are derived from the parallel form of [concept] 3.2 by the chain rule.
 * With N_t, D_t the numerator and denominator of wkv_t, g_t = dy_t sigmoid(r_t) and
 * h_t = g_t / D_t (0-based, sums over t > i):
 *   beta_i   = sum h_t e^{-(t-1-i)w},          gamma_i   = sum h_t wkv_t e^{-(t-1-i)w}
 *   betad_i  = sum (t-1-i) h_t e^{-(t-1-i)w},  gammad_i  = sum (t-1-i) h_t wkv_t e^{-(t-1-i)w}
 *   dv_i = e^{k_i} (h_i e^u + beta_i)
 *   dk_i = e^{k_i} (h_i e^u (v_i - wkv_i) + v_i beta_i - gamma_i)
 *   dw   = -sum_{b,i} e^{k_i} (v_i betad_i - gammad_i)      (w is the positive decay rate)
 *   du   =  sum_{b,t} h_t e^{u+k_t} (v_t - wkv_t)
 *   dr_t = dy_t wkv_t sigmoid(r_t) (1 - sigmoid(r_t))
 * computed by the reverse recurrences beta_{i-1} = h_i + e^{-w} beta_i and
 * betad_{i-1} = e^{-w} (betad_i + beta_i) (and the same for gamma).
 * r == NULL: no gate (g_t = dy_t) and dr is not written. dr may be NULL.
 * dw, du [C] are overwritten with the sums over b and t. dw_abs, du_abs [C] (may be NULL)
 * receive the scale against which a float computation of them is judged: the sums of the
 * absolute values of the terms of their full expansion,
 *   dw = -sum_{i<t} (t-1-i) e^{k_i-(t-1-i)w} h_t v_i + sum_{i<t} (t-1-i) e^{k_i-(t-1-i)w} h_t wkv_t,
 *   du =  sum_t h_t e^{u+k_t} v_t - sum_t h_t e^{u+k_t} wkv_t,
 * accumulated by the same recurrences run on |h_t|, |v_i|, |wkv_t|.
 * dk_abs, dv_abs (B, T, C) (may be NULL) do the same for dk and dv, which are sums over
 * the tokens t >= i that token i reaches:
 *   dv_i = e^{k_i} h_i e^u + sum_{t>i} e^{k_i-(t-1-i)w} h_t,
 *   dk_i = e^{k_i} h_i e^u v_i - e^{k_i} h_i e^u wkv_i
 *        + sum_{t>i} e^{k_i-(t-1-i)w} h_t v_i - sum_{t>i} e^{k_i-(t-1-i)w} h_t wkv_t,
 * so dv_abs_i = e^{k_i} (|h_i| e^u + sum |h_t| e^{-(t-1-i)w}) and dk_abs_i the same with
 * (|v_i| + |wkv_t|) in each term: where the terms cancel, a float evaluation still
 * rounds at their size.
 */
int oracle_wkv_backward(int64_t B, int64_t T, int64_t C, const double *w, const double *u,
                        const double *k, const double *v, const double *r, const double *dy,
                        double *dk, double *dv, double *dw, double *du, double *dr,
                        double *dw_abs, double *du_abs, double *dk_abs, double *dv_abs)
{
    if (B < 0 || T < 0 || C < 0 || !w || !u || !k || !v || !dy || !dk || !dv || !dw || !du)
        return -1;
    double *wkv = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *D = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!wkv || !D) { free(wkv); free(D); return -1; }
    for (int64_t c = 0; c < C; ++c) {
        dw[c] = 0.0;
        du[c] = 0.0;
        if (dw_abs) dw_abs[c] = 0.0;
        if (du_abs) du_abs[c] = 0.0;
    }
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c) {
            double decay = exp(-w[c]), eu = exp(u[c]);
            double a = 0.0, d = 0.0;
            for (int64_t t = 0; t < T; ++t) {                /* forward, as O2 */
                double kt = k[AT(b, t, c)], vt = v[AT(b, t, c)];
                double cur = exp(u[c] + kt);
                D[t] = d + cur;
                wkv[t] = (a + cur * vt) / D[t];
                double ek = exp(kt);
                a = decay * a + ek * vt;
                d = decay * d + ek;
            }
            double beta = 0.0, gamma = 0.0, betad = 0.0, gammad = 0.0;
            double abeta = 0.0, agamma = 0.0, abetad = 0.0, agammad = 0.0;
            double dwc = 0.0, duc = 0.0, dwa = 0.0, dua = 0.0;
            for (int64_t i = T - 1; i >= 0; --i) {           /* reverse */
                double ki = k[AT(b, i, c)], vi = v[AT(b, i, c)], dyi = dy[AT(b, i, c)];
                double s = r ? sigm(r[AT(b, i, c)]) : 1.0;
                double h = dyi * s / D[i];
                double ek = exp(ki);
                dv[AT(b, i, c)] = ek * (h * eu + beta);
                dk[AT(b, i, c)] = ek * (h * eu * (vi - wkv[i]) + vi * beta - gamma);
                if (dv_abs) dv_abs[AT(b, i, c)] = ek * (fabs(h) * eu + abeta);
                if (dk_abs)
                    dk_abs[AT(b, i, c)] = ek * (fabs(h) * eu * (fabs(vi) + fabs(wkv[i]))
                                                + fabs(vi) * abeta + agamma);
                dwc += -ek * (vi * betad - gammad);
                duc += h * eu * ek * (vi - wkv[i]);
                dwa += ek * (fabs(vi) * abetad + agammad);
                dua += fabs(h) * eu * ek * (fabs(vi) + fabs(wkv[i]));
                if (r && dr) dr[AT(b, i, c)] = dyi * wkv[i] * s * (1.0 - s);
                betad = decay * (betad + beta);
                gammad = decay * (gammad + gamma);
                beta = h + decay * beta;
                gamma = h * wkv[i] + decay * gamma;
                abetad = decay * (abetad + abeta);
                agammad = decay * (agammad + agamma);
                abeta = fabs(h) + decay * abeta;
                agamma = fabs(h * wkv[i]) + decay * agamma;
            }
            dw[c] += dwc;
            du[c] += duc;
            if (dw_abs) dw_abs[c] += dwa;
            if (du_abs) du_abs[c] += dua;
        }
    free(wkv);
    free(D);
    return 0;
}

/*
 * O5: gradients of the stateful forward (the backward through a state that enters and
 * leaves, as when a long sequence is trained in consecutive pieces), by reverse-mode
 * differentiation of the recurrence of [notes] "一句话总结" / "关键设计 2", written as
 * its adjoint step by step. For 0-based t, with (A_{-1}, B_{-1}) = (A0, B0):
 *   D_t   = B_{t-1} + e^{u+k_t},   wkv_t = (A_{t-1} + e^{u+k_t} v_t) / D_t,
 *   y_t   = sigmoid(r_t) wkv_t,
 *   A_t   = e^{-w} A_{t-1} + e^{k_t} v_t,   B_t = e^{-w} B_{t-1} + e^{k_t},
 * and the loss L = sum_t dy_t y_t + gA A_{T-1} + gB B_{T-1} (gA, gB: the gradients of a
 * later loss with respect to the final numerator and denominator). The adjoints
 * Abar_t = dL/dA_t, Bbar_t = dL/dB_t run backward from (gA, gB):
 *   g_t = dy_t sigmoid(r_t),
 *   Abar_{t-1} = e^{-w} Abar_t + g_t / D_t,
 *   Bbar_{t-1} = e^{-w} Bbar_t - g_t wkv_t / D_t,
 *   dv_t = e^{k_t} Abar_t + g_t e^{u+k_t} / D_t,
 *   dk_t = e^{k_t} (v_t Abar_t + Bbar_t) + g_t e^{u+k_t} (v_t - wkv_t) / D_t,
 *   dw  -= e^{-w} (A_{t-1} Abar_t + B_{t-1} Bbar_t),
 *   du  += g_t e^{u+k_t} (v_t - wkv_t) / D_t,
 *   dr_t = dy_t wkv_t sigmoid(r_t) (1 - sigmoid(r_t)),
 * and finally dA0 = Abar_{-1}, dB0 = Bbar_{-1}.
 * A0, B0, gA, gB, dA0, dB0 are [B*C] and may be NULL (zero state / zero gradient / not
 * wanted). dw_abs, du_abs, dA0_abs, dB0_abs, dk_abs, dv_abs (may be NULL) receive the
 * same sums run on absolute values (|v|, |g|, |wkv|, |A0|, |gA|, |gB| in place of v, g,
 * wkv, A0, gA, gB; dk_abs and dv_abs are (B, T, C) like dk and dv): the scale against
 * which a float evaluation of these sums is judged.
 */
int oracle_wkv_backward_state(int64_t B, int64_t T, int64_t C, const double *w,
                              const double *u, const double *k, const double *v,
                              const double *r, const double *dy, const double *A0,
                              const double *B0, const double *gA, const double *gB,
                              double *dk, double *dv, double *dw, double *du, double *dr,
                              double *dA0, double *dB0, double *dw_abs, double *du_abs,
                              double *dA0_abs, double *dB0_abs, double *dk_abs,
                              double *dv_abs)
{
    if (B < 0 || T < 0 || C < 0 || !w || !u || !dw || !du) return -1;
    if (T > 0 && (!k || !v || !dy || !dk || !dv)) return -1;
    size_t n = (size_t)(T > 0 ? T : 1) + 1;
    /* Aprev[t] = A_{t-1} (index 0 holds the initial state), likewise the others */
    double *Aprev = (double *)malloc(sizeof(double) * n);
    double *Bprev = (double *)malloc(sizeof(double) * n);
    double *Aabs = (double *)malloc(sizeof(double) * n);
    double *D = (double *)malloc(sizeof(double) * n);
    double *wkv = (double *)malloc(sizeof(double) * n);
    if (!Aprev || !Bprev || !Aabs || !D || !wkv) {
        free(Aprev); free(Bprev); free(Aabs); free(D); free(wkv);
        return -1;
    }
    for (int64_t c = 0; c < C; ++c) {
        dw[c] = 0.0;
        du[c] = 0.0;
        if (dw_abs) dw_abs[c] = 0.0;
        if (du_abs) du_abs[c] = 0.0;
    }
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c) {
            const int64_t sc = b * C + c;
            const double keep = exp(-w[c]);
            double A = A0 ? A0[sc] : 0.0, Bd = B0 ? B0[sc] : 0.0, Aa = fabs(A);
            for (int64_t t = 0; t < T; ++t) {                /* forward, keeping the past */
                double kt = k[AT(b, t, c)], vt = v[AT(b, t, c)];
                double bonus = exp(u[c] + kt);
                Aprev[t] = A;
                Bprev[t] = Bd;
                Aabs[t] = Aa;
                D[t] = Bd + bonus;
                wkv[t] = (A + bonus * vt) / D[t];
                A = keep * A + exp(kt) * vt;
                Bd = keep * Bd + exp(kt);
                Aa = keep * Aa + exp(kt) * fabs(vt);
            }
            double Abar = gA ? gA[sc] : 0.0, Bbar = gB ? gB[sc] : 0.0;
            double Abar_a = fabs(Abar), Bbar_a = fabs(Bbar);
            double dwc = 0.0, duc = 0.0, dwa = 0.0, dua = 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {           /* adjoint, last token first */
                double kt = k[AT(b, t, c)], vt = v[AT(b, t, c)], dyt = dy[AT(b, t, c)];
                double s = r ? sigm(r[AT(b, t, c)]) : 1.0;
                double g = dyt * s;
                double ek = exp(kt), bonus = exp(u[c] + kt);
                /* Abar, Bbar here are dL/dA_t, dL/dB_t (this token's update feeds them) */
                dv[AT(b, t, c)] = ek * Abar + g * bonus / D[t];
                dk[AT(b, t, c)] = ek * (vt * Abar + Bbar) + g * bonus * (vt - wkv[t]) / D[t];
                if (dv_abs) dv_abs[AT(b, t, c)] = ek * Abar_a + fabs(g) * bonus / D[t];
                if (dk_abs)
                    dk_abs[AT(b, t, c)] = ek * (fabs(vt) * Abar_a + Bbar_a)
                                        + fabs(g) * bonus * (fabs(vt) + fabs(wkv[t])) / D[t];
                dwc -= keep * (Aprev[t] * Abar + Bprev[t] * Bbar);
                duc += g * bonus * (vt - wkv[t]) / D[t];
                dwa += keep * (Aabs[t] * Abar_a + Bprev[t] * Bbar_a);
                dua += fabs(g) * bonus * (fabs(vt) + fabs(wkv[t])) / D[t];
                if (r && dr) dr[AT(b, t, c)] = dyt * wkv[t] * s * (1.0 - s);
                /* then step to dL/dA_{t-1}, dL/dB_{t-1} */
                Abar = keep * Abar + g / D[t];
                Bbar = keep * Bbar - g * wkv[t] / D[t];
                Abar_a = keep * Abar_a + fabs(g) / D[t];
                Bbar_a = keep * Bbar_a + fabs(g * wkv[t]) / D[t];
            }
            if (dA0) dA0[sc] = Abar;
            if (dB0) dB0[sc] = Bbar;
            if (dA0_abs) dA0_abs[sc] = Abar_a;
            if (dB0_abs) dB0_abs[sc] = Bbar_a;
            dw[c] += dwc;
            du[c] += duc;
            if (dw_abs) dw_abs[c] += dwa;
            if (du_abs) du_abs[c] += dua;
        }
    free(Aprev); free(Bprev); free(Aabs); free(D); free(wkv);
    return 0;
}

/*
 * O6: RWKV-7's generalised-delta-rule state update, per head, as written in the research
 * report "RWKV模型深度研究报告（截至2026年初）", section 1.3.3 "RWKV-7 (Goose)":
 *   S_t = S_{t-1} (diag(w_t) + a_t^T b_t) + v_t^T k_t
 * with row vectors w_t (the decay, per key channel), a_t, b_t, k_t, v_t of the head size N,
 * so S is N x N (row i: value channel, column j: key channel):
 *   S_t[i][j] = S_{t-1}[i][j] w_t[j] + (sum_l S_{t-1}[i][l] a_t[l]) b_t[j] + v_t[i] k_t[j].
 * The report gives no read-out; the reading used is the linear-attention one with the
 * receptance as the query: y_t = S_t r_t^T, y_t[i] = sum_j S_t[i][j] r_t[j].
 * Layout: r, w, k, v, a, b, y are (B, T, H, N) row-major; the state S0 (may be NULL =
 * zero) and S1 (may be NULL = not wanted) are (B, H, N, N) with S[i][j] at i * N + j.
 */
int oracle_wkv7_recurrent(int64_t B, int64_t T, int64_t H, int64_t N, const double *r,
                          const double *w, const double *k, const double *v, const double *a,
                          const double *b, double *y, const double *S0, double *S1)
{
    if (B < 0 || T < 0 || H < 0 || N < 0) return -1;
    if (T > 0 && (!r || !w || !k || !v || !a || !b || !y)) return -1;
    double *S = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N * N : 1));
    double *sa = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    if (!S || !sa) { free(S); free(sa); return -1; }
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t h = 0; h < H; ++h) {
            const int64_t s_off = (bb * H + h) * N * N;
            for (int64_t e = 0; e < N * N; ++e) S[e] = S0 ? S0[s_off + e] : 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const int64_t off = ((bb * T + t) * H + h) * N;
                for (int64_t i = 0; i < N; ++i) {            /* S_{t-1} a_t^T */
                    double acc = 0.0;
                    for (int64_t l = 0; l < N; ++l) acc += S[i * N + l] * a[off + l];
                    sa[i] = acc;
                }
                for (int64_t i = 0; i < N; ++i)
                    for (int64_t j = 0; j < N; ++j)
                        S[i * N + j] = S[i * N + j] * w[off + j] + sa[i] * b[off + j]
                                     + v[off + i] * k[off + j];
                for (int64_t i = 0; i < N; ++i) {            /* y_t = S_t r_t^T */
                    double acc = 0.0;
                    for (int64_t j = 0; j < N; ++j) acc += S[i * N + j] * r[off + j];
                    y[off + i] = acc;
                }
            }
            if (S1)
                for (int64_t e = 0; e < N * N; ++e) S1[s_off + e] = S[e];
        }
    free(S);
    free(sa);
    return 0;
}
