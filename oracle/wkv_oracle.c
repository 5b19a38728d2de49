/*
 * wkv_oracle.c -- plain, slow, fp64 CPU oracle for the RWKV-4 WKV operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * links, includes or calls anything here, and nothing here is shared with it.
 *
 * Source of the method: the article "RWKVアーキテクチャ徹底解説：Transformerに
 * 匹敵する線形アテンションRNN" (youngju.dev), sections
 *   - "コア計算" (core computation): the explicit-sum definition of wkv_t;
 *   - "リカレント定式化" (recurrent formulation): the alpha/beta state update;
 *   - "対数空間計算による数値安定性" (log-space stability): the running-max
 *     bookkeeping, new max = max(previous max - w, k);
 *   - "並列学習の定式化" (parallel training formulation): the order "output
 *     from the current (undecayed) state, then decay and add";
 * and the block diagram in "高レベル構造" (out_t = sigmoid(r_t) * wkv_t);
 * the token shift that precedes the projections follows "トークンシフト：秘密
 * の要素" (mixing each input with the previous token's).
 *
 * Conventions shared by every function (all arrays row-major):
 *   k, v, r, y : (B, T, C), channel fastest.   r may be NULL (no gate).
 *   w, u       : (C,).  w > 0 is the per-step decay (w = exp(decay)), u the bonus.
 *   state      : (3, B, C) = {a, b, p}.  It represents numerator N = a*e^p and
 *                denominator D = b*e^p of the sums over every token seen so far,
 *                *without* the decay for the next step applied.  A fresh state
 *                is (0, 0, -1e38); -1e38 is a finite stand-in for log(0).
 *   Output index t is 0-based.  The carried state contributes e^{-t*w} * N to
 *   output t, exactly like a token that sits just before the chunk.
 *
 * Floating point: inputs arrive as float32 (the values the GPU sees); all
 * arithmetic is IEEE double with libm exp().  Build without -ffast-math.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_FRESH_P (-1e38)

static double sigmoid_f64(double r) { return 1.0 / (1.0 + exp(-r)); }

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Explicit-sum definition ("コア計算"), O(T^2) per lane.
 *
 *   wkv_t = ( S0num_t + sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u+k_t} v_t )
 *         / ( S0den_t + sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u+k_t}     )
 *
 * with the carried state as one more past term, S0num_t = a0*e^{p0 - t*w} and
 * S0den_t = b0*e^{p0 - t*w}.  Every exponent of one output is shifted by the
 * largest of them before exp(), so keys of any size stay finite.
 * y_t = sigmoid(r_t) * wkv_t when r is given.  yscale (optional) receives
 * sigmoid(r_t) * (sum of |numerator terms|) / (denominator), the magnitude
 * scale of the weighted average, used as the denominator of relative errors.
 */
void oracle_wkv_brute(int64_t B, int64_t T, int64_t C,
                      const float* w, const float* u,
                      const float* k, const float* v, const float* r,
                      const double* state_in, double* y, double* yscale,
                      int nthreads) {
    set_threads(nthreads);
    const int64_t lanes = B * C;
#pragma omp parallel for schedule(static)
    for (int64_t lane = 0; lane < lanes; ++lane) {
        const int64_t b = lane / C, c = lane % C;
        const double wc = (double)w[c], uc = (double)u[c];
        double a0 = 0.0, b0 = 0.0, p0 = ORACLE_FRESH_P;
        if (state_in) {
            a0 = state_in[0 * lanes + lane];
            b0 = state_in[1 * lanes + lane];
            p0 = state_in[2 * lanes + lane];
        }
        for (int64_t t = 0; t < T; ++t) {
            const int64_t it = (b * T + t) * C + c;
            const double kt = (double)k[it], vt = (double)v[it];
            /* largest exponent among all terms of this output */
            double m = uc + kt;
            const double ps = p0 - (double)t * wc;
            if (ps > m) m = ps;
            for (int64_t i = 0; i < t; ++i) {
                const double x = (double)k[(b * T + i) * C + c] - (double)(t - 1 - i) * wc;
                if (x > m) m = x;
            }
            double num = 0.0, den = 0.0, mag = 0.0;
            const double es = exp(ps - m);
            num += es * a0;
            den += es * b0;
            mag += es * fabs(a0);
            for (int64_t i = 0; i < t; ++i) {
                const int64_t ii = (b * T + i) * C + c;
                const double e = exp((double)k[ii] - (double)(t - 1 - i) * wc - m);
                num += e * (double)v[ii];
                den += e;
                mag += e * fabs((double)v[ii]);
            }
            const double ec = exp(uc + kt - m);
            num += ec * vt;
            den += ec;
            mag += ec * fabs(vt);
            const double g = r ? sigmoid_f64((double)r[it]) : 1.0;
            y[it] = g * (num / den);
            if (yscale) yscale[it] = g * (mag / den);
        }
    }
}

/*
 * One token of the log-space recurrence on one lane, in place on (a, b, p);
 * c carries the magnitude sum for yscale.
 *   output (parallel formulation order): o = max(p, u+k);
 *     wkv = (e^{p-o} a + e^{u+k-o} v) / (e^{p-o} b + e^{u+k-o})
 *   update ("リカレント定式化" with the "対数空間" max): q = max(p-w, k);
 *     a <- e^{p-w-q} a + e^{k-q} v,  b <- e^{p-w-q} b + e^{k-q},  p <- q
 */
static double lane_step(double wc, double uc, double kt, double vt,
                        double* a, double* b, double* p, double* c, double* scale) {
    const double o = (*p > uc + kt) ? *p : uc + kt;
    const double e1 = exp(*p - o), e2 = exp(uc + kt - o);
    const double den = e1 * (*b) + e2;
    const double wkv = (e1 * (*a) + e2 * vt) / den;
    if (scale) *scale = (e1 * (*c) + e2 * fabs(vt)) / den;
    const double pd = *p - wc;
    const double q = (pd > kt) ? pd : kt;
    const double e3 = exp(pd - q), e4 = exp(kt - q);
    *a = e3 * (*a) + e4 * vt;
    *b = e3 * (*b) + e4;
    *c = e3 * (*c) + e4 * fabs(vt);
    *p = q;
    return wkv;
}

/*
 * Parallel ("GPT") mode over one chunk: the recurrence above for t = 0..T-1.
 * state_in NULL means a fresh state.  state_out (optional) receives the state
 * after the last token, with the same meaning as state_in, so chaining chunks
 * is exact.  y and yscale are (B,T,C); yscale is optional.
 */
void oracle_wkv_forward(int64_t B, int64_t T, int64_t C,
                        const float* w, const float* u,
                        const float* k, const float* v, const float* r,
                        const double* state_in, double* y, double* yscale,
                        double* state_out, int nthreads) {
    set_threads(nthreads);
    const int64_t lanes = B * C;
#pragma omp parallel for schedule(static)
    for (int64_t lane = 0; lane < lanes; ++lane) {
        const int64_t b = lane / C, c = lane % C;
        const double wc = (double)w[c], uc = (double)u[c];
        double sa = 0.0, sb = 0.0, sp = ORACLE_FRESH_P;
        if (state_in) {
            sa = state_in[0 * lanes + lane];
            sb = state_in[1 * lanes + lane];
            sp = state_in[2 * lanes + lane];
        }
        double sc = fabs(sa);
        for (int64_t t = 0; t < T; ++t) {
            const int64_t it = (b * T + t) * C + c;
            double scale = 0.0;
            const double wkv = lane_step(wc, uc, (double)k[it], (double)v[it],
                                         &sa, &sb, &sp, &sc, yscale ? &scale : NULL);
            const double g = r ? sigmoid_f64((double)r[it]) : 1.0;
            y[it] = g * wkv;
            if (yscale) yscale[it] = g * scale;
        }
        if (state_out) {
            state_out[0 * lanes + lane] = sa;
            state_out[1 * lanes + lane] = sb;
            state_out[2 * lanes + lane] = sp;
        }
    }
}

/*
 * RNN ("decode") mode: one token for L independent layers of B sequences.
 * w, u: (L, C); k, v, r, y: (L, B, C); state: (L, 3, B, C), updated in place.
 * Same arithmetic as one iteration of oracle_wkv_forward.
 */
void oracle_wkv_step(int64_t L, int64_t B, int64_t C,
                     const float* w, const float* u,
                     const float* k, const float* v, const float* r,
                     double* state, double* y, int nthreads) {
    set_threads(nthreads);
    const int64_t lanes = B * C;
#pragma omp parallel for schedule(static)
    for (int64_t ll = 0; ll < L * lanes; ++ll) {
        const int64_t l = ll / lanes, lane = ll % lanes, c = lane % C;
        double* st = state + l * 3 * lanes;
        double a = st[0 * lanes + lane], b = st[1 * lanes + lane], p = st[2 * lanes + lane];
        double cm = fabs(a);
        const int64_t it = l * lanes + lane;
        const double wkv = lane_step((double)w[l * C + c], (double)u[l * C + c],
                                     (double)k[it], (double)v[it], &a, &b, &p, &cm, NULL);
        y[it] = (r ? sigmoid_f64((double)r[it]) : 1.0) * wkv;
        st[0 * lanes + lane] = a;
        st[1 * lanes + lane] = b;
        st[2 * lanes + lane] = p;
    }
}

/*
 * Segment summary and combine, the associative form of the state update
 * (the scan that "並列学習の定式化" says the parallel mode performs).
 *
 * summary of tokens k[0..n-1], v[0..n-1] of one lane started from the empty
 * state: (q, A, Bd) with N = A e^q, D = Bd e^q -- exactly the state the
 * recurrence reaches from (0, 0, -1e38).
 */
void oracle_wkv_summary(double w, int64_t n, const double* k, const double* v, double out[3]) {
    double a = 0.0, b = 0.0, p = ORACLE_FRESH_P, c = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        lane_step(w, 0.0, k[i], v[i], &a, &b, &p, &c, NULL);
    }
    out[0] = p;
    out[1] = a;
    out[2] = b;
}

/*
 * combine(S, seg): the state after a segment of length n whose summary is
 * (q, A, Bd), starting from S = (p, a, b).  The old state decays by n*w:
 *   p' = max(p - n*w, q);  a' = e^{p-n*w-p'} a + e^{q-p'} A;  b' likewise.
 */
void oracle_wkv_combine(double w, double p, double a, double b,
                        double q, double A, double Bd, int64_t n, double out[3]) {
    const double pd = p - (double)n * w;
    const double pp = (pd > q) ? pd : q;
    const double e1 = exp(pd - pp), e2 = exp(q - pp);
    out[0] = pp;
    out[1] = e1 * a + e2 * A;
    out[2] = e1 * b + e2 * Bd;
}

/*
 * Reverse mode (gradients) of oracle_wkv_forward over one chunk.  The pages
 * state that the parallel mode trains the model but print no gradient; this
 * is the chain rule applied to the recurrence of "リカレント定式化" in the
 * output-then-update order of "並列学習の定式化", per lane (0-based t):
 *
 *   N_{t+1} = lam N_t + e^{k_t} v_t,   D_{t+1} = lam D_t + e^{k_t},   lam = e^{-w}
 *   num_t = N_t + e^{u+k_t} v_t,  den_t = D_t + e^{u+k_t},  wkv_t = num_t / den_t
 *   y_t = g_t wkv_t,  g_t = sigmoid(r_t) (1 without a gate)
 *
 * with (N_0, D_0) = (a0 e^{p0}, b0 e^{p0}) from state_in.  Given dy = dL/dy
 * and ds_out = dL/d(a_T, b_T) for the state the forward returns (its p plane
 * is not read: later uses of a state depend on it only through N = a e^p and
 * D = b e^p, so dL/dN_T = dL/da_T e^{-p_T}), with gN_t = dL/dN_t, gD_t =
 * dL/dD_t summed over every later use:
 *
 *   dnum_t = g_t dy_t / den_t,  dden_t = -g_t dy_t wkv_t / den_t
 *   gN_t = dnum_t + lam gN_{t+1},   gD_t = dden_t + lam gD_{t+1}
 *   dv_t = dnum_t e^{u+k_t} + gN_{t+1} e^{k_t}
 *   dk_t = (dnum_t v_t + dden_t) e^{u+k_t} + (gN_{t+1} v_t + gD_{t+1}) e^{k_t}
 *   du  += (dnum_t v_t + dden_t) e^{u+k_t}
 *   dw  += -lam (gN_{t+1} N_t + gD_{t+1} D_t)
 *   dr_t = dy_t wkv_t g_t (1 - g_t)
 *   ds_in = (gN_0 e^{p0}, gD_0 e^{p0}, a0 gN_0 e^{p0} + b0 gD_0 e^{p0})
 *
 * dw and du are summed over every sequence and token of their channel.
 * Arithmetic: plain IEEE double, with every exponent of a lane shifted by
 * the lane's largest weight exponent (all gradients are invariant to that
 * shift), so weights are <= 1.  Valid while the smallest terms that matter
 * stay inside double range, which holds for the test inputs (|k| <= 60,
 * T up to a few thousand).  p_T, the scale of the returned state, is taken
 * from the same log-space recurrence as oracle_wkv_forward.
 *
 * dr may be NULL (no gate); ds_out NULL means zero; ds_in may be NULL.
 */
void oracle_wkv_backward(int64_t B, int64_t T, int64_t C,
                         const float* w, const float* u,
                         const float* k, const float* v, const float* r,
                         const double* state_in, const double* dy, const double* ds_out,
                         double* dk, double* dv, double* dr, double* dw, double* du,
                         double* ds_in, int nthreads) {
    set_threads(nthreads);
    const int64_t lanes = B * C;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        const double wc = (double)w[c], uc = (double)u[c], lam = exp(-wc);
        double* Nt = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double* Dt = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double dw_c = 0.0, du_c = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            const int64_t lane = b * C + c;
            double a0 = 0.0, b0 = 0.0, p0 = ORACLE_FRESH_P;
            if (state_in) {
                a0 = state_in[0 * lanes + lane];
                b0 = state_in[1 * lanes + lane];
                p0 = state_in[2 * lanes + lane];
            }
            /* the lane's largest weight exponent, and p_T of the forward */
            double m = p0, sa = a0, sb = b0, sp = p0, sc = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const int64_t it = (b * T + t) * C + c;
                const double kt = (double)k[it];
                if (kt > m) m = kt;
                if (uc + kt > m) m = uc + kt;
                lane_step(wc, uc, kt, (double)v[it], &sa, &sb, &sp, &sc, NULL);
            }
            const double pT = sp;
            /* forward: N_t, D_t before token t, shifted by e^{-m} */
            double N = a0 * exp(p0 - m), D = b0 * exp(p0 - m);
            for (int64_t t = 0; t < T; ++t) {
                const int64_t it = (b * T + t) * C + c;
                Nt[t] = N;
                Dt[t] = D;
                const double et = exp((double)k[it] - m);
                N = lam * N + et * (double)v[it];
                D = lam * D + et;
            }
            /* reverse: gN, gD = dL/dN_{t+1}, dL/dD_{t+1} (shifted by e^{+m}) */
            double gN = 0.0, gD = 0.0;
            if (ds_out) {
                const double s = exp(m - pT);
                gN = ds_out[0 * lanes + lane] * s;
                gD = ds_out[1 * lanes + lane] * s;
            }
            for (int64_t t = T - 1; t >= 0; --t) {
                const int64_t it = (b * T + t) * C + c;
                const double kt = (double)k[it], vt = (double)v[it];
                const double et = exp(kt - m), Et = exp(uc + kt - m);
                const double num = Nt[t] + Et * vt, den = Dt[t] + Et;
                const double wkv = num / den;
                const double g = r ? sigmoid_f64((double)r[it]) : 1.0;
                const double h = g * dy[it];
                const double dnum = h / den, dden = -h * wkv / den;
                dv[it] = dnum * Et + gN * et;
                dk[it] = (dnum * vt + dden) * Et + (gN * vt + gD) * et;
                du_c += (dnum * vt + dden) * Et;
                dw_c += -lam * (gN * Nt[t] + gD * Dt[t]);
                if (dr) dr[it] = dy[it] * wkv * g * (1.0 - g);
                gN = dnum + lam * gN;
                gD = dden + lam * gD;
            }
            if (ds_in) {
                const double s = exp(p0 - m);
                const double ga = gN * s, gb = gD * s;
                ds_in[0 * lanes + lane] = ga;
                ds_in[1 * lanes + lane] = gb;
                ds_in[2 * lanes + lane] = a0 * ga + b0 * gb;
            }
        }
        dw[c] = dw_c;
        du[c] = du_c;
        free(Nt);
        free(Dt);
    }
}

/*
 * Token shift ("トークンシフト：秘密の要素"): before its R, K, V projections
 * every sub-layer mixes each token's input with the previous token's,
 *     x'_t = mu * x_t + (1 - mu) * x_{t-1},
 * with one learned interpolation weight mu per channel.  nmix mixes (one row
 * of mu each, e.g. one per projection) of the same input.
 *
 *   x      : (B, T, C)
 *   mu     : (nmix, C)
 *   x_prev : (B, C), the input of the token before x[:, 0, :] (carried from
 *            an earlier chunk or decode step), or NULL for a fresh sequence,
 *            whose first token mixes with zeros.
 *   out    : (nmix, B, T, C)
 *   x_last : (B, C) or NULL, receives the input the next call mixes its first
 *            token with: x[:, T-1, :], or x_prev (zeros) when T == 0.
 */
void oracle_token_shift(int64_t B, int64_t T, int64_t C, int64_t nmix, const float* x, const float* mu,
                        const float* x_prev, double* out, double* x_last) {
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < C; ++c) {
            double prev = x_prev ? (double)x_prev[b * C + c] : 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const double cur = (double)x[(b * T + t) * C + c];
                for (int64_t m = 0; m < nmix; ++m) {
                    const double mc = (double)mu[m * C + c];
                    out[((m * B + b) * T + t) * C + c] = mc * cur + (1.0 - mc) * prev;
                }
                prev = cur;
            }
            if (x_last) x_last[b * C + c] = prev;
        }
    }
}
