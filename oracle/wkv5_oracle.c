/*
 * wkv5_oracle.c -- plain, slow, fp64 CPU oracle for the multi-head
 * matrix-state WKV (RWKV v5 "Eagle", v6 "Finch").
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * links, includes or calls anything here, and nothing here is shared with it.
 *
 * Source: the article "RWKVアーキテクチャ徹底解説：Transformerに匹敵する線形
 * アテンションRNN" (youngju.dev), section "RWKVバージョンの進化 / v4からv7まで":
 * v5 (Eagle) has "multi-headed WKV, matrix-valued states" with a state of
 * h * (d/h)^2 numbers per layer; v6 (Finch) adds "data-dependent time decay";
 * the training configuration of "学習とファインチューニングの実践ガイド /
 * スクラッチからのフル学習" gives a head size of 64 for v5 and later, and
 * "状態サイズ vs 情報容量" counts h * (d/h)^2 = 32 * 64^2 state numbers per
 * layer for d = 2048.  The pages give no formula beyond this.  The
 * reading used here (the plainest one with a matrix state of that size):
 * every head of N = d/h channels keeps an N x N state S whose entry (i, j)
 * pairs key channel i with value channel j and which grows by the outer
 * product k_t^T v_t of each token; key channel i decays by the factor
 * e^{-w[i]} per token (v5: one rate per channel; v6: a rate per token and
 * channel).  As in the v4 operator of the same article ("並列学習の定式化":
 * output from the current state, then decay and add), token t reads the
 * state before its own decay and adds its own contribution with the bonus u:
 *
 *   y_t[j] = sum_i r_t[i] * ( S[i][j] + u[i] k_t[i] v_t[j] )
 *   S[i][j] <- e^{-w_t[i]} S[i][j] + k_t[i] v_t[j]
 *
 * Written out, with S0 the carried state and 0-based t,
 *   y_t[j] = sum_i r_t[i] ( P(0,t)[i] S0[i][j]
 *            + sum_{s<t} P(s+1,t)[i] k_s[i] v_s[j] + u[i] k_t[i] v_t[j] ),
 *   P(a,t)[i] = prod_{m=a}^{t-1} e^{-w_m[i]}.
 * With N = 1, r = 1, keys e^{k} and bonus e^{u}, y is the v4 operator's
 * numerator (and with v = 1 its denominator): the v4 sum before the division.
 *
 * Layouts (row-major):
 *   r, k, v, y : (B, T, C), C = H * N, head h owns channels [h N, (h+1) N).
 *   w          : wmode 0: (C,);  wmode 1: (B, T, C).  Decay rates w >= 0.
 *   u          : (C,).
 *   state      : (B, H, N, N), S[b][h][i][j].  NULL in: zeros.
 *   yscale     : optional, the same sum over |terms| (each product taken in
 *                absolute value), the magnitude scale of relative errors.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

void oracle_wkv5_forward(int64_t B, int64_t T, int64_t H, int64_t N, int wmode,
                         const float* w, const float* u, const float* k, const float* v, const float* r,
                         const double* state_in, double* y, double* yscale, double* state_out) {
    const int64_t C = H * N;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)(N * N));
        double* A = (double*)malloc(sizeof(double) * (size_t)(N * N));   /* |S| recurrence */
        double* dec = (double*)malloc(sizeof(double) * (size_t)N);
        for (int64_t e = 0; e < N * N; ++e) {
            S[e] = state_in ? state_in[bh * N * N + e] : 0.0;
            A[e] = fabs(S[e]);
        }
        for (int64_t t = 0; t < T; ++t) {
            const int64_t row = (b * T + t) * C + h * N;
            for (int64_t j = 0; j < N; ++j) {
                double acc = 0.0, mag = 0.0;
                for (int64_t i = 0; i < N; ++i) {
                    const double ri = (double)r[row + i];
                    const double bonus = (double)u[h * N + i] * (double)k[row + i] * (double)v[row + j];
                    acc += ri * (S[i * N + j] + bonus);
                    mag += fabs(ri) * (A[i * N + j] + fabs(bonus));
                }
                y[row + j] = acc;
                if (yscale) yscale[row + j] = mag;
            }
            for (int64_t i = 0; i < N; ++i) {
                const double wi = wmode == 0 ? (double)w[h * N + i] : (double)w[row + i];
                dec[i] = exp(-wi);
            }
            for (int64_t i = 0; i < N; ++i) {
                for (int64_t j = 0; j < N; ++j) {
                    const double kv = (double)k[row + i] * (double)v[row + j];
                    S[i * N + j] = dec[i] * S[i * N + j] + kv;
                    A[i * N + j] = dec[i] * A[i * N + j] + fabs(kv);
                }
            }
        }
        if (state_out) memcpy(state_out + bh * N * N, S, sizeof(double) * (size_t)(N * N));
        free(S);
        free(A);
        free(dec);
    }
}
