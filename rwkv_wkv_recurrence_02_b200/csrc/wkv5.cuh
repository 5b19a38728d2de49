// wkv5.cuh -- multi-head matrix-state WKV (v5: a decay rate per channel;
// v6: a decay rate per token and channel), recurrent form.
//
// The article "RWKVアーキテクチャ徹底解説" lists, in "RWKVバージョンの進化 /
// v4からv7まで", v5 (Eagle) with "multi-headed WKV, matrix-valued states" of
// h * (d/h)^2 numbers per layer and v6 (Finch) with "data-dependent time
// decay".  Per head of N channels the state is an N x N matrix S (key channel
// i, value channel j); token t reads it before its own update and adds its
// own outer product with the bonus u, then every key row decays and the
// token's outer product is added:
//
//   y_t[j] = sum_i r_t[i] S[i][j] + (sum_i r_t[i] u[i] k_t[i]) v_t[j]
//   S[i][j] <- e^{-w_t[i]} S[i][j] + k_t[i] v_t[j]
//
// One CTA per (sequence, head), 4 N threads: thread (g, j) keeps rows
// [g N/4, (g+1) N/4) of column j of S in registers (packed fp32 pairs of
// rows).  Tokens go in blocks of TB: the block's r, k, v (and decay factors)
// are staged in shared memory as fp32, each token's four partial sums of
// column j land in shared memory, and after the block every thread adds the
// partials and the bonus term of its outputs and stores them.  Three CTA
// barriers per block of TB tokens.
//
// Per element the recurrence costs 2 N multiply-adds (N/4 rows per thread
// for the output, and for the update): this form is bound by FP32
// arithmetic, not by memory.
#pragma once

#include "wkv_common.cuh"

namespace wkv {

struct Wkv5Args {
    const float* w;      // (C,) or (B, T, C) decay rates, factor e^{-w}
    const float* u;      // (C,)
    const void* r;
    const void* k;
    const void* v;
    const float* s_in;   // (B, H, N, N) or null (zeros)
    void* y;
    float* s_out;        // (B, H, N, N) or null
    int64_t B, T, C, H;
};

template <int N, int TB>
struct Wkv5Geometry {
    static constexpr int THREADS = 4 * N;
    static constexpr int NR = N / 4;   // rows of S per thread
    // r, k, decay, v staged as fp32 [TB][N], then the partial sums [4][TB][N]
    static constexpr uint32_t SMEM = (4 + 4) * TB * N * sizeof(float) + TB * sizeof(float) + N * sizeof(float);
};

template <typename IO>
__device__ __forceinline__ float io_load(const IO* p);
template <>
__device__ __forceinline__ float io_load<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float io_load<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p))) << 16);
}
template <typename IO>
__device__ __forceinline__ void io_store(IO* p, float x);
template <>
__device__ __forceinline__ void io_store<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void io_store<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename IO, int N, int TB, bool PERTOK>
__global__ void __launch_bounds__(4 * N)
wkv5_forward_kernel(const Wkv5Args A) {
    using G = Wkv5Geometry<N, TB>;
    constexpr int NT = G::THREADS;
    constexpr int NR = G::NR;
    extern __shared__ __align__(16) float sm5[];
    float* sr = sm5;                      // [TB][N]
    float* sk = sr + TB * N;
    float* sd = sk + TB * N;              // decay factors e^{-w}
    float* sv = sd + TB * N;
    float* sp = sv + TB * N;              // partial sums [4][TB][N]
    float* sruk = sp + 4 * TB * N;        // sum_i r u k per token [TB]
    float* su = sruk + TB;                // u of the head [N]

    pdl_begin();
    const int tid = threadIdx.x;
    const int j = tid % N, g = tid / N;
    const int64_t b = blockIdx.x / A.H, h = blockIdx.x % A.H;
    const int64_t C = A.C, T = A.T;
    const int64_t c0 = h * N;
    const IO* rp = static_cast<const IO*>(A.r);
    const IO* kp = static_cast<const IO*>(A.k);
    const IO* vp = static_cast<const IO*>(A.v);
    IO* yp = static_cast<IO*>(A.y);

    // state rows [g NR, (g+1) NR) of column j, as packed pairs of rows
    F2 S[NR / 2];
    const int64_t sbase = ((b * A.H + h) * N) * N + j;
#pragma unroll
    for (int q = 0; q < NR / 2; ++q) {
        const int i = g * NR + 2 * q;
        const float s0 = A.s_in ? A.s_in[sbase + int64_t(i) * N] : 0.f;
        const float s1 = A.s_in ? A.s_in[sbase + int64_t(i + 1) * N] : 0.f;
        S[q] = f2(s0, s1);
    }
    if (tid < N) su[tid] = A.u[c0 + tid];
    float dconst[NR];   // v5: this thread's rows' decay factors
#pragma unroll
    for (int q = 0; q < NR; ++q) dconst[q] = PERTOK ? 0.f : expf(-A.w[c0 + g * NR + q]);

    for (int64_t t0 = 0; t0 < T; t0 += TB) {
        const int nt = static_cast<int>(min(static_cast<int64_t>(TB), T - t0));
        // ---- stage the block (coalesced along channels) ----
        for (int e = tid; e < nt * N; e += NT) {
            const int t = e / N, c = e % N;
            const int64_t o = (b * T + t0 + t) * C + c0 + c;
            sr[e] = io_load<IO>(rp + o);
            sk[e] = io_load<IO>(kp + o);
            sv[e] = io_load<IO>(vp + o);
            if (PERTOK) sd[e] = expf(-__ldg(A.w + o));
        }
        __syncthreads();
        // ---- bonus dot products, one token per warp at a time ----
        {
            const int warp = tid >> 5, lane = tid & 31;
            for (int t = warp; t < nt; t += NT / 32) {
                float s = 0.f;
                for (int i = lane; i < N; i += 32) s = fmaf(sr[t * N + i] * su[i], sk[t * N + i], s);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) sruk[t] = s;
            }
        }
        // ---- the recurrence over the block ----
        for (int t = 0; t < nt; ++t) {
            const float* rr = sr + t * N + g * NR;
            const float* kk = sk + t * N + g * NR;
            const float* dd = sd + t * N + g * NR;
            const F2 vj = f2s(sv[t * N + j]);
            F2 acc = f2s(0.f);
#pragma unroll
            for (int q = 0; q < NR / 2; ++q) {
                const float2 r2 = *reinterpret_cast<const float2*>(rr + 2 * q);
                const float2 k2 = *reinterpret_cast<const float2*>(kk + 2 * q);
                F2 d2;
                if (PERTOK) {
                    const float2 x = *reinterpret_cast<const float2*>(dd + 2 * q);
                    d2 = f2(x.x, x.y);
                } else {
                    d2 = f2(dconst[2 * q], dconst[2 * q + 1]);
                }
                acc = fma2(f2(r2.x, r2.y), S[q], acc);
                S[q] = fma2(S[q], d2, mul2(f2(k2.x, k2.y), vj));
            }
            sp[(g * TB + t) * N + j] = f2lo(acc) + f2hi(acc);
        }
        __syncthreads();
        // ---- outputs of the block ----
        for (int e = tid; e < nt * N; e += NT) {
            const int t = e / N, c = e % N;
            const float yv = sp[(0 * TB + t) * N + c] + sp[(1 * TB + t) * N + c] + sp[(2 * TB + t) * N + c] +
                             sp[(3 * TB + t) * N + c] + sv[e] * sruk[t];
            io_store<IO>(yp + (b * T + t0 + t) * C + c0 + c, yv);
        }
        __syncthreads();
    }
    if (A.s_out != nullptr) {
#pragma unroll
        for (int q = 0; q < NR / 2; ++q) {
            const int i = g * NR + 2 * q;
            A.s_out[sbase + int64_t(i) * N] = f2lo(S[q]);
            A.s_out[sbase + int64_t(i + 1) * N] = f2hi(S[q]);
        }
    }
}

}  // namespace wkv
