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
// rows).  Tokens go in blocks of TB: every thread also stages 8 channels of
// one token of the next block (one 16-byte load per array, fetched a block
// ahead, stored into the other of two shared-memory buffers as fp32 with its
// share of the token's bonus dot product), each token's four partial sums of
// column j land in shared memory, and after the block every thread adds the
// partials and the bonus term of its outputs and stores them.  Two CTA
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
    static constexpr int TPR = N / 8;  // staging threads per token row (8 channels each)
    static_assert(TB * TPR == THREADS, "one 8-channel vector per staging thread per block");
    // a staging buffer: r, k, v, decay as fp32 [TB][N] and the bonus dot
    // products [TB]; two of them, then the partial sums [4][TB][N] and u [N]
    static constexpr uint32_t STAGE = (4 * TB * N + TB) * sizeof(float);
    static constexpr uint32_t SMEM = 2 * STAGE + 4 * TB * N * sizeof(float) + N * sizeof(float);
};

// Eight consecutive channels of one row, read as fp32.
template <typename IO>
struct Row8;
template <>
struct Row8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ float get(int i) const {
        return i < 4 ? (i == 0 ? a.x : i == 1 ? a.y : i == 2 ? a.z : a.w)
                     : (i == 4 ? b.x : i == 5 ? b.y : i == 6 ? b.z : b.w);
    }
};
template <>
struct Row8<__nv_bfloat16> {
    uint4 a;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { a = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ float get(int i) const {
        const uint32_t x = (i >> 1) == 0 ? a.x : (i >> 1) == 1 ? a.y : (i >> 1) == 2 ? a.z : a.w;
        return __uint_as_float((i & 1) ? (x & 0xffff0000u) : (x << 16));
    }
};

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
    constexpr int TPR = G::TPR;
    constexpr int SF = G::STAGE / sizeof(float);
    extern __shared__ __align__(16) float sm5[];
    float* sp = sm5 + 2 * SF;             // partial sums [4][TB][N]
    float* su = sp + 4 * TB * N;          // u of the head [N]

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
    // staging role: token row st of a block, channels [sc, sc + 8)
    const int st = tid / TPR, sc = (tid % TPR) * 8;

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
    float uu[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) uu[e] = A.u[c0 + sc + e];
    float dconst[NR];   // v5: this thread's rows' decay factors
#pragma unroll
    for (int q = 0; q < NR; ++q) dconst[q] = PERTOK ? 0.f : expf(-A.w[c0 + g * NR + q]);

    // one token row of 8 channels per staging thread, fetched a block ahead
    Row8<IO> pr, pk, pv;
    Row8<float> pw;
    bool pvalid = false;
    auto fetch = [&](int64_t t0) {
        pvalid = t0 + st < T;
        if (pvalid) {
            const int64_t o = (b * T + t0 + st) * C + c0 + sc;
            pr.load(rp + o);
            pk.load(kp + o);
            pv.load(vp + o);
            if (PERTOK) pw.load(A.w + o);
        }
    };
    // the fetched row into staging buffer `buf` as fp32, with its share of
    // the token's bonus dot product sum_i r_i u_i k_i
    auto put = [&](int buf) {
        float* sr = sm5 + buf * SF;
        float* sk = sr + TB * N;
        float* sv = sk + TB * N;
        float* sd = sv + TB * N;
        float* sruk = sd + TB * N;
        float part = 0.f;
        float rr[8], kk[8], vv[8], dd[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            rr[e] = pvalid ? pr.get(e) : 0.f;
            kk[e] = pvalid ? pk.get(e) : 0.f;
            vv[e] = pvalid ? pv.get(e) : 0.f;
            dd[e] = (PERTOK && pvalid) ? expf(-pw.get(e)) : 0.f;
            part = fmaf(rr[e] * uu[e], kk[e], part);
        }
        const int o = st * N + sc;
        *reinterpret_cast<float4*>(sr + o) = make_float4(rr[0], rr[1], rr[2], rr[3]);
        *reinterpret_cast<float4*>(sr + o + 4) = make_float4(rr[4], rr[5], rr[6], rr[7]);
        *reinterpret_cast<float4*>(sk + o) = make_float4(kk[0], kk[1], kk[2], kk[3]);
        *reinterpret_cast<float4*>(sk + o + 4) = make_float4(kk[4], kk[5], kk[6], kk[7]);
        *reinterpret_cast<float4*>(sv + o) = make_float4(vv[0], vv[1], vv[2], vv[3]);
        *reinterpret_cast<float4*>(sv + o + 4) = make_float4(vv[4], vv[5], vv[6], vv[7]);
        if (PERTOK) {
            *reinterpret_cast<float4*>(sd + o) = make_float4(dd[0], dd[1], dd[2], dd[3]);
            *reinterpret_cast<float4*>(sd + o + 4) = make_float4(dd[4], dd[5], dd[6], dd[7]);
        }
        // the TPR staging threads of a token are consecutive lanes of one warp
#pragma unroll
        for (int o2 = TPR / 2; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
        if (tid % TPR == 0) sruk[st] = part;
    };

    fetch(0);
    put(0);
    if (TB < T) fetch(TB);
    __syncthreads();
    int cur = 0;
    for (int64_t t0 = 0; t0 < T; t0 += TB) {
        const int nt = static_cast<int>(min(static_cast<int64_t>(TB), T - t0));
        const float* sr = sm5 + cur * SF;
        const float* sk = sr + TB * N;
        const float* sv = sk + TB * N;
        const float* sd = sv + TB * N;
        const float* sruk = sd + TB * N;
        // ---- the recurrence over the block ----
        for (int t = 0; t < nt; ++t) {
            const float* rr = sr + t * N + g * NR;
            const float* kk = sk + t * N + g * NR;
            const float* dd = sd + t * N + g * NR;
            const F2 vj = f2s(sv[t * N + j]);
            F2 acc0 = f2s(0.f), acc1 = f2s(0.f);
#pragma unroll
            for (int q4 = 0; q4 < NR / 4; ++q4) {
                const float4 r4 = *reinterpret_cast<const float4*>(rr + 4 * q4);
                const float4 k4 = *reinterpret_cast<const float4*>(kk + 4 * q4);
                F2 da, db;
                if (PERTOK) {
                    const float4 d4 = *reinterpret_cast<const float4*>(dd + 4 * q4);
                    da = f2(d4.x, d4.y);
                    db = f2(d4.z, d4.w);
                } else {
                    da = f2(dconst[4 * q4], dconst[4 * q4 + 1]);
                    db = f2(dconst[4 * q4 + 2], dconst[4 * q4 + 3]);
                }
                acc0 = fma2(f2(r4.x, r4.y), S[2 * q4], acc0);
                acc1 = fma2(f2(r4.z, r4.w), S[2 * q4 + 1], acc1);
                S[2 * q4] = fma2(S[2 * q4], da, mul2(f2(k4.x, k4.y), vj));
                S[2 * q4 + 1] = fma2(S[2 * q4 + 1], db, mul2(f2(k4.z, k4.w), vj));
            }
            const F2 acc = add2(acc0, acc1);
            sp[(g * TB + t) * N + j] = f2lo(acc) + f2hi(acc);
        }
        __syncthreads();
        // ---- outputs of the block; the next block's rows go into the other buffer ----
        for (int e = tid; e < nt * N; e += NT) {
            const int t = e / N, c = e % N;
            const float yv = sp[(0 * TB + t) * N + c] + sp[(1 * TB + t) * N + c] + sp[(2 * TB + t) * N + c] +
                             sp[(3 * TB + t) * N + c] + sv[e] * sruk[t];
            io_store<IO>(yp + (b * T + t0 + t) * C + c0 + c, yv);
        }
        if (t0 + TB < T) {
            put(cur ^ 1);
            if (t0 + 2 * TB < T) fetch(t0 + 2 * TB);
        }
        __syncthreads();
        cur ^= 1;
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
