// wkv_segment.cuh -- the per-segment arithmetic the chunked kernels share.
//
// A warp owns a segment of LS consecutive tokens of 64 channels (a thread
// holds two adjacent channels as a packed fp32 pair); the segment's rows sit
// in a shared-memory tile that a TMA copy filled.
//
//   pass 0  key range of the segment and its running-max exponent q.
//   pass 1  the segment's summary (the state it reaches from the empty
//           state).  Fast path: every token scaled by the segment's largest
//           key, one ex2 per token; if the keys (with the bonus) span too
//           wide a range for one reference, the exact running-max recurrence.
//   pass 2  outputs from the segment's start state: the fast path reuses the
//           cached exponentials (or recomputes them), else the exact
//           recurrence.
//
// Also the mbarrier arrive and the bulk copy the TMA kernels use.
#pragma once

#include "wkv_chunk.cuh"

namespace wkv {

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <bool GATE>
__device__ __forceinline__ constexpr int NARR_OF() { return GATE ? 3 : 2; }

// Per-thread state of one unit between pass 1 and pass 2.  A thread owns
// V = 2 adjacent channels; their arithmetic runs on packed fp32 pairs.
template <int V, int LS>
struct SegCtx {
    static_assert(V == 2, "the segment code works on channel pairs");
    static_assert(LS % 2 == 0, "pass 0 takes rows two at a time");
    float w2[V], u2[V], dk[V], eu[V];
    float kmax[V], kmin[V];   // base 2
    F2 kf[LS];                // raw keys after pass 0; 2^(k2 - kmax) after a fast pass 1
    int64_t base;
    int nvalid;
    bool cvalid, fast1;
};

// Per-channel parameters of this thread's V channels (base 2): w2, u2 and
// the per-step decay 2^-w2 and bonus factor 2^u2.  Channels past C get
// harmless stand-ins.
template <int V, int LS>
__device__ __forceinline__ void set_params(SegCtx<V, LS>& cx, const float* w, const float* u) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
        cx.w2[j] = cx.cvalid ? w[j] * kLog2e : 1.f;
        cx.u2[j] = cx.cvalid ? u[j] * kLog2e : 0.f;
        cx.dk[j] = ex2(-cx.w2[j]);
        cx.eu[j] = ex2(cx.u2[j]);
    }
}

template <typename IO>
__device__ __forceinline__ F2 raw_pair(typename Vec<IO, 2>::raw x);
template <>
__device__ __forceinline__ F2 raw_pair<float>(float2 x) { return f2(x.x, x.y); }
template <>
__device__ __forceinline__ F2 raw_pair<__nv_bfloat16>(uint32_t x) {
    return f2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Pass 0 + pass 1 of one warp's segment; returns the segment summary.
// PARAMS_IN_STAGE: read w, u from the stage's parameter area (else the
// caller has set them in cx already).  CACHE: keep the per-token
// exponentials of the fast path in cx.kf for pass 2 (else pass 2 recomputes
// them from the keys in the stage, and kf is dead after pass 1).
// EXACT_Q: form every candidate exponent of pass 0 from one product,
// k2_i - (n-1-i) w2, instead of running sums of w2; the running sums round
// once per token, which long segments (32 tokens) with a fast decay make
// visible in q.
//
// Pass 0 works on raw keys: the key range (max, min) and the segment's
// running-max exponent q = max_i (k2_i + i w2) - (n-1) w2, which equals the
// recurrence p <- max(p - w2, k2) over the segment.  Pass 1 (fast path)
// scales every token by the largest key: one ex2 per token, whose argument
// fuses the base-2 conversion.
template <typename IO, int V, bool GATE, int W, int LS, bool FULL, bool PARAMS_IN_STAGE = true, bool CACHE = true,
          bool EXACT_Q = false>
__device__ __forceinline__ void seg_pass01(const ChunkArgs& A, int64_t chunk, int64_t b, int64_t c,
                                           const unsigned char* stage, SegCtx<V, LS>& cx, St* seg) {
    constexpr int CB = 32 * V;
    constexpr int TT = W * LS;
    constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    constexpr int TILE = TT * ROW;
    using Raw = typename Vec<IO, V>::raw;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    cx.cvalid = c < A.C;
    const int64_t t_seg = chunk * TT + warp * LS;
    cx.nvalid = FULL ? LS : static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), A.T - t_seg)));
    cx.base = (b * A.T + t_seg) * A.C + c;
    if (PARAMS_IN_STAGE) set_params<V>(cx, reinterpret_cast<const float*>(stage + NARR_OF<GATE>() * TILE) + lane * V,
                                       reinterpret_cast<const float*>(stage + NARR_OF<GATE>() * TILE) + CB + lane * V);
    const unsigned char* srow = stage + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));
    const F2 L2 = f2s(kLog2e);
    const F2 W2 = f2(cx.w2[0], cx.w2[1]);

    // ---- pass 0 ----
    const float nm1 = static_cast<float>(cx.nvalid - 1);
    float kx0 = -3.0e38f, kx1 = -3.0e38f, kn0 = 3.0e38f, kn1 = 3.0e38f;
    float qa0 = -3.0e38f, qa1 = -3.0e38f;
    F2 iw = f2s(0.f);
#pragma unroll
    for (int i = 0; i < LS; i += 2) {
        const bool two = FULL || i + 1 < cx.nvalid;
        if (FULL || i < cx.nvalid) {
            const F2 ka = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + i * ROW));
            const F2 kb = two ? raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + (i + 1) * ROW)) : ka;
            cx.kf[i] = ka;
            cx.kf[i + 1] = kb;
            kx0 = max3(kx0, f2lo(ka), f2lo(kb));
            kx1 = max3(kx1, f2hi(ka), f2hi(kb));
            kn0 = min3(kn0, f2lo(ka), f2lo(kb));
            kn1 = min3(kn1, f2hi(ka), f2hi(kb));
            F2 qa, qb;
            if constexpr (EXACT_Q) {
                const float oa = static_cast<float>(i) - nm1, ob = oa + 1.f;
                qa = fma2(ka, L2, f2(oa * cx.w2[0], oa * cx.w2[1]));
                qb = two ? fma2(kb, L2, f2(ob * cx.w2[0], ob * cx.w2[1])) : qa;
            } else {
                qa = fma2(ka, L2, iw);
                iw = add2(iw, W2);
                qb = two ? fma2(kb, L2, iw) : qa;
                iw = add2(iw, W2);
            }
            qa0 = max3(qa0, f2lo(qa), f2lo(qb));
            qa1 = max3(qa1, f2hi(qa), f2hi(qb));
        }
    }
    const float q[2] = {EXACT_Q ? qa0 : qa0 - nm1 * cx.w2[0], EXACT_Q ? qa1 : qa1 - nm1 * cx.w2[1]};
    cx.kmax[0] = kx0 * kLog2e;
    cx.kmax[1] = kx1 * kLog2e;
    cx.kmin[0] = kn0 * kLog2e;
    cx.kmin[1] = kn1 * kLog2e;
    cx.fast1 = (cx.kmax[0] - cx.kmin[0] + fabsf(cx.u2[0]) <= kFastSpan) &&
               (cx.kmax[1] - cx.kmin[1] + fabsf(cx.u2[1]) <= kFastSpan);

    // ---- pass 1: segment summary ----
    if (cx.nvalid == 0) {
        seg[0] = seg[1] = st_identity();
    } else if (cx.fast1) {
        const F2 KM = f2(-cx.kmax[0], -cx.kmax[1]);
        const F2 DK = f2(cx.dk[0], cx.dk[1]);
        F2 n = f2s(0.f), db = f2s(0.f);
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < cx.nvalid) {
                const F2 ek = ex2x2(fma2(cx.kf[i], L2, KM));
                if constexpr (CACHE) cx.kf[i] = ek;
                const F2 ekv = mul2(ek, raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + TILE + i * ROW)));
                n = fma2(n, DK, ekv);
                db = fma2(db, DK, ek);
            }
        }
        const float sc0 = ex2(cx.kmax[0] - q[0]), sc1 = ex2(cx.kmax[1] - q[1]);
        seg[0] = St{q[0], f2lo(n) * sc0, f2lo(db) * sc0};
        seg[1] = St{q[1], f2hi(n) * sc1, f2hi(db) * sc1};
    } else {
        // keys too spread for one reference: the exact running-max
        // recurrence, its exponent held as pb - m w2 (see lane_token_pm)
        float pb[V], m[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            seg[j] = st_identity();
            pb[j] = seg[j].p;
            m[j] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < cx.nvalid) {
                const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + TILE + i * ROW));
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float k2 = (j == 0 ? f2lo(cx.kf[i]) : f2hi(cx.kf[i])) * kLog2e;
                    const float v1 = j == 0 ? f2lo(vv) : f2hi(vv);
                    const float pd = fmaf(-(m[j] + 1.f), cx.w2[j], pb[j]);
                    const float d2 = pd - k2;
                    const float e = ex2(-fabsf(d2));
                    if (d2 >= 0.f) {
                        seg[j].a = fmaf(e, v1, seg[j].a);
                        seg[j].b += e;
                        m[j] += 1.f;
                    } else {
                        seg[j].a = fmaf(e, seg[j].a, v1);
                        seg[j].b = fmaf(e, seg[j].b, 1.f);
                        pb[j] = k2;
                        m[j] = 0.f;
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) seg[j].p = fmaf(-m[j], cx.w2[j], pb[j]);
    }
}

// One token of the exact recurrence (as lane_token, base 2) with the
// running-max exponent held as pb - m w: pb is the last new maximum, m the
// decay steps since.  Each token forms its exponents from pb with one
// rounding; p <- p - w would round once per token, and at exponents near the
// largest keys (|p| ~ 70 for keys of 50) that error accumulates along the
// segment into the relative weights of old and new terms.
__device__ __forceinline__ float lane_token_pm(float& a, float& b, float& pb, float& m, float w, float u, float k,
                                               float v, float gate_den) {
    const float p = fmaf(-m, w, pb);
    const float d1 = p - (u + k);
    const float e1 = ex2(-fabsf(d1));
    float num, den;
    if (d1 >= 0.f) {
        num = fmaf(e1, v, a);
        den = b + e1;
    } else {
        num = fmaf(e1, a, v);
        den = fmaf(e1, b, 1.f);
    }
    const float y = num * rcp(den * gate_den);
    const float pd = fmaf(-(m + 1.f), w, pb);
    const float d2 = pd - k;
    const float e2 = ex2(-fabsf(d2));
    if (d2 >= 0.f) {
        a = fmaf(e2, v, a);
        b = b + e2;
        m += 1.f;
    } else {
        a = fmaf(e2, a, v);
        b = fmaf(e2, b, 1.f);
        pb = k;
        m = 0.f;
    }
    return y;
}
// Pass 2 of one warp's segment: outputs from the segment's start state st.
// Fast path: every term rescaled to R = max(kmax, p) and the cached
// exponentials reused (CACHE; else one more ex2 per token, straight to the
// scale R); one ex2 (gate) and one rcp per output.  Otherwise the exact
// running-max recurrence from keys read again from the stage.
template <typename IO, int V, bool GATE, int W, int LS, bool FULL, bool CACHE = true>
__device__ __forceinline__ void seg_pass2(const ChunkArgs& A, const unsigned char* stage, SegCtx<V, LS>& cx,
                                          St* st) {
    constexpr int CB = 32 * V;
    constexpr int TT = W * LS;
    constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    constexpr int TILE = TT * ROW;
    using Ld = Vec<IO, V>;
    using Raw = typename Ld::raw;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned char* srow = stage + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));
    bool fast2 = cx.fast1;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const bool near = st[j].p >= cx.kmax[j] - kFastState;
        const bool negligible = st[j].p < cx.kmax[j] - 1.5f * kFastState && st[j].b <= 16777216.f;
        fast2 = fast2 && (st[j].p - cx.kmin[j] + fabsf(cx.u2[j]) <= kFastState) && (near || negligible);
    }
    IO* yp = static_cast<IO*>(A.y) + cx.base;
    const int64_t C = A.C;
    if (fast2) {
        float sl[V], ss[V], nr[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float R = fmaxf(cx.kmax[j], st[j].p);
            sl[j] = CACHE ? ex2(cx.kmax[j] - R) : 0.f;
            ss[j] = ex2(st[j].p - R);
            nr[j] = -R;
        }
        const F2 SL = f2(sl[0], sl[1]);
        const F2 NR = f2(nr[0], nr[1]);
        const F2 L2 = f2s(kLog2e);
        const F2 EU = f2(cx.eu[0], cx.eu[1]);
        const F2 DK = f2(cx.dk[0], cx.dk[1]);
        const F2 NL = f2s(-kLog2e);
        F2 n = f2(st[0].a * ss[0], st[1].a * ss[1]);
        F2 db = f2(st[0].b * ss[0], st[1].b * ss[1]);
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < cx.nvalid) {
                F2 ek;
                if constexpr (CACHE) ek = mul2(cx.kf[i], SL);
                else ek = ex2x2(fma2(raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + i * ROW)), L2, NR));
                const F2 ekv = mul2(ek, raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + TILE + i * ROW)));
                const F2 num = fma2(EU, ekv, n);
                F2 den = fma2(EU, ek, db);
                if (GATE) {
                    const F2 g = ex2x2(mul2(raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + 2 * TILE + i * ROW)), NL));
                    den = fma2(den, g, den);
                }
                const F2 y = mul2(num, rcpx2(den));
                n = fma2(n, DK, ekv);
                db = fma2(db, DK, ek);
                const float out[2] = {f2lo(y), f2hi(y)};
                Ld::store(yp, out);
            }
            yp += C;
        }
    } else {
        float pb[V], m[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            pb[j] = st[j].p;
            m[j] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < cx.nvalid) {
                const F2 kk = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + i * ROW));
                const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + TILE + i * ROW));
                F2 rv = f2s(0.f);
                if (GATE) rv = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + 2 * TILE + i * ROW));
                float out[V];
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float gd = GATE ? gate_den(j == 0 ? f2lo(rv) : f2hi(rv)) : 1.f;
                    const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                    out[j] = lane_token_pm(st[j].a, st[j].b, pb[j], m[j], cx.w2[j], cx.u2[j], k2,
                                           j == 0 ? f2lo(vv) : f2hi(vv), gd);
                }
                Ld::store(yp, out);
            }
            yp += C;
        }
#pragma unroll
        for (int j = 0; j < V; ++j) st[j].p = fmaf(-m[j], cx.w2[j], pb[j]);
    }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

}  // namespace wkv
