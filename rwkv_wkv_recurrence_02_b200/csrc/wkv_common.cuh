// wkv_common.cuh -- device helpers shared by the WKV kernels (sm_100a).
//
// All kernels work in base-2 log space: exponents are scaled by log2(e) once
// when they are loaded (k, u, w, the state's p), so every exponential is one
// ex2.approx (MUFU) instruction.  The state crosses the ABI in natural-log
// units and is converted on load and store.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// The empty state's p is -1e38 (natural log), a finite stand-in for log(0):
// p - w and p - (u + k) stay finite, and 2^(huge negative) is exactly 0.
constexpr float kFreshP = -1e38f;
constexpr float kFreshP2 = -1e38f * 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A state in max form, base 2: numerator = a * 2^p, denominator = b * 2^p.
struct St {
    float p, a, b;
};

__device__ __forceinline__ St st_identity() { return St{kFreshP2, 0.f, 0.f}; }

// State after a segment whose own summary (from the empty state) is x, when
// the segment starts from s.  s decays by `decay` = (segment length) * w2.
// Exactly one of the two scale factors is 1, so this is one ex2.
__device__ __forceinline__ St st_combine(St s, St x, float decay) {
    const float pd = s.p - decay;
    const float diff = pd - x.p;
    const float e = ex2(-fabsf(diff));
    St o;
    if (diff >= 0.f) {
        o.p = pd;
        o.a = fmaf(e, x.a, s.a);
        o.b = fmaf(e, x.b, s.b);
    } else {
        o.p = x.p;
        o.a = fmaf(e, s.a, x.a);
        o.b = fmaf(e, s.b, x.b);
    }
    return o;
}

// ---------------------------------------------------------------------------
// element I/O: V consecutive channels of one row as one vector access
// ---------------------------------------------------------------------------
template <typename IO, int V>
struct Vec;

template <>
struct Vec<float, 1> {
    using raw = float;
    static __device__ __forceinline__ raw load(const float* p) { return __ldg(p); }
    static __device__ __forceinline__ float get(raw x, int) { return x; }
    static __device__ __forceinline__ void store(float* p, const float* y) { *p = y[0]; }
};

template <>
struct Vec<float, 2> {
    using raw = float2;
    static __device__ __forceinline__ raw load(const float* p) {
        return __ldg(reinterpret_cast<const float2*>(p));
    }
    static __device__ __forceinline__ float get(raw x, int j) { return j == 0 ? x.x : x.y; }
    static __device__ __forceinline__ void store(float* p, const float* y) {
        *reinterpret_cast<float2*>(p) = make_float2(y[0], y[1]);
    }
};

template <>
struct Vec<__nv_bfloat16, 1> {
    using raw = unsigned short;
    static __device__ __forceinline__ raw load(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const unsigned short*>(p));
    }
    static __device__ __forceinline__ float get(raw x, int) {
        return __uint_as_float(static_cast<uint32_t>(x) << 16);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* y) {
        *p = __float2bfloat16_rn(y[0]);
    }
};

template <>
struct Vec<__nv_bfloat16, 2> {
    using raw = uint32_t;
    static __device__ __forceinline__ raw load(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const unsigned int*>(p));
    }
    static __device__ __forceinline__ float get(raw x, int j) {
        return __uint_as_float(j == 0 ? (x << 16) : (x & 0xffff0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* y) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(y[0], y[1]);
    }
};

// One log-space token on one lane (the plain recurrence):
//   output  o = max(p, u+k): y = (e^(p-o) a + e^(u+k-o) v) / (e^(p-o) b + e^(u+k-o))
//   update  q = max(p-w, k): a <- e^(p-w-q) a + e^(k-q) v, b likewise, p <- q
// p, w, u, k are in the units of `to2`: natural log with to2 = log2(e), or
// already base 2 with to2 = 1.  Exactly one of each pair of factors is 1, so
// a token costs two ex2.  `gate_den` multiplies the denominator (1 + e^-r
// for the sigmoid gate, else 1).
__device__ __forceinline__ float lane_token(float& a, float& b, float& p, float w, float u,
                                            float k, float v, float gate_den, float to2) {
    const float d1 = p - (u + k);
    const float e1 = ex2(-fabsf(d1) * to2);
    float num, den;
    if (d1 >= 0.f) {
        num = fmaf(e1, v, a);
        den = b + e1;
    } else {
        num = fmaf(e1, a, v);
        den = fmaf(e1, b, 1.f);
    }
    const float y = num * rcp(den * gate_den);
    const float pd = p - w;
    const float d2 = pd - k;
    const float e2 = ex2(-fabsf(d2) * to2);
    if (d2 >= 0.f) {
        a = fmaf(e2, v, a);
        b = b + e2;
        p = pd;
    } else {
        a = fmaf(e2, a, v);
        b = fmaf(e2, b, 1.f);
        p = k;
    }
    return y;
}

// ---------------------------------------------------------------------------
// packed fp32 pairs (sm_100 f32x2 arithmetic): the two channels a thread owns
// ---------------------------------------------------------------------------
struct F2 {
    unsigned long long v;
};

__device__ __forceinline__ F2 f2(float a, float b) {
    F2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ F2 f2s(float a) { return f2(a, a); }
__device__ __forceinline__ float f2lo(F2 x) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x.v));
    return a;
}
__device__ __forceinline__ float f2hi(F2 x) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x.v));
    return b;
}
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
    F2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
    return d;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
    F2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
    F2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}
__device__ __forceinline__ F2 ex2x2(F2 x) { return f2(ex2(f2lo(x)), ex2(f2hi(x))); }
__device__ __forceinline__ F2 rcpx2(F2 x) { return f2(rcp(f2lo(x)), rcp(f2hi(x))); }

// Programmatic dependent launch: let the next kernel of the stream be
// scheduled as this one's CTAs retire, then wait until the previous kernel
// of the stream has finished and its writes are visible.  Nothing before
// this may read or write global memory (kernel parameters, tensor maps
// included, are not global memory).  Without the launch attribute both are
// no-ops.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 1 + e^-r, the denominator factor of sigmoid(r) = 1 / (1 + e^-r).
__device__ __forceinline__ float gate_den(float r) { return 1.f + ex2(-r * kLog2e); }

}  // namespace wkv
