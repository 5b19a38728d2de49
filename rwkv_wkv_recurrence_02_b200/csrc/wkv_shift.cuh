// wkv_shift.cuh -- token shift: every token's input mixed with the previous
// token's before the R, K, V projections ("トークンシフト：秘密の要素"),
// out_m[t] = mu_m * x[t] + (1 - mu_m) * x[t-1], for nmix mixes at once.
//
// A thread owns V consecutive channels (16 bytes of one row) of one sequence
// over TS consecutive tokens: it reads the row before its first token once
// (x_prev for the first tokens of the sequence), keeps the previous row in
// registers, and writes nmix output rows per token.  A whole unit issues its
// TS row loads before using the first (6% faster than loading each row when
// it is needed, on the 14B layer shape); a partial unit at the end of a
// sequence loads row by row.  Units run channel group
// fastest, so a warp's accesses to every array are contiguous.  The thread
// that owns a sequence's first tokens also writes x_last, after reading
// x_prev, so x_last may be x_prev itself.
#pragma once

#include "wkv_common.cuh"

namespace wkv {

constexpr int kShiftMaxMix = 8;
// mixes whose mu a whole unit keeps in registers (more take the per-token loop)
constexpr int kShiftRegMix = 4;

template <typename IO, int V>
struct ShiftVec;

// load: read-only path (x, mu); load_rw: plain load (x_prev, which this
// kernel may overwrite as x_last); load_raw + widen_raw: a read-only load
// kept packed in registers and widened when it is used
template <>
struct ShiftVec<float, 1> {
    using Raw = float;
    static __device__ __forceinline__ Raw load_raw(const float* p) { return __ldg(p); }
    static __device__ __forceinline__ void widen_raw(Raw v, float* o) { o[0] = v; }
    static __device__ __forceinline__ void load(const float* p, float* o) { o[0] = __ldg(p); }
    static __device__ __forceinline__ void load_rw(const float* p, float* o) { o[0] = *p; }
    static __device__ __forceinline__ void store(float* p, const float* o) { *p = o[0]; }
};
template <>
struct ShiftVec<float, 4> {
    using Raw = float4;
    static __device__ __forceinline__ Raw load_raw(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
    static __device__ __forceinline__ void widen_raw(Raw v, float* o) { o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w; }
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
    }
    static __device__ __forceinline__ void load_rw(const float* p, float* o) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* o) {
        *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
    }
};
template <>
struct ShiftVec<__nv_bfloat16, 1> {
    using Raw = __nv_bfloat16;
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16* p) { return __ldg(p); }
    static __device__ __forceinline__ void widen_raw(Raw v, float* o) { o[0] = __bfloat162float(v); }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) { o[0] = __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ void load_rw(const __nv_bfloat16* p, float* o) { o[0] = __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* o) { *p = __float2bfloat16_rn(o[0]); }
};
template <>
struct ShiftVec<__nv_bfloat16, 8> {
    using Raw = uint4;
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
    static __device__ __forceinline__ void widen_raw(Raw v, float* o) { widen(v, o); }
    static __device__ __forceinline__ void widen(uint4 v, float* o) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* o) {
        widen(__ldg(reinterpret_cast<const uint4*>(p)), o);
    }
    static __device__ __forceinline__ void load_rw(const __nv_bfloat16* p, float* o) {
        widen(*reinterpret_cast<const uint4*>(p), o);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* o) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// One unit: V channels of sequence b over tokens [t0, t1).  The unit with
// the sequence's first tokens also writes x_last: the last input row (read
// again unless it lies in the unit's own tokens).
template <typename IO, int V, int TS>
__global__ void __launch_bounds__(256)
token_shift_kernel(int64_t B, int64_t T, int64_t C, int nmix, const IO* __restrict__ x, const float* __restrict__ mu,
                   const IO* x_prev, IO* __restrict__ out, IO* x_last) {
    const int64_t cg = C / V;
    const int64_t nT = (T + TS - 1) / TS;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    pdl_begin();
    if (g >= B * nT * cg) return;
    const int64_t c = (g % cg) * V;
    const int64_t rest = g / cg;
    const int64_t tc = rest % nT;
    const int64_t b = rest / nT;
    const int64_t t0 = tc * TS;
    const int64_t t1 = t0 + TS < T ? t0 + TS : T;

    float prev[V];
    if (t0 > 0) {
        ShiftVec<IO, V>::load(x + (b * T + t0 - 1) * C + c, prev);
    } else if (x_prev != nullptr) {
        ShiftVec<IO, V>::load_rw(x_prev + b * C + c, prev);
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) prev[j] = 0.f;
    }
    const int64_t plane = B * T * C;
    if (t1 - t0 == TS && nmix <= kShiftRegMix) {
        // a whole unit: all TS rows in flight before the first is used, and
        // the mixes' mu of the unit's channels held in registers
        typename ShiftVec<IO, V>::Raw raw[TS];
#pragma unroll
        for (int i = 0; i < TS; ++i) raw[i] = ShiftVec<IO, V>::load_raw(x + (b * T + t0 + i) * C + c);
        float mm[kShiftRegMix][V];
#pragma unroll
        for (int m = 0; m < kShiftRegMix; ++m) {
            if (m < nmix) {
                ShiftVec<float, V == 8 ? 4 : V>::load(mu + m * C + c, mm[m]);
                if constexpr (V == 8) ShiftVec<float, 4>::load(mu + m * C + c + 4, mm[m] + 4);
            }
        }
#pragma unroll
        for (int i = 0; i < TS; ++i) {
            float cur[V];
            ShiftVec<IO, V>::widen_raw(raw[i], cur);
#pragma unroll
            for (int m = 0; m < kShiftRegMix; ++m) {
                if (m < nmix) {
                    float o[V];
#pragma unroll
                    for (int j = 0; j < V; ++j) o[j] = fmaf(mm[m][j], cur[j], (1.f - mm[m][j]) * prev[j]);
                    ShiftVec<IO, V>::store(out + m * plane + (b * T + t0 + i) * C + c, o);
                }
            }
#pragma unroll
            for (int j = 0; j < V; ++j) prev[j] = cur[j];
        }
    } else
    for (int64_t t = t0; t < t1; ++t) {
        float cur[V];
        ShiftVec<IO, V>::load(x + (b * T + t) * C + c, cur);
#pragma unroll
        for (int m = 0; m < kShiftMaxMix; ++m) {
            if (m < nmix) {
                // mu of the unit's channels (L1-resident after the first token)
                float mm[V], o[V];
                ShiftVec<float, V == 8 ? 4 : V>::load(mu + m * C + c, mm);
                if constexpr (V == 8) ShiftVec<float, 4>::load(mu + m * C + c + 4, mm + 4);
#pragma unroll
                for (int j = 0; j < V; ++j) o[j] = fmaf(mm[j], cur[j], (1.f - mm[j]) * prev[j]);
                ShiftVec<IO, V>::store(out + m * plane + (b * T + t) * C + c, o);
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) prev[j] = cur[j];
    }
    if (tc == 0 && x_last != nullptr) {
        float last[V];
        if (t1 == T) {
#pragma unroll
            for (int j = 0; j < V; ++j) last[j] = prev[j];
        } else {
            ShiftVec<IO, V>::load(x + (b * T + T - 1) * C + c, last);
        }
        ShiftVec<IO, V>::store(x_last + b * C + c, last);
    }
}

}  // namespace wkv
