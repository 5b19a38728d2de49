// wkv_seq.cuh -- sequential-over-T forward kernel: one thread owns V lanes.
// (y == NULL: only the state is wanted; no output is written.)
//
// The plain log-space recurrence (running max, one ex2 per max) walked token
// by token, the parallel-mode loop of "並列学習の定式化" with the max
// bookkeeping of "対数空間計算による数値安定性".  Each warp reads one row
// (one t) of 32*V consecutive channels per access, so loads are coalesced.
// It needs no workspace; it is the path for short sequences with many lanes
// and the fallback for shapes the chunked kernel does not take.
#pragma once

#include "wkv_common.cuh"

namespace wkv {

template <typename IO, int V, bool GATE>
__global__ void __launch_bounds__(256)
seq_forward_kernel(int64_t B, int64_t T, int64_t C, const float* __restrict__ w,
                   const float* __restrict__ u, const IO* __restrict__ k,
                   const IO* __restrict__ v, const IO* __restrict__ r,
                   const float* __restrict__ s_in, IO* __restrict__ y, float* __restrict__ s_out) {
    using Ld = Vec<IO, V>;
    const int64_t groups = (C / V) * B;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (g >= groups) return;
    const int64_t cg = C / V;
    const int64_t b = g / cg;
    const int64_t c = (g % cg) * V;
    const int64_t lanes = B * C;
    const int64_t lane0 = b * C + c;

    float wj[V], uj[V], sa[V], sb[V], sp[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        wj[j] = __ldg(w + c + j);
        uj[j] = __ldg(u + c + j);
        if (s_in) {
            sa[j] = s_in[lane0 + j];
            sb[j] = s_in[lanes + lane0 + j];
            sp[j] = s_in[2 * lanes + lane0 + j];
        } else {
            sa[j] = 0.f;
            sb[j] = 0.f;
            sp[j] = kFreshP;
        }
    }
    const IO* kp = k + b * T * C + c;
    const IO* vp = v + b * T * C + c;
    const IO* rp = GATE ? r + b * T * C + c : nullptr;
    IO* yp = y + b * T * C + c;
    for (int64_t t = 0; t < T; ++t) {
        const auto kr = Ld::load(kp);
        const auto vr = Ld::load(vp);
        typename Ld::raw rr{};
        if (GATE) rr = Ld::load(rp);
        float out[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float gd = GATE ? gate_den(Ld::get(rr, j)) : 1.f;
            out[j] = lane_token(sa[j], sb[j], sp[j], wj[j], uj[j], Ld::get(kr, j), Ld::get(vr, j), gd,
                                kLog2e);
        }
        if (y != nullptr) Ld::store(yp, out);
        kp += C;
        vp += C;
        if (GATE) rp += C;
        yp += C;
    }
    if (s_out) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            s_out[lane0 + j] = sa[j];
            s_out[lanes + lane0 + j] = sb[j];
            s_out[2 * lanes + lane0 + j] = sp[j];
        }
    }
}

// Fold of segment summaries: state_out = the state after n consecutive
// segments of len[0..n-1] tokens entered from state_in (or the empty state),
// where summary j is segment j's own state from the empty state.  Each fold
// is the scan combine of the segment summaries (max form, one ex2).  One
// thread per lane; states in natural-log units at the boundary.
constexpr int kCombineMax = 64;
struct CombineLens {
    int64_t len[kCombineMax];
};

__global__ void __launch_bounds__(256)
state_combine_kernel(int64_t B, int64_t C, int n, const float* __restrict__ w, CombineLens lens,
                     const float* __restrict__ seg, const float* __restrict__ s_in, float* __restrict__ s_out) {
    const int64_t lanes = B * C;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= lanes) return;
    const float w2 = __ldg(w + i % C) * kLog2e;
    St s = st_identity();
    if (s_in != nullptr) s = St{s_in[2 * lanes + i] * kLog2e, s_in[i], s_in[lanes + i]};
    for (int j = 0; j < n; ++j) {
        const float* x = seg + static_cast<int64_t>(j) * 3 * lanes;
        const St xs{x[2 * lanes + i] * kLog2e, x[i], x[lanes + i]};
        s = st_combine(s, xs, static_cast<float>(lens.len[j]) * w2);
    }
    s_out[i] = s.a;
    s_out[lanes + i] = s.b;
    s_out[2 * lanes + i] = s.p * kLn2;
}

// T == 0: state_out = state_in (or the empty state).
__global__ void copy_state_kernel(int64_t lanes, const float* __restrict__ s_in,
                                  float* __restrict__ s_out) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= lanes) return;
    if (s_in) {
        const float a = s_in[i], b = s_in[lanes + i], p = s_in[2 * lanes + i];
        s_out[i] = a;
        s_out[lanes + i] = b;
        s_out[2 * lanes + i] = p;
    } else {
        s_out[i] = 0.f;
        s_out[lanes + i] = 0.f;
        s_out[2 * lanes + i] = kFreshP;
    }
}

}  // namespace wkv
