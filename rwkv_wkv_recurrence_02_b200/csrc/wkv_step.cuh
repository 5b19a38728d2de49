// wkv_step.cuh -- batched decode step: one token for L layers x B sequences.
//
// RNN mode of "二重性：Transformerモード vs RNNモード": the same token update
// as the forward kernels, applied once, with the state streamed from and back
// to HBM in place.  A thread owns V consecutive channels of one (layer, batch)
// row; a warp's accesses to every array are contiguous.  Launched as a
// programmatic dependent of the stream's previous kernel, so that a chain of
// small calls (one per layer) overlaps each launch with the previous drain.
#pragma once

#include "wkv_common.cuh"

namespace wkv {

template <typename IO, int V, bool GATE>
__global__ void __launch_bounds__(256)
step_kernel(int64_t L, int64_t B, int64_t C, const float* __restrict__ w,
            const float* __restrict__ u, const IO* __restrict__ k, const IO* __restrict__ v,
            const IO* __restrict__ r, float* __restrict__ state, IO* __restrict__ y) {
    using Ld = Vec<IO, V>;
    using Lf = Vec<float, V>;
    const int64_t cg = C / V;
    const int64_t total = L * B * cg;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    pdl_begin();
    if (g >= total) return;
    const int64_t row = g / cg;          // (l, b)
    const int64_t c = (g % cg) * V;
    const int64_t l = row / B;
    const int64_t b = row % B;
    const int64_t lanes = B * C;
    const int64_t io = row * C + c;       // (L, B, C) index
    float* sp = state + l * 3 * lanes + b * C + c;

    const auto wr = Lf::load(w + l * C + c);
    const auto ur = Lf::load(u + l * C + c);
    const auto kr = Ld::load(k + io);
    const auto vr = Ld::load(v + io);
    typename Ld::raw rr{};
    if (GATE) rr = Ld::load(r + io);
    float sa[V], sb[V], sq[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sa[j] = sp[j];
        sb[j] = sp[lanes + j];
        sq[j] = sp[2 * lanes + j];
    }
    float out[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const float gd = GATE ? gate_den(Ld::get(rr, j)) : 1.f;
        out[j] = lane_token(sa[j], sb[j], sq[j], Lf::get(wr, j), Lf::get(ur, j), Ld::get(kr, j),
                            Ld::get(vr, j), gd, kLog2e);
    }
    Ld::store(y + io, out);
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sp[j] = sa[j];
        sp[lanes + j] = sb[j];
        sp[2 * lanes + j] = sq[j];
    }
}

}  // namespace wkv
