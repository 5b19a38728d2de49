// wkv_backward.cuh -- reverse mode (gradients) of the WKV operator.
//
// The pages say the parallel mode is what trains the model ("並列学習の定式化")
// but print no gradient; this is the chain rule through the recurrence of
// "リカレント定式化" in the output-then-update order, per lane (0-based t,
// natural units, lam = e^{-w}):
//
//   N_{t+1} = lam N_t + e^{k_t} v_t,   D_{t+1} = lam D_t + e^{k_t}
//   wkv_t = (N_t + e^{u+k_t} v_t) / (D_t + e^{u+k_t}),   y_t = g_t wkv_t
//
// With gN_t, gD_t = dL/dN_t, dL/dD_t and c_t = (dnum_t, dden_t) =
// (g_t dy_t, -g_t dy_t wkv_t) / den_t, the gradients obey the reverse
// recurrence gN_t = c_t + lam gN_{t+1} (and gD likewise), and
//
//   dv_t = dnum_t e^{u+k_t} + gN_{t+1} e^{k_t}
//   dk_t = (dnum_t v_t + dden_t) e^{u+k_t} + (gN_{t+1} v_t + gD_{t+1}) e^{k_t}
//   du = sum (dnum_t v_t + dden_t) e^{u+k_t},  dw = -lam sum (gN_{t+1} N_t + gD_{t+1} D_t)
//   dr_t = dy_t wkv_t g_t (1 - g_t)
//
// Everything is kept in base-2 max form like the forward: a forward state is
// (p, a, b) with N = a 2^p, and a reverse state is (x, A, B) with gN = A 2^x,
// gD = B 2^x, so st_combine folds both.  Every product of a forward weight
// and a reverse weight is formed as one 2^(sum of exponents), which stays in
// range.
//
// Work split: one CTA per lane block (64 channels of one sequence) walks its
// 64-token chunks from the last to the first, carrying the reverse state; a
// producer warp streams the k, v, dy (and r) tiles of each chunk, and the
// forward state entering the chunk (from the checkpoint sweep), into a ring
// of S shared-memory stages with TMA.  Warp s of the W compute warps owns the
// chunk's segment s of LS tokens:
//
//   sweep 0   the segment's forward summary from the empty state; the warps'
//             summaries meet in shared memory, and each warp's entering
//             forward state F is the chunk's checkpoint followed by the
//             summaries before its own.
//   sweep A   forward from F: outputs, c_t (kept in registers as
//             (exponent, dnum, dden)), dr_t, du, and the segment's reverse
//             summary (the reverse state the segment alone produces at its
//             start).
//   fold      each warp's reverse state at its segment end is the chunk's
//             carried reverse state followed by the reverse summaries of the
//             segments after its own; warp 0 also forms the carry for the
//             chunk before.
//   sweep B   backward from there: dk_t, dv_t; the registers of c_t now keep
//             the reverse state after token t.
//   sweep C   forward from F again: dw.
//
// The checkpoint sweep is the lane-resident forward kernel in its checkpoint
// mode; a last kernel sums the per-lane-block dw, du partials per channel.
#pragma once

#include "wkv_lane.cuh"

namespace wkv {

struct BwdArgs {
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const void* r;
    const void* dy;
    const float* s_in;
    const float* ds_out;
    void* dk;
    void* dv;
    void* dr;
    float* ds_in;
    const St* ckpt;     // [nchunks + 1][nLB][CB], see ChunkArgs::ckpt
    float* part;        // [2][nLB][CB]: dw, du of each lane block (zeroed by the caller)
    WsHeader* hdr;      // null when every CTA owns whole lane blocks
    Word* incw;         // [nLB][CB] reverse states handed between neighbouring CTAs
    int64_t B, T, C;
    int64_t nCB, nLB, nchunks;
    uint64_t wait_limit_ns;
};

template <typename IO, bool GATE, int W, int LS, int S>
struct BwdGeometry {
    static constexpr int V = 2;
    static constexpr int CB = 32 * V;
    static constexpr int TT = W * LS;
    static constexpr int NARR = GATE ? 4 : 3;   // k, v, dy (, r)
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = TT * ROW;
    static constexpr uint32_t CKPT = CB * sizeof(St);
    static constexpr uint32_t STAGE = NARR * TILE + CKPT;
    static constexpr uint32_t SMEM = S * STAGE;
    static constexpr int THREADS = (W + 1) * 32;
};

// Fixed-scale fast path limits (base 2): the segment's keys plus |u| span at
// most kBwdFastSpan, and the entering state, |u| and the carried reverse
// state lie within kBwdFastState of the segment's scale.
constexpr float kBwdFastSpan = 96.f;
constexpr float kBwdFastState = 60.f;

// Output of the current (undecayed) state and token, base 2: wkv, 1/den and
// the scale o of num and den (num = num_hat 2^o), and e2 = 2^(u2+k2-o).
// One ex2: exactly one of the two scale factors is 1.
__device__ __forceinline__ void bwd_out(const St& s, float u2, float k2, float v, float& wkv, float& inv_den,
                                        float& o, float& e2) {
    const float uk = u2 + k2;
    const float diff = s.p - uk;
    const float e = ex2(-fabsf(diff));
    float num, den;
    if (diff >= 0.f) {
        o = s.p;
        e2 = e;
        num = fmaf(e, v, s.a);
        den = s.b + e;
    } else {
        o = uk;
        e2 = 1.f;
        num = fmaf(e, s.a, v);
        den = fmaf(e, s.b, 1.f);
    }
    inv_den = rcp(den);
    wkv = num * inv_den;
}

// State update of the forward recurrence, base 2, one ex2.
__device__ __forceinline__ void bwd_update(St& s, float w2, float k2, float v) {
    const float pd = s.p - w2;
    const float diff = pd - k2;
    const float e = ex2(-fabsf(diff));
    if (diff >= 0.f) {
        s.a = fmaf(e, v, s.a);
        s.b += e;
        s.p = pd;
    } else {
        s.a = fmaf(e, s.a, v);
        s.b = fmaf(e, s.b, 1.f);
        s.p = k2;
    }
}

__device__ __forceinline__ void finish_bwd_launch(const BwdArgs& A, uint32_t ctas) {
    const uint32_t before = atomicAdd(&A.hdr->done, 1u);
    if (before == ctas - 1u) {
        A.hdr->done = 0u;
        A.hdr->ticket = 0u;
        __threadfence();
        atomicAdd(&A.hdr->epoch, 1u);
    }
}

// Reverse state handed over by the CTA that walked the later chunks of lane
// block lb (one 16-byte word per channel; bounded wait, NaN on expiry).
template <int V>
__device__ __noinline__ void bwd_wait_carry(const Word* incw, WsHeader* hdr, uint64_t limit_ns, int64_t lb,
                                            uint32_t epoch, St* out) {
    constexpr int CB = 32 * V;
    const int lane = threadIdx.x & 31;
    const Word* src = incw + lb * CB + lane * V;
    const uint64_t t0 = global_ns();
    unsigned sleep_ns = 32;
    for (;;) {
        Word wv[V];
        bool mine = true;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            wv[j] = ld_word(src + j);
            mine = mine && wv[j].tag == word_tag(epoch, kKindInc);
        }
        if (__all_sync(0xffffffffu, mine)) {
#pragma unroll
            for (int j = 0; j < V; ++j) out[j] = word_state(wv[j]);
            return;
        }
        if (global_ns() - t0 > limit_ns) {
            if (lane == 0) {
                atomicOr(&hdr->error, kErrTimeout);
                atomicExch(&hdr->err_unit, static_cast<uint32_t>(lb));
            }
            const float nan = __int_as_float(0x7fc00000);
#pragma unroll
            for (int j = 0; j < V; ++j) out[j] = St{nan, nan, nan};
            return;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 256) sleep_ns <<= 1;
    }
}

template <typename IO, bool GATE, int W, int LS, int S, int MAXREG>
__global__ void __launch_bounds__(BwdGeometry<IO, GATE, W, LS, S>::THREADS) __maxnreg__(MAXREG)
lane_backward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tdy, const __grid_constant__ CUtensorMap tr,
                     const BwdArgs A) {
    using G = BwdGeometry<IO, GATE, W, LS, S>;
    constexpr int V = G::V;
    constexpr int CB = G::CB;
    constexpr int TT = G::TT;
    using Raw = typename Vec<IO, V>::raw;
    using Ld = Vec<IO, V>;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[S], empty[S];
    __shared__ St s_fseg[W][V][32];     // forward summaries of the segments
    __shared__ St s_rseg[W][V][32];     // reverse summaries of the segments
    __shared__ St s_gcarry[2][V][32];   // reverse state at the end of a chunk, by chunk parity
    __shared__ float s_red[2][W][V][32];
    __shared__ LaneRange s_range;       // this CTA's share of the lane-major chunk order
    __shared__ uint32_t s_epoch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        prefetch_tensormap(&tdy);
        if (GATE) prefetch_tensormap(&tr);
    }
    pdl_begin();
    if (threadIdx.x == 0) {
        s_range.init(A.nLB, A.nchunks, blockIdx.x, gridDim.x, A.hdr == nullptr);
        s_epoch = A.hdr != nullptr ? ld_relaxed_u32(&A.hdr->epoch) : 0u;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], W);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const LaneRange& R = s_range;
    const uint32_t epoch = s_epoch;
    const int64_t nch = A.nchunks;

    if (warp == W) {
        // ---------------- producer: each item's chunks from the last to the first ----------------
        if (lane == 0) {
            int64_t it = 0, issued = 0;
            bool stop = false;
            for (int item = 0; item < R.count && !stop; ++item) {
                int64_t lb, c0, c1;
                bool to_prev, from_next;
                R.item_back(item, lb, c0, c1, to_prev, from_next);
                const int x0 = static_cast<int>((lb % A.nCB) * CB), z = static_cast<int>(lb / A.nCB);
                for (int64_t chunk = c1 - 1; chunk >= c0; --chunk, ++it) {
                    const int s = static_cast<int>(it % S);
                    if (it >= S &&
                        !mbar_wait(&empty[s], static_cast<uint32_t>(((it / S) - 1) & 1), A.wait_limit_ns)) {
                        stop = true;
                        break;
                    }
                    unsigned char* st = smem + s * G::STAGE;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_expect_tx(&full[s], G::NARR * G::TILE + G::CKPT);
                    const int y = static_cast<int>(chunk * TT);
                    tma_load_3d(st, &tk, x0, y, z, &full[s]);
                    tma_load_3d(st + G::TILE, &tv, x0, y, z, &full[s]);
                    tma_load_3d(st + 2 * G::TILE, &tdy, x0, y, z, &full[s]);
                    if (GATE) tma_load_3d(st + 3 * G::TILE, &tr, x0, y, z, &full[s]);
                    bulk_load(st + G::NARR * G::TILE, A.ckpt + (chunk * A.nLB + lb) * CB, G::CKPT, &full[s]);
                    ++issued;
                }
            }
            // every copy issued lands before this warp (and so the CTA) exits
            for (int64_t q = issued > S ? issued - S : 0; q < issued; ++q)
                mbar_wait(&full[q % S], static_cast<uint32_t>((q / S) & 1), kCopyWaitNs);
        }
        return;
    }

    // ---------------- compute ----------------
    const int64_t lanes = A.B * A.C;
    // the sizes the forward kernels' segment pass reads
    ChunkArgs ca{};
    ca.T = A.T;
    ca.C = A.C;
    int64_t it = 0;
    bool ok = true;
    for (int item = 0; item < R.count && ok; ++item) {
        int64_t lb, c0, c1;
        bool to_prev, from_next;
        R.item_back(item, lb, c0, c1, to_prev, from_next);
        const int64_t bs = lb / A.nCB;
        const int64_t c = (lb % A.nCB) * CB + lane * V;
        const bool cvalid = c < A.C;
        float w2[V], u2[V], lam[V], wv[V], uv[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            wv[j] = cvalid ? __ldg(A.w + c + j) : 1.f;
            uv[j] = cvalid ? __ldg(A.u + c + j) : 0.f;
            w2[j] = cvalid ? wv[j] * kLog2e : 1.f;
            u2[j] = cvalid ? uv[j] * kLog2e : 0.f;
            lam[j] = ex2(-w2[j]);
        }
        // reverse state after the item's last chunk
        if (warp == 0) {
            St g0[V] = {st_identity(), st_identity()};
            if (from_next) {
                bwd_wait_carry<V>(A.incw, A.hdr, A.wait_limit_ns, lb, epoch, g0);
            } else if (A.ds_out != nullptr && cvalid) {
                // the end of the sequence: dL/d(a_T, b_T) of the returned state
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const St fin = A.ckpt[(nch * A.nLB + lb) * CB + lane * V + j];
                    const int64_t li = bs * A.C + c + j;
                    g0[j] = St{-fin.p, A.ds_out[li], A.ds_out[lanes + li]};
                }
            }
#pragma unroll
            for (int j = 0; j < V; ++j) s_gcarry[it & 1][j][lane] = g0[j];
        }
        float dw_acc[V] = {0.f, 0.f}, du_acc[V] = {0.f, 0.f};
        for (int64_t chunk = c1 - 1; chunk >= c0; --chunk, ++it) {
            const int s = static_cast<int>(it % S);
            const int par = static_cast<int>(it & 1);
            const bool got = mbar_wait(&full[s], static_cast<uint32_t>((it / S) & 1), kCopyWaitNs);
            const unsigned char* stage = smem + s * G::STAGE;
            const int64_t t_seg = chunk * TT + warp * LS;
            const int n = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), A.T - t_seg)));
            const unsigned char* srow = stage + warp * LS * G::ROW + lane * V * static_cast<int>(sizeof(IO));
            auto row = [&](int arr, int i) -> F2 {
                return raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + arr * G::TILE + i * G::ROW));
            };
            // ---- sweep 0: forward summary and key range of the segment (the
            // forward kernels' pass 0/1: fixed-scale fast path, exact fallback) ----
            St fs[V] = {st_identity(), st_identity()};
            float kmax[V] = {-3.0e38f, -3.0e38f}, kmin[V] = {3.0e38f, 3.0e38f};
            if (got) {
                SegCtx<V, LS> cx;
                cx.cvalid = cvalid;
                set_params<V, LS>(cx, wv, uv);
                if ((chunk + 1) * TT <= A.T) seg_pass01<IO, V, false, W, LS, true, false, false>(ca, chunk, bs, c, stage, cx, fs);
                else seg_pass01<IO, V, false, W, LS, false, false, false>(ca, chunk, bs, c, stage, cx, fs);
                if (n > 0) {
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        kmax[j] = cx.kmax[j];
                        kmin[j] = cx.kmin[j];
                    }
                }
#pragma unroll
                for (int j = 0; j < V; ++j) s_fseg[warp][j][lane] = fs[j];
            }
            // a copy that did not land stops every compute warp together
            if (!named_sync_and(1, W * 32, got)) {
                if (threadIdx.x == 0 && A.hdr != nullptr) atomicOr(&A.hdr->error, kErrTimeout);
                ok = false;
                break;
            }
            // entering forward state of the segment
            const St* ck = reinterpret_cast<const St*>(stage + G::NARR * G::TILE) + lane * V;
            St F[V] = {ck[0], ck[1]};
            for (int sg = 0; sg < warp; ++sg) {
                const int len = static_cast<int>(max(static_cast<int64_t>(0),
                                                     min(static_cast<int64_t>(LS), A.T - (chunk * TT + sg * LS))));
#pragma unroll
                for (int j = 0; j < V; ++j) F[j] = st_combine(F[j], s_fseg[sg][j][lane], static_cast<float>(len) * w2[j]);
            }
            // Fixed-scale fast path of this lane's two channels: every weight of
            // the segment is taken relative to R = max(largest key, entering
            // exponent), so each token costs one ex2 and the recurrences are
            // plain FMAs.  It needs the keys (with the bonus) to span at most
            // 96 in base 2 and the entering state not to dwarf them; the exact
            // per-token max form covers the rest.
            float R[V], eu[V];
            bool fastA = true;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                R[j] = fmaxf(kmax[j], F[j].p);
                eu[j] = ex2(u2[j]);
                fastA = fastA && (kmax[j] - kmin[j] + fabsf(u2[j]) <= kBwdFastSpan) && (F[j].p - kmax[j] <= kBwdFastState) &&
                        (fabsf(u2[j]) <= kBwdFastState);
            }
            // ---- sweep A: outputs, c_t, dr, du, reverse summary ----
            // registers per token, the lane's two channels packed: fast
            // (2^(k-R), dnum 2^R, dden 2^R); exact (-o_t, dnum 2^o_t, dden 2^o_t)
            F2 co[LS], cn[LS], cd[LS];
            St rs[V];
            const F2 L2 = f2s(kLog2e), ONE = f2s(1.f), MONE = f2s(-1.f);
            const F2 LAM = f2(lam[0], lam[1]), EU = f2(eu[0], eu[1]), NR = f2(-R[0], -R[1]);
            {
                IO* drp = GATE ? static_cast<IO*>(A.dr) + (bs * A.T + t_seg) * A.C + c : nullptr;
                if (fastA) {
                    const float s00 = ex2(F[0].p - R[0]), s01 = ex2(F[1].p - R[1]);
                    F2 nh = f2(F[0].a * s00, F[1].a * s01), dh = f2(F[0].b * s00, F[1].b * s01);
                    F2 pw = ONE, rn = f2s(0.f), rd = f2s(0.f), dus = f2s(0.f);
#pragma unroll
                    for (int i = 0; i < LS; ++i) {
                        if (i < n) {
                            const F2 vv = row(1, i), dd = row(2, i);
                            const F2 ek = ex2x2(fma2(row(0, i), L2, NR));
                            const F2 eek = mul2(EU, ek);
                            const F2 inv = rcpx2(add2(dh, eek));
                            const F2 wkv = mul2(fma2(eek, vv, nh), inv);
                            F2 dn = mul2(dd, inv);
                            if (GATE) {
                                const F2 g = rcpx2(add2(ONE, ex2x2(mul2(row(3, i), f2s(-kLog2e)))));
                                dn = mul2(dn, g);
                                if (cvalid) {
                                    const F2 dr2 = mul2(mul2(dd, wkv), mul2(g, fma2(g, MONE, ONE)));
                                    const float drv[V] = {f2lo(dr2), f2hi(dr2)};
                                    Ld::store(drp, drv);
                                }
                            }
                            const F2 dd2 = mul2(mul2(dn, wkv), MONE);
                            dus = fma2(fma2(dn, vv, dd2), eek, dus);
                            co[i] = ek;
                            cn[i] = dn;
                            cd[i] = dd2;
                            rn = fma2(pw, dn, rn);
                            rd = fma2(pw, dd2, rd);
                            pw = mul2(pw, LAM);
                            nh = fma2(LAM, nh, mul2(ek, vv));
                            dh = fma2(LAM, dh, ek);
                        }
                        if (GATE) drp += A.C;
                    }
                    du_acc[0] += f2lo(dus);
                    du_acc[1] += f2hi(dus);
                    rs[0] = St{-R[0], f2lo(rn), f2lo(rd)};
                    rs[1] = St{-R[1], f2hi(rn), f2hi(rd)};
                } else {
                    St S_[V] = {F[0], F[1]};
                    rs[0] = rs[1] = st_identity();
#pragma unroll
                    for (int i = 0; i < LS; ++i) {
                        if (i < n) {
                            const F2 kk = row(0, i), vv = row(1, i), dd = row(2, i);
                            F2 rr = f2s(0.f);
                            if (GATE) rr = row(3, i);
                            float drv[V], to[V], tn[V], td[V];
#pragma unroll
                            for (int j = 0; j < V; ++j) {
                                const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                                const float vj = j == 0 ? f2lo(vv) : f2hi(vv);
                                const float dyj = j == 0 ? f2lo(dd) : f2hi(dd);
                                float wkv, inv, o, e2;
                                bwd_out(S_[j], u2[j], k2, vj, wkv, inv, o, e2);
                                float g = 1.f;
                                if (GATE) {
                                    g = rcp(1.f + ex2(-(j == 0 ? f2lo(rr) : f2hi(rr)) * kLog2e));
                                    drv[j] = dyj * wkv * g * (1.f - g);
                                }
                                const float dn = g * dyj * inv;
                                const float dd2 = -dn * wkv;
                                du_acc[j] = fmaf(fmaf(dn, vj, dd2), e2, du_acc[j]);
                                to[j] = -o;
                                tn[j] = dn;
                                td[j] = dd2;
                                rs[j] = st_combine(rs[j], St{-o - static_cast<float>(i) * w2[j], dn, dd2}, 0.f);
                                bwd_update(S_[j], w2[j], k2, vj);
                            }
                            co[i] = f2(to[0], to[1]);
                            cn[i] = f2(tn[0], tn[1]);
                            cd[i] = f2(td[0], td[1]);
                            if (GATE && cvalid) Ld::store(drp, drv);
                        }
                        if (GATE) drp += A.C;
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < V; ++j) s_rseg[warp][j][lane] = rs[j];
            named_sync(1, W * 32);
            // ---- fold: reverse state at the end of this warp's segment ----
            St gend[V] = {s_gcarry[par][0][lane], s_gcarry[par][1][lane]};
            for (int sg = W - 1; sg > warp; --sg) {
                const int len = static_cast<int>(max(static_cast<int64_t>(0),
                                                     min(static_cast<int64_t>(LS), A.T - (chunk * TT + sg * LS))));
#pragma unroll
                for (int j = 0; j < V; ++j) gend[j] = st_combine(gend[j], s_rseg[sg][j][lane], static_cast<float>(len) * w2[j]);
            }
            // the fast reverse walk also needs the carried reverse state in range at scale 2^-R
            bool fastB = fastA;
#pragma unroll
            for (int j = 0; j < V; ++j) fastB = fastB && (gend[j].p + R[j] <= kBwdFastState);
            // ---- sweep B: dk, dv from the reverse walk ----
            {
                St g0[V];
                IO* dkp = static_cast<IO*>(A.dk) + (bs * A.T + t_seg) * A.C + c;
                IO* dvp = static_cast<IO*>(A.dv) + (bs * A.T + t_seg) * A.C + c;
                if (fastB) {
                    const float sc0 = ex2(gend[0].p + R[0]), sc1 = ex2(gend[1].p + R[1]);
                    F2 gN = f2(gend[0].a * sc0, gend[1].a * sc1), gD = f2(gend[0].b * sc0, gend[1].b * sc1);
#pragma unroll
                    for (int i = LS - 1; i >= 0; --i) {
                        if (i < n) {
                            const F2 vv = row(1, i);
                            const F2 ek = co[i], eek = mul2(EU, ek);
                            const F2 dv2 = fma2(cn[i], eek, mul2(gN, ek));
                            const F2 dk2 = fma2(fma2(cn[i], vv, cd[i]), eek, mul2(fma2(gN, vv, gD), ek));
                            const F2 nN = fma2(LAM, gN, cn[i]);
                            const F2 nD = fma2(LAM, gD, cd[i]);
                            // keep the reverse state after token t for sweep C
                            cn[i] = gN;
                            cd[i] = gD;
                            gN = nN;
                            gD = nD;
                            if (cvalid) {
                                const float dkv[V] = {f2lo(dk2), f2hi(dk2)}, dvv[V] = {f2lo(dv2), f2hi(dv2)};
                                Ld::store(dkp + i * A.C, dkv);
                                Ld::store(dvp + i * A.C, dvv);
                            }
                        }
                    }
                    g0[0] = St{-R[0], f2lo(gN), f2lo(gD)};
                    g0[1] = St{-R[1], f2hi(gN), f2hi(gD)};
                } else {
                    St g[V] = {gend[0], gend[1]};
#pragma unroll
                    for (int i = LS - 1; i >= 0; --i) {
                        if (i < n) {
                            const F2 kk = row(0, i), vv = row(1, i);
                            float dkv[V], dvv[V], to[V], tn[V], td[V];
#pragma unroll
                            for (int j = 0; j < V; ++j) {
                                const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                                const float vj = j == 0 ? f2lo(vv) : f2hi(vv);
                                const float coj = j == 0 ? f2lo(co[i]) : f2hi(co[i]);
                                const float cnj = j == 0 ? f2lo(cn[i]) : f2hi(cn[i]);
                                const float cdj = j == 0 ? f2lo(cd[i]) : f2hi(cd[i]);
                                // c_t as a max-form state, whichever way sweep A kept it
                                const float cx = fastA ? -R[j] : coj;
                                const float e2 = fastA ? eu[j] * coj : ex2(u2[j] + k2 + cx);
                                const float ek = ex2(g[j].p + k2);                 // e^{k_t} gN_{t+1} / A
                                dvv[j] = fmaf(cnj, e2, g[j].a * ek);
                                dkv[j] = fmaf(fmaf(cnj, vj, cdj), e2, fmaf(g[j].a, vj, g[j].b) * ek);
                                const St gn = st_combine(g[j], St{cx, cnj, cdj}, w2[j]);
                                // keep the reverse state after token t for sweep C
                                to[j] = g[j].p;
                                tn[j] = g[j].a;
                                td[j] = g[j].b;
                                g[j] = gn;
                            }
                            co[i] = f2(to[0], to[1]);
                            cn[i] = f2(tn[0], tn[1]);
                            cd[i] = f2(td[0], td[1]);
                            if (cvalid) {
                                Ld::store(dkp + i * A.C, dkv);
                                Ld::store(dvp + i * A.C, dvv);
                            }
                        }
                    }
                    g0[0] = g[0];
                    g0[1] = g[1];
                }
                if (warp == 0) {
#pragma unroll
                    for (int j = 0; j < V; ++j) s_gcarry[par ^ 1][j][lane] = g0[j];
                    if (chunk == c0 && to_prev) publish<V>(A.incw + lb * CB, g0, epoch, kKindInc, lane);
                    if (chunk == 0 && A.ds_in != nullptr && cvalid) {
                        // gradient of the initial state: dL/da0 = gN_0 e^{p0}, ...
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            const int64_t li = bs * A.C + c + j;
                            float a0 = 0.f, b0 = 0.f, p2 = kFreshP2;
                            if (A.s_in != nullptr) {
                                a0 = A.s_in[li];
                                b0 = A.s_in[lanes + li];
                                p2 = A.s_in[2 * lanes + li] * kLog2e;
                            }
                            const float sc = ex2(g0[j].p + p2);
                            const float ga = g0[j].a * sc, gb = g0[j].b * sc;
                            A.ds_in[li] = ga;
                            A.ds_in[lanes + li] = gb;
                            A.ds_in[2 * lanes + li] = fmaf(a0, ga, b0 * gb);
                        }
                    }
                }
            }
            // ---- sweep C: dw from the forward states and the reverse states ----
            if (fastB) {
                const float s00 = ex2(F[0].p - R[0]), s01 = ex2(F[1].p - R[1]);
                F2 nh = f2(F[0].a * s00, F[1].a * s01), dh = f2(F[0].b * s00, F[1].b * s01), dws = f2s(0.f);
#pragma unroll
                for (int i = 0; i < LS; ++i) {
                    if (i < n) {
                        dws = fma2(cn[i], nh, fma2(cd[i], dh, dws));
                        nh = fma2(LAM, nh, mul2(co[i], row(1, i)));
                        dh = fma2(LAM, dh, co[i]);
                    }
                }
                dw_acc[0] += f2lo(dws);
                dw_acc[1] += f2hi(dws);
            } else {
                St S_[V] = {F[0], F[1]};
#pragma unroll
                for (int i = 0; i < LS; ++i) {
                    if (i < n) {
                        const F2 kk = row(0, i), vv = row(1, i);
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            const float coj = j == 0 ? f2lo(co[i]) : f2hi(co[i]);
                            const float cnj = j == 0 ? f2lo(cn[i]) : f2hi(cn[i]);
                            const float cdj = j == 0 ? f2lo(cd[i]) : f2hi(cd[i]);
                            const float z = fmaf(cnj, S_[j].a, cdj * S_[j].b) * ex2(coj + S_[j].p);
                            dw_acc[j] += z;
                            bwd_update(S_[j], w2[j], (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e,
                                       j == 0 ? f2lo(vv) : f2hi(vv));
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (!ok) break;
        // ---- this item's share of dw, du for its lane block ----
#pragma unroll
        for (int j = 0; j < V; ++j) {
            s_red[0][warp][j][lane] = -lam[j] * dw_acc[j];
            s_red[1][warp][j][lane] = du_acc[j];
        }
        named_sync(1, W * 32);
        if (warp == 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                float sw = 0.f, su = 0.f;
                for (int q = 0; q < W; ++q) {
                    sw += s_red[0][q][j][lane];
                    su += s_red[1][q][j][lane];
                }
                // at most two items (a head and a tail) share a lane block,
                // and two additions onto zero commute exactly
                atomicAdd(A.part + lb * CB + lane * V + j, sw);
                atomicAdd(A.part + (A.nLB + lb) * CB + lane * V + j, su);
            }
        }
    }
    if (warp == 0 && lane == 0 && A.hdr != nullptr) finish_bwd_launch(A, gridDim.x);
}

// dw[c], du[c]: sums of the lane blocks' partials over the sequences.
__global__ void bwd_reduce_kernel(const float* part, int64_t B, int64_t C, int64_t nCB, float* dw, float* du) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= C) return;
    const int64_t nLB = B * nCB, cb = c / 64, o = c % 64;
    float sw = 0.f, su = 0.f;
    for (int64_t b = 0; b < B; ++b) {
        sw += part[(b * nCB + cb) * 64 + o];
        su += part[(nLB + b * nCB + cb) * 64 + o];
    }
    dw[c] = sw;
    du[c] = su;
}

// T == 0: the returned state is the given one, so its gradient passes
// through; dw = du = 0 are set by the caller.
__global__ void bwd_passthrough_kernel(int64_t lanes, const float* s_in, const float* ds_out, float* ds_in) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= lanes) return;
    const float ga = ds_out != nullptr ? ds_out[i] : 0.f;
    const float gb = ds_out != nullptr ? ds_out[lanes + i] : 0.f;
    const float a0 = s_in != nullptr ? s_in[i] : 0.f, b0 = s_in != nullptr ? s_in[lanes + i] : 0.f;
    ds_in[i] = ga;
    ds_in[lanes + i] = gb;
    ds_in[2 * lanes + i] = fmaf(a0, ga, b0 * gb);
}

}  // namespace wkv
