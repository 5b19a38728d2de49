// wkv_chunk_ws.cuh -- warp-specialised persistent chunked-scan kernel.
//
// Same units, per-segment arithmetic and cross-chunk protocol as the kernel in
// wkv_chunk.cuh (see there), arranged as a pipeline inside each CTA:
//
//   warps 0..W-1  compute: pass 0/1 of a unit (segment summaries into shared
//                 memory), then pass 2 (outputs) once the unit's start state
//                 is known.
//   warps W, W+1  scan (alternating units): take the chunk summary from the
//                 aggregator, look back over the chunks before it (a window
//                 of four per round trip), hand the start state to the
//                 compute warps, then publish the state after the chunk.
//                 Before the summary is ready they already fold whatever the
//                 chunks before it have published, so the look-back usually
//                 costs nothing on the compute warps' path.
//   warp W+2      aggregator: folds the W segment summaries into the chunk
//                 summary and publishes it immediately.
//   warp W+3      producer (one lane): claims units from the ticket counter
//                 (or round-robin without a workspace) and issues their TMA
//                 copies (k, v, r tiles; w, u and the initial state as bulk
//                 copies) into a ring of S shared-memory stages.
//
// Hand-offs use mbarriers: full[s] (TMA bytes landed), aggready[s] (W segment
// summaries written), foldready[s] (chunk summary folded), xready[s] (start
// state written), empty[s] (W compute warps done with the stage).  Every wait
// is bounded in time.
#pragma once

#include "wkv_chunk.cuh"

namespace wkv {

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <typename IO, int V, bool GATE, int W, int LS, int S>
struct WsGeometry {
    static constexpr int CB = 32 * V;
    static constexpr int TT = W * LS;
    static constexpr int NARR = GATE ? 3 : 2;
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = TT * ROW;
    static constexpr uint32_t TILES = NARR * TILE;
    // per-channel parameters copied next to the tiles: w, u, and for the
    // first chunk of a sequence the initial state a, b, p
    static constexpr uint32_t PARAM = 5 * CB * sizeof(float);
    static constexpr uint32_t STAGE = TILES + PARAM;
    static constexpr uint32_t AGGBUF = W * V * 32 * sizeof(St);   // per stage
    static constexpr uint32_t XBUF = V * 32 * sizeof(St);         // per stage
    static constexpr uint32_t FOLDBUF = V * 32 * sizeof(St);      // per stage
    static constexpr uint32_t SMEM = S * (STAGE + AGGBUF + XBUF + FOLDBUF);
    static constexpr int SCAN = 2;                                // scan warps, alternating units
    static constexpr int THREADS = (W + SCAN + 2) * 32;
};

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
//
// Pass 0 works on raw keys: the key range (max, min) and the segment's
// running-max exponent q = max_i (k2_i + i w2) - (n-1) w2, which equals the
// recurrence p <- max(p - w2, k2) over the segment.  Pass 1 (fast path)
// scales every token by the largest key: one ex2 per token, whose argument
// fuses the base-2 conversion.
template <typename IO, int V, bool GATE, int W, int LS, bool FULL, bool PARAMS_IN_STAGE = true, bool CACHE = true>
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
            const F2 qa = fma2(ka, L2, iw);
            iw = add2(iw, W2);
            const F2 qb = two ? fma2(kb, L2, iw) : qa;
            iw = add2(iw, W2);
            qa0 = max3(qa0, f2lo(qa), f2lo(qb));
            qa1 = max3(qa1, f2hi(qa), f2hi(qb));
        }
    }
    const float nm1 = static_cast<float>(cx.nvalid - 1);
    const float q[2] = {qa0 - nm1 * cx.w2[0], qa1 - nm1 * cx.w2[1]};
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
        // keys too spread for one reference: the exact running-max recurrence
#pragma unroll
        for (int j = 0; j < V; ++j) seg[j] = st_identity();
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < cx.nvalid) {
                const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(srow + TILE + i * ROW));
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float k2 = (j == 0 ? f2lo(cx.kf[i]) : f2hi(cx.kf[i])) * kLog2e;
                    const float v1 = j == 0 ? f2lo(vv) : f2hi(vv);
                    const float pd = seg[j].p - cx.w2[j];
                    const float d2 = pd - k2;
                    const float e = ex2(-fabsf(d2));
                    if (d2 >= 0.f) {
                        seg[j].a = fmaf(e, v1, seg[j].a);
                        seg[j].b += e;
                        seg[j].p = pd;
                    } else {
                        seg[j].a = fmaf(e, seg[j].a, v1);
                        seg[j].b = fmaf(e, seg[j].b, 1.f);
                        seg[j].p = k2;
                    }
                }
            }
        }
    }
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
                    out[j] = lane_token(st[j].a, st[j].b, st[j].p, cx.w2[j], cx.u2[j], k2,
                                        j == 0 ? f2lo(vv) : f2hi(vv), gd, 1.f);
                }
                Ld::store(yp, out);
            }
            yp += C;
        }
    }
}

// (chunk, lane block, sequence, first channel) of a unit.
struct UnitCoord {
    int64_t chunk, lb, b, c0;
};

// Compute warps, first half of a unit: wait for its tiles, pass 0/1, hand
// the segment summary to the scan warp.  False at the end of the stream (or
// on a timeout).
template <typename IO, int V, bool GATE, int W, int LS, int S>
__device__ __forceinline__ bool compute_front(const ChunkArgs& A, int64_t it, unsigned char* smem, uint64_t* full,
                                              uint64_t* aggready, const int64_t* unitbuf, const UnitCoord* coord,
                                              St* aggbuf, SegCtx<V, LS>& cx) {
    using G = WsGeometry<IO, V, GATE, W, LS, S>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = static_cast<int>(it % S);
    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
    if (!mbar_wait(&full[s], ph, kCopyWaitNs)) {
        if (threadIdx.x == 0 && A.hdr != nullptr) record_timeout(A, -1);
        return false;
    }
    const int64_t u = unitbuf[s];
    if (u >= A.units) return false;
    const unsigned char* stage = smem + s * G::STAGE;
    St seg[V];
    const int64_t chunk = coord[s].chunk, b = coord[s].b, c = coord[s].c0 + lane * V;
    if ((chunk + 1) * G::TT <= A.T) seg_pass01<IO, V, GATE, W, LS, true>(A, chunk, b, c, stage, cx, seg);
    else seg_pass01<IO, V, GATE, W, LS, false>(A, chunk, b, c, stage, cx, seg);
    St* ab = aggbuf + static_cast<int64_t>(s) * W * V * 32;
#pragma unroll
    for (int j = 0; j < V; ++j) ab[(warp * V + j) * 32 + lane] = seg[j];
    __syncwarp();
    if (lane == 0) mbar_arrive(&aggready[s]);
    return true;
}

// Compute warps, second half: wait for the unit's start state, pass 2,
// release the stage.  False on a timeout.
template <typename IO, int V, bool GATE, int W, int LS, int S>
__device__ __forceinline__ bool compute_back(const ChunkArgs& A, int64_t it, unsigned char* smem, uint64_t* xready,
                                             uint64_t* empty, const int64_t* unitbuf, const UnitCoord* coord,
                                             const St* aggbuf, const St* xbuf, SegCtx<V, LS>& cx) {
    using G = WsGeometry<IO, V, GATE, W, LS, S>;
    constexpr int TT = G::TT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = static_cast<int>(it % S);
    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
    const bool ok = mbar_wait(&xready[s], ph, A.wait_limit_ns);
    if (!ok && threadIdx.x == 0 && A.hdr != nullptr) record_timeout(A, -1);
    const int64_t chunk = coord[s].chunk;
    if (ok && cx.nvalid > 0 && cx.cvalid) {
        const int64_t chunk_rows = min(static_cast<int64_t>(TT), A.T - chunk * TT);
        const St* ab = aggbuf + static_cast<int64_t>(s) * W * V * 32;
        const St* xb = xbuf + static_cast<int64_t>(s) * V * 32;
        St st[V], lp[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            st[j] = xb[j * 32 + lane];
            lp[j] = st_identity();
        }
        for (int sg = 0; sg < warp; ++sg) {
            const int len = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), chunk_rows - sg * LS)));
#pragma unroll
            for (int j = 0; j < V; ++j)
                lp[j] = st_combine(lp[j], ab[(sg * V + j) * 32 + lane], static_cast<float>(len) * cx.w2[j]);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) st[j] = st_combine(st[j], lp[j], static_cast<float>(warp * LS) * cx.w2[j]);
        const unsigned char* stage = smem + s * G::STAGE;
        if ((chunk + 1) * TT <= A.T) seg_pass2<IO, V, GATE, W, LS, true>(A, stage, cx, st);
        else seg_pass2<IO, V, GATE, W, LS, false>(A, stage, cx, st);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    return ok;
}

// Scan warps skip ring positions (each takes every SCAN-th), so the end of
// the stream can land on a position another warp owns: wait for a phase OR
// for the producer's end position to be at or before `it`.  1 = phase
// complete, 0 = end of stream, -1 = timed out.
__device__ __noinline__ int mbar_wait_or_end(uint64_t* bar, uint32_t parity, const volatile int64_t* endpos,
                                             int64_t it, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t n = 0; n < (1u << 26); ++n) {
        if (mbar_try_wait(bar, parity)) return 1;
        if (*endpos <= it) return 0;
        if ((n & 15u) == 15u && global_ns() - t0 > limit_ns) return -1;
    }
    return -1;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <typename IO, int V, bool GATE, int W, int LS, int S>
__global__ void __launch_bounds__(WsGeometry<IO, V, GATE, W, LS, S>::THREADS)
chunk_ws_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tr, const ChunkArgs A) {
    using G = WsGeometry<IO, V, GATE, W, LS, S>;
    constexpr int CB = G::CB;
    constexpr int TT = G::TT;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[S], empty[S], aggready[S], xready[S], foldready[S];
    __shared__ int64_t unitbuf[S];
    __shared__ UnitCoord coord[S];   // decoded by the producer: no divisions in the other warps
    __shared__ int64_t s_endpos;   // first ring position with no unit (set by the producer)
    __shared__ uint32_t s_epoch;
    St* aggbuf = reinterpret_cast<St*>(smem + S * G::STAGE);                 // [S][W][V][32]
    St* xbuf = reinterpret_cast<St*>(smem + S * (G::STAGE + G::AGGBUF));     // [S][V][32]
    St* foldbuf = reinterpret_cast<St*>(smem + S * (G::STAGE + G::AGGBUF + G::XBUF));  // [S][V][32]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool ticket = A.hdr != nullptr;
    constexpr int kProducer = W + G::SCAN + 1;
    constexpr int kAggregator = W + G::SCAN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], W);
            mbar_init(&aggready[s], W);
            mbar_init(&xready[s], 1);
            mbar_init(&foldready[s], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_epoch = ticket ? ld_relaxed_u32(&A.hdr->epoch) : 0u;
        s_endpos = INT64_MAX;
    }
    __syncthreads();
    const uint32_t epoch = s_epoch;
    volatile int64_t* endpos = &s_endpos;

    if (warp == kProducer) {
        // ---------------- producer ----------------
        if (lane == 0) {
            const int64_t lanes = A.B * A.C;
            for (int64_t it = 0;; ++it) {
                const int s = static_cast<int>(it % S);
                if (it >= S && !mbar_wait(&empty[s], static_cast<uint32_t>(((it / S) - 1) & 1), A.wait_limit_ns)) {
                    if (ticket) record_timeout(A, -1);
                    *endpos = it;
                    break;
                }
                const int64_t u = ticket ? static_cast<int64_t>(atomicAdd(&A.hdr->ticket, 1u))
                                         : static_cast<int64_t>(blockIdx.x) + it * gridDim.x;
                unitbuf[s] = u;
                if (u >= A.units) {
                    *endpos = it;           // end of the stream for this CTA
                    mbar_arrive(&full[s]);
                    break;
                }
                const int64_t chunk = u / A.nLB, lb = u % A.nLB;
                const int64_t c0 = (lb % A.nCB) * CB;
                const int64_t b = lb / A.nCB;
                coord[s] = UnitCoord{chunk, lb, b, c0};
                // channels of this block inside C; a multiple of 4 because C is
                const uint32_t pbytes = static_cast<uint32_t>(min(static_cast<int64_t>(CB), A.C - c0)) * 4u;
                const bool first = chunk == 0 && A.s_in != nullptr;
                unsigned char* st = smem + s * G::STAGE;
                float* prm = reinterpret_cast<float*>(st + G::TILES);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect_tx(&full[s], G::TILES + pbytes * (first ? 5u : 2u));
                const int x = static_cast<int>(c0), y = static_cast<int>(chunk * TT), z = static_cast<int>(b);
                tma_load_3d(st, &tk, x, y, z, &full[s]);
                tma_load_3d(st + G::TILE, &tv, x, y, z, &full[s]);
                if (GATE) tma_load_3d(st + 2 * G::TILE, &tr, x, y, z, &full[s]);
                bulk_load(prm, A.w + c0, pbytes, &full[s]);
                bulk_load(prm + CB, A.u + c0, pbytes, &full[s]);
                if (first) {
                    const float* si = A.s_in + b * A.C + c0;
                    bulk_load(prm + 2 * CB, si, pbytes, &full[s]);
                    bulk_load(prm + 3 * CB, si + lanes, pbytes, &full[s]);
                    bulk_load(prm + 4 * CB, si + 2 * lanes, pbytes, &full[s]);
                }
            }
        }
    } else if (warp == kAggregator) {
        // ---------------- aggregator ----------------
        // Folds each unit's segment summaries into the chunk summary and
        // publishes it at once, so the chunks after it can look past this one
        // without waiting for its inclusive state.
        for (int64_t it = 0;; ++it) {
            const int s = static_cast<int>(it % S);
            const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
            if (!mbar_wait(&full[s], ph, kCopyWaitNs)) {
                if (lane == 0 && ticket) record_timeout(A, -1);
                break;
            }
            const int64_t u = unitbuf[s];
            if (u >= A.units) break;
            const int64_t chunk = coord[s].chunk;
            const int64_t c = coord[s].c0 + lane * V;
            const bool cvalid = c < A.C;
            const int64_t chunk_rows = min(static_cast<int64_t>(TT), A.T - chunk * TT);
            const float* prm = reinterpret_cast<const float*>(smem + s * G::STAGE + G::TILES);
            float w2[V];
#pragma unroll
            for (int j = 0; j < V; ++j) w2[j] = cvalid ? prm[lane * V + j] * kLog2e : 1.f;
            const bool ok = mbar_wait(&aggready[s], ph, A.wait_limit_ns);
            if (!ok && lane == 0 && ticket) record_timeout(A, -1);
            St agg[V];
            const St* ab = aggbuf + static_cast<int64_t>(s) * W * V * 32;
#pragma unroll
            for (int j = 0; j < V; ++j) agg[j] = st_identity();
            for (int sg = 0; sg < W; ++sg) {
                const int len = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), chunk_rows - sg * LS)));
#pragma unroll
                for (int j = 0; j < V; ++j) agg[j] = st_combine(agg[j], ab[(sg * V + j) * 32 + lane], static_cast<float>(len) * w2[j]);
            }
            St* fb = foldbuf + static_cast<int64_t>(s) * V * 32;
#pragma unroll
            for (int j = 0; j < V; ++j) fb[j * 32 + lane] = agg[j];
            __syncwarp();
            if (lane == 0) mbar_arrive(&foldready[s]);
            if (!ok) break;
            if (chunk > 0 && chunk < A.nchunks - 1) publish<V>(A.aggw + u * CB, agg, epoch, kKindAgg, lane);
        }
    } else if (warp >= W) {
        // ---------------- scan (warps W .. W+SCAN-1, alternating units) ----
        // Ring positions it = r, r+SCAN, ... with S a multiple of SCAN, so a
        // scan warp sees every phase of its stages in order.
        static_assert(S % G::SCAN == 0, "ring depth must be a multiple of the scan warps");
        const int64_t lanes = A.B * A.C;
        for (int64_t it = warp - W;; it += G::SCAN) {
            const int s = static_cast<int>(it % S);
            const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
            const int got = mbar_wait_or_end(&full[s], ph, endpos, it, kCopyWaitNs);
            if (got < 0 && lane == 0 && ticket) record_timeout(A, -1);
            if (got <= 0) break;
            const int64_t u = unitbuf[s];
            if (u >= A.units) break;
            const int64_t chunk = coord[s].chunk, lb = coord[s].lb;
            const int64_t b = coord[s].b;
            const int64_t c = coord[s].c0 + lane * V;
            const bool cvalid = c < A.C;
            const int64_t chunk_rows = min(static_cast<int64_t>(TT), A.T - chunk * TT);
            const bool last = chunk == A.nchunks - 1;
            const float* prm = reinterpret_cast<const float*>(smem + s * G::STAGE + G::TILES);
            float w2[V];
            St sin[V];
#pragma unroll
            for (int j = 0; j < V; ++j) {
                w2[j] = cvalid ? prm[lane * V + j] * kLog2e : 1.f;
                if (chunk == 0 && A.s_in != nullptr && cvalid)
                    sin[j] = St{prm[4 * CB + lane * V + j] * kLog2e, prm[2 * CB + lane * V + j],
                                prm[3 * CB + lane * V + j]};
                else
                    sin[j] = st_identity();
            }
            LookState<V> L;
            look_init<V>(L, chunk);
            if (chunk == 0) {
#pragma unroll
                for (int j = 0; j < V; ++j) L.x[j] = sin[j];
                L.done = true;
            } else {
                // fold whatever is already published, without waiting
                while (!L.done && lookback_round<V, TT>(A, lb, epoch, w2, sin, L, lane)) {
                }
            }
            bool ok = mbar_wait(&foldready[s], ph, A.wait_limit_ns);
            St agg[V];
            const St* fb = foldbuf + static_cast<int64_t>(s) * V * 32;
#pragma unroll
            for (int j = 0; j < V; ++j) agg[j] = fb[j * 32 + lane];
            if (ok && !L.done) ok = lookback_finish<V, TT>(A, lb, epoch, w2, sin, L, lane);
            if (!ok) {
                if (lane == 0 && ticket) record_timeout(A, u);
                const float nan = __int_as_float(0x7fc00000);
#pragma unroll
                for (int j = 0; j < V; ++j) L.x[j] = St{nan, nan, nan};
            }
            St* xb = xbuf + static_cast<int64_t>(s) * V * 32;
#pragma unroll
            for (int j = 0; j < V; ++j) xb[j * 32 + lane] = L.x[j];
            __syncwarp();
            if (lane == 0) mbar_arrive(&xready[s]);
            St incl[V];
#pragma unroll
            for (int j = 0; j < V; ++j) incl[j] = st_combine(L.x[j], agg[j], static_cast<float>(chunk_rows) * w2[j]);
            if (A.nchunks > 1 && !last) publish<V>(A.incw + u * CB, incl, epoch, kKindInc, lane);
            if (last && A.s_out != nullptr && cvalid) {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const int64_t li = b * A.C + c + j;
                    A.s_out[li] = incl[j].a;
                    A.s_out[lanes + li] = incl[j].b;
                    A.s_out[2 * lanes + li] = incl[j].p * kLn2;
                }
            }
            if (!ok) break;
        }
    } else {
        // ---------------- compute ----------------
        // Lag-1 pipeline: pass 0/1 of unit it+1 runs before pass 2 of unit
        // it, so every unit's segment summaries (and hence its chunk summary)
        // are out before this CTA waits for the start state of the previous
        // unit.  Two register contexts, unrolled by two.
        SegCtx<V, LS> cxa, cxb;
        bool end_a = !compute_front<IO, V, GATE, W, LS, S>(A, 0, smem, full, aggready, unitbuf, coord, aggbuf, cxa);
        for (int64_t it = 0; !end_a; it += 2) {
            const bool end_b = !compute_front<IO, V, GATE, W, LS, S>(A, it + 1, smem, full, aggready, unitbuf, coord, aggbuf, cxb);
            if (!compute_back<IO, V, GATE, W, LS, S>(A, it, smem, xready, empty, unitbuf, coord, aggbuf, xbuf, cxa) || end_b) break;
            end_a = !compute_front<IO, V, GATE, W, LS, S>(A, it + 2, smem, full, aggready, unitbuf, coord, aggbuf, cxa);
            if (!compute_back<IO, V, GATE, W, LS, S>(A, it + 1, smem, xready, empty, unitbuf, coord, aggbuf, xbuf, cxb)) break;
        }
    }
    __syncthreads();
    if (ticket && threadIdx.x == 0) finish_launch(A, gridDim.x);
}

}  // namespace wkv
