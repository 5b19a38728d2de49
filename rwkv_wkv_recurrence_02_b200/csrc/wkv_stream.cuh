// wkv_stream.cuh -- stream kernel: one chunk of a carried stream.
//
// A chunk of a long sequence (the skill page "rwkv-architecture", "Process
// million-token sequences": a document fed chunk by chunk with the state
// carried) is a call with few lane blocks and at most a few thousand tokens.
// Its outputs need the state the previous chunk leaves, but most of its work
// does not: the scan that "並列学習の定式化" (article "RWKVアーキテクチャ徹底
// 解説") says the parallel mode performs splits the chunk into segments whose
// summaries (states reached from the empty state) and their prefixes are
// independent of the state entering the chunk.  This kernel does all of that
// first and only then touches the entering state:
//
//   load      k rows straight into registers (each thread: its two channels
//             of its segment); the v (and r) tile of the part by one TMA copy
//             into shared memory, w and u by bulk copies.
//   pass 0/1  segment summary per warp (fixed-scale fast path, exact
//             running-max fallback), from k in registers and v in shared
//             memory.
//   fold      summaries of the warps before each warp (shared memory), the
//             part's summary, and through distributed shared memory the
//             summaries of the cluster's earlier parts: every warp ends with
//             the summary of all tokens from the chunk start to its segment.
//   -------- the entering state is needed from here on --------
//   state     each warp reads state_in for its channels and folds it with
//             its prefix (one combine).
//   pass 2    outputs: k from registers, v (and r) from shared memory; the
//             per-token exponentials are recomputed rather than held, which
//             keeps the kernel small enough that the next chunk's CTAs fit
//             beside this chunk's.
//   state_out the last part's warp W-1 writes it, after a cluster barrier at
//             which every CTA has read state_in (state_out may be state_in).
//
// One thread block cluster of P = ceil(T / PT) CTAs per 64-channel lane block,
// one CTA per part of PT = W * LS tokens.  With the launch flag `early` (the
// caller declares that k, v, r, w, u are not written by work still running
// on the stream) everything above the line runs before griddepcontrol.wait,
// so under programmatic dependent launch it overlaps the previous call.
// Otherwise the kernel waits at entry like the others.  No workspace, no wait
// on another cluster; every thread reaches both cluster barriers on every
// path (a copy that does not land turns into NaN outputs).
#pragma once

#include "wkv_cluster.cuh"

namespace wkv {

template <typename IO, bool GATE, int W, int LS>
struct StreamGeometry {
    static constexpr int V = 2;
    static constexpr int CB = 32 * V;
    static constexpr int PT = W * LS;
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = PT * ROW;                 // one array's part tile
    static constexpr int NT = GATE ? 2 : 1;                    // tiles in shared memory: v (, r)
    static constexpr uint32_t PARAM = 2 * CB * sizeof(float);  // w, u of the lane block
    static constexpr uint32_t SMEM = NT * TILE + PARAM;
    static constexpr int THREADS = W * 32;
};

template <typename IO>
__device__ __forceinline__ typename Vec<IO, 2>::raw ldg_pair(const IO* p) {
    return Vec<IO, 2>::load(p);
}

template <typename IO, bool GATE, int W, int LS, int MINB>
__global__ void __launch_bounds__(W * 32, MINB)
stream_forward_kernel(const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tr,
                      const ChunkArgs A) {
    using G = StreamGeometry<IO, GATE, W, LS>;
    constexpr int V = 2;
    constexpr int CB = G::CB;
    constexpr int PT = G::PT;
    constexpr int ROW = G::ROW;
    using Raw = typename Vec<IO, V>::raw;
    using Ld = Vec<IO, V>;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full;
    __shared__ St s_seg[W][V][32];                   // segment summaries of the part
    __shared__ __align__(16) float4 s_slot[V][32];   // the part's summary, read by later parts
    __shared__ St s_x[V][32];                        // summary of the chunk before this part
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = cluster_ctarank();             // part index along T
    const int64_t last = static_cast<int64_t>(cluster_nctarank()) - 1;
    const int64_t lb = cluster_id_x();               // lane block
    const int64_t bs = lb / A.nCB;
    const int x0 = static_cast<int>((lb % A.nCB) * CB);
    const int64_t c = x0 + lane * V;
    const bool cvalid = c < A.C;                     // C is even: both channels or neither
    const bool early = A.early != 0;
    const float nan = __int_as_float(0x7fc00000);

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tv);
        if (GATE) prefetch_tensormap(&tr);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- load: v (, r) tiles and w, u by TMA; k rows into registers ----
    const int64_t t_part = q * PT;
    const int part_len = static_cast<int>(min(static_cast<int64_t>(PT), A.T - t_part));
    float* prm = reinterpret_cast<float*>(smem + G::NT * G::TILE);
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const uint32_t pbytes = static_cast<uint32_t>(min(static_cast<int64_t>(CB), A.C - x0)) * 4u;
        mbar_expect_tx(&full, G::NT * G::TILE + 2u * pbytes);
        tma_load_3d(smem, &tv, x0, static_cast<int>(t_part), static_cast<int>(bs), &full);
        if (GATE) tma_load_3d(smem + G::TILE, &tr, x0, static_cast<int>(t_part), static_cast<int>(bs), &full);
        bulk_load(prm, A.w + x0, pbytes, &full);
        bulk_load(prm + CB, A.u + x0, pbytes, &full);
    }
    const int64_t t_seg = t_part + warp * LS;
    const int nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), A.T - t_seg)));
    Raw kr[LS];
    {
        const IO* kp = static_cast<const IO*>(A.k) + (bs * A.T + t_seg) * A.C + c;
#pragma unroll
        for (int i = 0; i < LS; ++i) kr[i] = (cvalid && i < nvalid) ? ldg_pair<IO>(kp + i * A.C) : Raw{};
    }
    __syncthreads();   // the barrier's initialisation is visible to every waiter
    const bool got = mbar_wait(&full, 0u, kCopyWaitNs);

    float w2[V], u2[V], dk[V], eu[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        w2[j] = cvalid ? prm[lane * V + j] * kLog2e : 1.f;
        u2[j] = cvalid ? prm[CB + lane * V + j] * kLog2e : 0.f;
        dk[j] = ex2(-w2[j]);
        eu[j] = ex2(u2[j]);
    }
    const unsigned char* vrow = smem + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));
    const F2 L2 = f2s(kLog2e);

    // ---- pass 0: key range and the segment's running-max exponent q ----
    // q = max_i (k2_i - (n-1-i) w2), each candidate from one product
    float kx[V] = {-3.0e38f, -3.0e38f}, kn[V] = {3.0e38f, 3.0e38f}, qm[V] = {-3.0e38f, -3.0e38f};
#pragma unroll
    for (int i = 0; i < LS; ++i) {
        if (i < nvalid) {
            const F2 kk = raw_pair<IO>(kr[i]);
            const float o = static_cast<float>(i - (nvalid - 1));
            const F2 cand = fma2(kk, L2, f2(o * w2[0], o * w2[1]));
            kx[0] = fmaxf(kx[0], f2lo(kk));
            kx[1] = fmaxf(kx[1], f2hi(kk));
            kn[0] = fminf(kn[0], f2lo(kk));
            kn[1] = fminf(kn[1], f2hi(kk));
            qm[0] = fmaxf(qm[0], f2lo(cand));
            qm[1] = fmaxf(qm[1], f2hi(cand));
        }
    }
    float kmax[V], kmin[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        kmax[j] = kx[j] * kLog2e;
        kmin[j] = kn[j] * kLog2e;
    }
    const bool fast1 = (kmax[0] - kmin[0] + fabsf(u2[0]) <= kFastSpan) &&
                       (kmax[1] - kmin[1] + fabsf(u2[1]) <= kFastSpan);

    // ---- pass 1: segment summary ----
    St seg[V];
    if (nvalid == 0 || !got) {
        seg[0] = seg[1] = st_identity();
    } else if (fast1) {
        const F2 KM = f2(-kmax[0], -kmax[1]);
        const F2 DK = f2(dk[0], dk[1]);
        F2 n = f2s(0.f), db = f2s(0.f);
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (i < nvalid) {
                const F2 ek = ex2x2(fma2(raw_pair<IO>(kr[i]), L2, KM));
                const F2 ekv = mul2(ek, raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW)));
                n = fma2(n, DK, ekv);
                db = fma2(db, DK, ek);
            }
        }
        const float sc0 = ex2(kmax[0] - qm[0]), sc1 = ex2(kmax[1] - qm[1]);
        seg[0] = St{qm[0], f2lo(n) * sc0, f2lo(db) * sc0};
        seg[1] = St{qm[1], f2hi(n) * sc1, f2hi(db) * sc1};
    } else {
        // keys too spread for one reference: the exact running-max recurrence
        // with its exponent held as pb - m w2 (see lane_token_pm)
        float pb[V], m[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            seg[j] = st_identity();
            pb[j] = seg[j].p;
            m[j] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (i < nvalid) {
                const F2 kk = raw_pair<IO>(kr[i]);
                const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW));
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                    const float v1 = j == 0 ? f2lo(vv) : f2hi(vv);
                    const float pd = fmaf(-(m[j] + 1.f), w2[j], pb[j]);
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
        for (int j = 0; j < V; ++j) seg[j].p = fmaf(-m[j], w2[j], pb[j]);
    }
#pragma unroll
    for (int j = 0; j < V; ++j) s_seg[warp][j][lane] = seg[j];
    const bool ok = __syncthreads_and(got);

    // ---- fold: summary of the part's segments before this warp's own ----
    St pre[V];
#pragma unroll
    for (int j = 0; j < V; ++j) pre[j] = st_identity();
    for (int sg = 0; sg < warp; ++sg) {
        const int len = max(0, min(LS, part_len - sg * LS));
#pragma unroll
        for (int j = 0; j < V; ++j) pre[j] = st_combine(pre[j], s_seg[sg][j][lane], static_cast<float>(len) * w2[j]);
    }
    const int pre_len = min(warp * LS, part_len);
    St agg[V];   // warp W-1: the part's summary
    if (warp == W - 1) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            agg[j] = ok ? st_combine(pre[j], seg[j], static_cast<float>(nvalid) * w2[j]) : St{nan, nan, nan};
            s_slot[j][lane] = make_float4(agg[j].p, agg[j].a, agg[j].b, 0.f);
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    // the parts before this one (all full), from the chunk start
    if (warp == W - 1) {
        St xs[V];
#pragma unroll
        for (int j = 0; j < V; ++j) xs[j] = st_identity();
        for (int64_t r = 0; r < q; ++r) {
#pragma unroll
            for (int j = 0; j < V; ++j)
                xs[j] = st_combine(xs[j], ld_cluster_state(&s_slot[j][lane], static_cast<uint32_t>(r)),
                                   static_cast<float>(PT) * w2[j]);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) s_x[j][lane] = xs[j];
    }
    __syncthreads();
    // summary of every token from the chunk start to this warp's segment
    St z[V];
#pragma unroll
    for (int j = 0; j < V; ++j) z[j] = st_combine(s_x[j][lane], pre[j], static_cast<float>(pre_len) * w2[j]);
    St chunk_sum[V];   // the last part's warp W-1: summary of the whole chunk
    if (warp == W - 1 && q == last) {
#pragma unroll
        for (int j = 0; j < V; ++j) chunk_sum[j] = st_combine(s_x[j][lane], agg[j], static_cast<float>(part_len) * w2[j]);
    }

    // -------- the entering state from here on --------
    if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t lanes = A.B * A.C;
    St sin[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sin[j] = st_identity();
        if (A.s_in != nullptr && cvalid) {
            const int64_t li = bs * A.C + c + j;
            sin[j] = St{A.s_in[2 * lanes + li] * kLog2e, A.s_in[li], A.s_in[lanes + li]};
        }
    }
    // every CTA has read state_in (and its remote reads are done) once all
    // arrive here; the last part writes state_out after that
    cluster_arrive_release();
    if (warp == W - 1 && q == last) {
        cluster_wait_acquire();
        if (A.s_out != nullptr && cvalid) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const St so = ok ? st_combine(sin[j], chunk_sum[j], static_cast<float>(A.T) * w2[j]) : St{nan, nan, nan};
                const int64_t li = bs * A.C + c + j;
                A.s_out[li] = so.a;
                A.s_out[lanes + li] = so.b;
                A.s_out[2 * lanes + li] = so.p * kLn2;
            }
        }
    }

    // ---- pass 2: outputs from the segment's start state ----
    if (ok && nvalid > 0 && cvalid && A.y != nullptr) {
        St st[V];
#pragma unroll
        for (int j = 0; j < V; ++j) st[j] = st_combine(sin[j], z[j], static_cast<float>(t_seg) * w2[j]);
        bool fast2 = fast1;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const bool near = st[j].p >= kmax[j] - kFastState;
            const bool negligible = st[j].p < kmax[j] - 1.5f * kFastState && st[j].b <= 16777216.f;
            fast2 = fast2 && (st[j].p - kmin[j] + fabsf(u2[j]) <= kFastState) && (near || negligible);
        }
        IO* yp = static_cast<IO*>(A.y) + (bs * A.T + t_seg) * A.C + c;
        const unsigned char* rrow = vrow + G::TILE;
        if (fast2) {
            float nr[V], ss[V];
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float R = fmaxf(kmax[j], st[j].p);
                nr[j] = -R;
                ss[j] = ex2(st[j].p - R);
            }
            const F2 NR = f2(nr[0], nr[1]);
            const F2 EU = f2(eu[0], eu[1]);
            const F2 DK = f2(dk[0], dk[1]);
            const F2 NL = f2s(-kLog2e);
            F2 n = f2(st[0].a * ss[0], st[1].a * ss[1]);
            F2 db = f2(st[0].b * ss[0], st[1].b * ss[1]);
#pragma unroll
            for (int i = 0; i < LS; ++i) {
                if (i < nvalid) {
                    const F2 ek = ex2x2(fma2(raw_pair<IO>(kr[i]), L2, NR));
                    const F2 ekv = mul2(ek, raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW)));
                    const F2 num = fma2(EU, ekv, n);
                    F2 den = fma2(EU, ek, db);
                    if (GATE) {
                        const F2 g = ex2x2(mul2(raw_pair<IO>(*reinterpret_cast<const Raw*>(rrow + i * ROW)), NL));
                        den = fma2(den, g, den);
                    }
                    const F2 y = mul2(num, rcpx2(den));
                    n = fma2(n, DK, ekv);
                    db = fma2(db, DK, ek);
                    const float out[2] = {f2lo(y), f2hi(y)};
                    Ld::store(yp + i * A.C, out);
                }
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
                if (i < nvalid) {
                    const F2 kk = raw_pair<IO>(kr[i]);
                    const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW));
                    F2 rv = f2s(0.f);
                    if (GATE) rv = raw_pair<IO>(*reinterpret_cast<const Raw*>(rrow + i * ROW));
                    float out[V];
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        const float gd = GATE ? gate_den(j == 0 ? f2lo(rv) : f2hi(rv)) : 1.f;
                        const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                        out[j] = lane_token_pm(st[j].a, st[j].b, pb[j], m[j], w2[j], u2[j], k2,
                                               j == 0 ? f2lo(vv) : f2hi(vv), gd);
                    }
                    Ld::store(yp + i * A.C, out);
                }
            }
        }
    } else if (!ok && nvalid > 0 && cvalid && A.y != nullptr) {
        // a copy that did not land: NaN outputs, never stale values
        IO* yp = static_cast<IO*>(A.y) + (bs * A.T + t_seg) * A.C + c;
        const float out[2] = {nan, nan};
        for (int i = 0; i < nvalid; ++i) Ld::store(yp + i * A.C, out);
    }
    if (!ok && threadIdx.x == 0) {
        if (A.hdr != nullptr) record_timeout(A, q * A.nLB + lb);
        // let the copy land before the CTA's shared memory is released
        mbar_wait(&full, 0u, kCopyWaitNs);
    }
    if (!(warp == W - 1 && q == last)) cluster_wait_acquire();
}

}  // namespace wkv
