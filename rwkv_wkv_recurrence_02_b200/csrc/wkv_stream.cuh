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
//   load      the k, v (and r) tiles of the part by one TMA copy each into
//             shared memory, w and u by bulk copies.
//   pass 0/1  segment summary per warp (fixed-scale fast path, exact
//             running-max fallback).
//   fold      summaries of the warps before each warp (shared memory), the
//             part's summary, and through distributed shared memory the
//             summaries of the cluster's earlier parts: every warp ends with
//             the summary of all tokens from the chunk start to its segment.
//   -------- the entering state is needed from here on --------
//   state     each warp reads state_in for its channels and folds it with
//             its prefix (one combine).
//   pass 2    outputs; the per-token exponentials are recomputed rather than
//             held in registers, which keeps the kernel small enough that
//             most of the next chunk's CTAs fit beside this chunk's.  Each
//             output overwrites the v entry it was
//             computed from, and every warp stores its finished rows with one
//             TMA copy (rows and channels outside the arrays are clipped).
//   state_out the last part's warp W-1 writes it, after a cluster barrier at
//             which every CTA has read state_in (state_out may be state_in).
//
// Full parts (every segment LS tokens long) run a copy of the passes without
// per-token bounds tests; a part that ends inside T takes the checked copy.
//
// One thread block cluster of P = ceil(T / PT) CTAs per 64-channel lane block,
// one CTA per part of PT = W * LS tokens.  The launch covers tokens
// [A.t0, A.t0 + T) of the arrays (A.t0 > 0 when one long call runs as a
// chain of launches).  With the launch flag `early` (the
// caller declares that k, v, r, w, u are not written by work still running
// on the stream) everything above the line runs before griddepcontrol.wait,
// so under programmatic dependent launch it overlaps the previous call.
// Otherwise the kernel waits at entry like the others.  No workspace, no wait
// on another cluster; every thread reaches both cluster barriers on every
// path (a copy that does not land turns into NaN outputs).
//
// Chunk chains (A.chain set): the last part's warp W-1 publishes the state
// after the chunk as tagged words (tag = A.chain_out, the next call's
// position in the chain) right after writing state_out, before pass 2.  A call that
// continues a chain (A.chain_in > 0) does not wait for the previous kernel
// to end: one warp per CTA polls for the words tagged with its position
// (bounded in time), and one CTA waits for the previous kernel before it
// exits, so the stream's kernels still end in order.  Its outputs then
// overlap the previous call's outputs, and the chain's serial part is only
// the fold of the entering state.  Programmatic launch starts a kernel only
// once every CTA of the previous one has started, so the CTAs a call waits
// on are resident and the wait ends.
#pragma once

#include "wkv_cluster.cuh"

namespace wkv {

// unroll depth of the per-token loops: deep enough to overlap the shared
// memory loads and MUFU latencies, shallow enough that the code of the three
// passes stays resident in the instruction cache
constexpr int kStreamUnroll = 16;

template <typename IO, bool GATE, int W, int LS>
struct StreamGeometry {
    static constexpr int V = 2;
    static constexpr int CB = 32 * V;
    static constexpr int PT = W * LS;
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = PT * ROW;                 // one array's part tile
    static constexpr int NT = GATE ? 3 : 2;                    // tiles in shared memory: k, v (, r)
    static constexpr uint32_t PARAM = 2 * CB * sizeof(float);  // w, u of the lane block
    static constexpr uint32_t SMEM = NT * TILE + PARAM;
    static constexpr int THREADS = W * 32;
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Per-thread values of one segment between the passes.
template <int LS>
struct StreamSeg {
    float w2[2], u2[2], dk[2], eu[2];
    float kmax[2], kmin[2];
    bool fast1;
};

// Pass 0 + pass 1 of one warp's segment: key range, running-max exponent
// and the segment's summary (fixed-scale fast path, or the exact running-max
// recurrence when the keys span too wide a range).  FULL: every one of the
// LS tokens is valid, so no per-token test.
template <typename IO, int LS, bool FULL>
__device__ __forceinline__ void stream_pass01(const unsigned char* krow, const unsigned char* vrow, int nvalid,
                                              StreamSeg<LS>& sg, St* seg) {
    using Raw = typename Vec<IO, 2>::raw;
    constexpr int ROW = 64 * static_cast<int>(sizeof(IO));
    auto kr = [&](int i) { return *reinterpret_cast<const Raw*>(krow + i * ROW); };
    const F2 L2 = f2s(kLog2e);
    const F2 W2 = f2(sg.w2[0], sg.w2[1]);
    const int n = FULL ? LS : nvalid;
    // ---- pass 0: q = max_i (k2_i - (n-1-i) w2), each candidate from one product ----
    float kx[2] = {-3.0e38f, -3.0e38f}, kn[2] = {3.0e38f, 3.0e38f}, qm[2] = {-3.0e38f, -3.0e38f};
    float back = static_cast<float>(1 - n);   // i - (n-1), exact in float
#pragma unroll kStreamUnroll
    for (int i = 0; i < n; ++i) {
        const F2 kk = raw_pair<IO>(kr(i));
        const F2 cand = fma2(kk, L2, mul2(f2s(back), W2));
        back += 1.f;
        kx[0] = fmaxf(kx[0], f2lo(kk));
        kx[1] = fmaxf(kx[1], f2hi(kk));
        kn[0] = fminf(kn[0], f2lo(kk));
        kn[1] = fminf(kn[1], f2hi(kk));
        qm[0] = fmaxf(qm[0], f2lo(cand));
        qm[1] = fmaxf(qm[1], f2hi(cand));
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        sg.kmax[j] = kx[j] * kLog2e;
        sg.kmin[j] = kn[j] * kLog2e;
    }
    sg.fast1 = (sg.kmax[0] - sg.kmin[0] + fabsf(sg.u2[0]) <= kFastSpan) &&
               (sg.kmax[1] - sg.kmin[1] + fabsf(sg.u2[1]) <= kFastSpan);
    // ---- pass 1: the segment's summary ----
    if (sg.fast1) {
        const F2 KM = f2(-sg.kmax[0], -sg.kmax[1]);
        const F2 DK = f2(sg.dk[0], sg.dk[1]);
        F2 nn = f2s(0.f), db = f2s(0.f);
#pragma unroll kStreamUnroll
        for (int i = 0; i < n; ++i) {
            const F2 ek = ex2x2(fma2(raw_pair<IO>(kr(i)), L2, KM));
            const F2 ekv = mul2(ek, raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW)));
            nn = fma2(nn, DK, ekv);
            db = fma2(db, DK, ek);
        }
        const float sc0 = ex2(sg.kmax[0] - qm[0]), sc1 = ex2(sg.kmax[1] - qm[1]);
        seg[0] = St{qm[0], f2lo(nn) * sc0, f2lo(db) * sc0};
        seg[1] = St{qm[1], f2hi(nn) * sc1, f2hi(db) * sc1};
    } else {
        // keys too spread for one reference: the exact running-max recurrence
        // with its exponent held as pb - m w2 (see lane_token_pm)
        float pb[2], m[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            seg[j] = st_identity();
            pb[j] = seg[j].p;
            m[j] = 0.f;
        }
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            {
                const F2 kk = raw_pair<IO>(kr(i));
                const F2 vv = raw_pair<IO>(*reinterpret_cast<const Raw*>(vrow + i * ROW));
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                    const float v1 = j == 0 ? f2lo(vv) : f2hi(vv);
                    const float pd = fmaf(-(m[j] + 1.f), sg.w2[j], pb[j]);
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
        for (int j = 0; j < 2; ++j) seg[j].p = fmaf(-m[j], sg.w2[j], pb[j]);
    }
}

// Pass 2 of one warp's segment: the outputs from the segment's start state
// st, each written over the v entry it was computed from (in shared memory).
template <typename IO, bool GATE, int LS, bool FULL>
__device__ __forceinline__ void stream_pass2(const unsigned char* krow, unsigned char* vrow, const unsigned char* rrow,
                                             int nvalid, const StreamSeg<LS>& sg, St* st) {
    using Raw = typename Vec<IO, 2>::raw;
    using Ld = Vec<IO, 2>;
    constexpr int ROW = 64 * static_cast<int>(sizeof(IO));
    auto kr = [&](int i) { return *reinterpret_cast<const Raw*>(krow + i * ROW); };
    const F2 L2 = f2s(kLog2e);
    const int cnt = FULL ? LS : nvalid;
    bool fast2 = sg.fast1;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool near = st[j].p >= sg.kmax[j] - kFastState;
        const bool negligible = st[j].p < sg.kmax[j] - 1.5f * kFastState && st[j].b <= 16777216.f;
        fast2 = fast2 && (st[j].p - sg.kmin[j] + fabsf(sg.u2[j]) <= kFastState) && (near || negligible);
    }
    if (fast2) {
        float nr[2], ss[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float R = fmaxf(sg.kmax[j], st[j].p);
            nr[j] = -R;
            ss[j] = ex2(st[j].p - R);
        }
        const F2 NR = f2(nr[0], nr[1]);
        const F2 EU = f2(sg.eu[0], sg.eu[1]);
        const F2 DK = f2(sg.dk[0], sg.dk[1]);
        const F2 NL = f2s(-kLog2e);
        F2 n = f2(st[0].a * ss[0], st[1].a * ss[1]);
        F2 db = f2(st[0].b * ss[0], st[1].b * ss[1]);
#pragma unroll kStreamUnroll
        for (int i = 0; i < cnt; ++i) {
            {
                Raw* vp = reinterpret_cast<Raw*>(vrow + i * ROW);
                const F2 ek = ex2x2(fma2(raw_pair<IO>(kr(i)), L2, NR));
                const F2 ekv = mul2(ek, raw_pair<IO>(*vp));
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
                Ld::store(reinterpret_cast<IO*>(vp), out);
            }
        }
    } else {
        float pb[2], m[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            pb[j] = st[j].p;
            m[j] = 0.f;
        }
#pragma unroll 1
        for (int i = 0; i < cnt; ++i) {
            {
                Raw* vp = reinterpret_cast<Raw*>(vrow + i * ROW);
                const F2 kk = raw_pair<IO>(kr(i));
                const F2 vv = raw_pair<IO>(*vp);
                F2 rv = f2s(0.f);
                if (GATE) rv = raw_pair<IO>(*reinterpret_cast<const Raw*>(rrow + i * ROW));
                float out[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float gd = GATE ? gate_den(j == 0 ? f2lo(rv) : f2hi(rv)) : 1.f;
                    const float k2 = (j == 0 ? f2lo(kk) : f2hi(kk)) * kLog2e;
                    out[j] = lane_token_pm(st[j].a, st[j].b, pb[j], m[j], sg.w2[j], sg.u2[j], k2,
                                           j == 0 ? f2lo(vv) : f2hi(vv), gd);
                }
                Ld::store(reinterpret_cast<IO*>(vp), out);
            }
        }
    }
}

// Entering state of a chained call: the words the previous call of the chain
// published for this lane's channels, tagged with this call's position.
// Polled by one warp with a time bound; on expiry NaN and a recorded error.
__device__ __forceinline__ void chain_take(const ChunkArgs& A, int64_t li, bool cvalid, St* out) {
    const uint32_t want = word_tag(A.chain_in, kKindChain);
    const Word* src = A.chain + li;
    const uint64_t t0 = global_ns();
    unsigned sleep_ns = 32;
    for (;;) {
        Word wv[2];
        bool mine = true;
        if (cvalid) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                wv[j] = ld_word(src + j);
                mine = mine && wv[j].tag == want;
            }
        }
        if (__all_sync(0xffffffffu, mine)) {
#pragma unroll
            for (int j = 0; j < 2; ++j) out[j] = cvalid ? word_state(wv[j]) : st_identity();
            break;
        }
        if (global_ns() - t0 > A.wait_limit_ns) {
            if ((threadIdx.x & 31) == 0 && A.hdr != nullptr) record_timeout(A, -2);
            const float nan = __int_as_float(0x7fc00000);
#pragma unroll
            for (int j = 0; j < 2; ++j) out[j] = St{nan, nan, nan};
            break;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 256) sleep_ns <<= 1;
    }
    // acquire: the previous call's state_out write is ordered before this
    // call's (the word was published after it)
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

template <typename IO, bool GATE, int W, int LS, int MINB>
__global__ void __launch_bounds__(W * 32, MINB)
stream_forward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap ty,
                      const ChunkArgs A) {
    using G = StreamGeometry<IO, GATE, W, LS>;
    constexpr int V = 2;
    constexpr int CB = G::CB;
    constexpr int PT = G::PT;
    constexpr int ROW = G::ROW;
    using Raw = typename Vec<IO, V>::raw;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full;
    __shared__ St s_seg[W][V][32];                   // segment summaries of the part
    __shared__ __align__(16) float4 s_slot[V][32];   // the part's summary, read by later parts
    __shared__ St s_x[V][32];                        // summary of the chunk before this part
    __shared__ St s_in_chain[V][32];                 // entering state of a chained call
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = cluster_ctarank();             // part index along T
    const int64_t last = static_cast<int64_t>(cluster_nctarank()) - 1;
    const int64_t lb = cluster_id_x();               // lane block
    const int64_t bs = lb / A.nCB;
    const int x0 = static_cast<int>((lb % A.nCB) * CB);
    const int64_t c = x0 + lane * V;
    const bool cvalid = c < A.C;                     // C is even: both channels or neither
    const bool early = A.early != 0;
    const bool chained = A.chain != nullptr && A.chain_in != 0u;
    const float nan = __int_as_float(0x7fc00000);

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (GATE) prefetch_tensormap(&tr);
        prefetch_tensormap(&ty);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- load: k, v (, r) tiles and w, u by TMA ----
    const int64_t t_part = q * PT;
    const int part_len = static_cast<int>(min(static_cast<int64_t>(PT), A.T - t_part));
    const bool full_part = part_len == PT;
    float* prm = reinterpret_cast<float*>(smem + G::NT * G::TILE);
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const uint32_t pbytes = static_cast<uint32_t>(min(static_cast<int64_t>(CB), A.C - x0)) * 4u;
        mbar_expect_tx(&full, G::NT * G::TILE + 2u * pbytes);
        const int ty0 = static_cast<int>(A.t0 + t_part);   // row of the part in the arrays
        tma_load_3d(smem, &tk, x0, ty0, static_cast<int>(bs), &full);
        tma_load_3d(smem + G::TILE, &tv, x0, ty0, static_cast<int>(bs), &full);
        if (GATE) tma_load_3d(smem + 2 * G::TILE, &tr, x0, ty0, static_cast<int>(bs), &full);
        bulk_load(prm, A.w + x0, pbytes, &full);
        bulk_load(prm + CB, A.u + x0, pbytes, &full);
    }
    const int64_t t_seg = t_part + warp * LS;
    const int nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), A.T - t_seg)));
    __syncthreads();   // the barrier's initialisation is visible to every waiter
    const bool got = mbar_wait(&full, 0u, kCopyWaitNs);

    StreamSeg<LS> sg;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sg.w2[j] = cvalid ? prm[lane * V + j] * kLog2e : 1.f;
        sg.u2[j] = cvalid ? prm[CB + lane * V + j] * kLog2e : 0.f;
        sg.dk[j] = ex2(-sg.w2[j]);
        sg.eu[j] = ex2(sg.u2[j]);
    }
    const unsigned char* krow = smem + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));
    unsigned char* vrow = smem + G::TILE + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));

    // ---- pass 0/1: the segment's summary ----
    St seg[V];
    if (nvalid == 0 || !got) {
        seg[0] = seg[1] = st_identity();
        sg.kmax[0] = sg.kmax[1] = sg.kmin[0] = sg.kmin[1] = 0.f;
        sg.fast1 = false;
    } else if (full_part) {
        stream_pass01<IO, LS, true>(krow, vrow, nvalid, sg, seg);
    } else {
        stream_pass01<IO, LS, false>(krow, vrow, nvalid, sg, seg);
    }
#pragma unroll
    for (int j = 0; j < V; ++j) s_seg[warp][j][lane] = seg[j];
    const bool ok = __syncthreads_and(got);

    // ---- fold: summary of the part's segments before this warp's own ----
    St pre[V];
#pragma unroll
    for (int j = 0; j < V; ++j) pre[j] = st_identity();
    for (int s = 0; s < warp; ++s) {
        const int len = max(0, min(LS, part_len - s * LS));
#pragma unroll
        for (int j = 0; j < V; ++j) pre[j] = st_combine(pre[j], s_seg[s][j][lane], static_cast<float>(len) * sg.w2[j]);
    }
    const int pre_len = min(warp * LS, part_len);
    St agg[V];   // warp W-1: the part's summary
    if (warp == W - 1) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            agg[j] = ok ? st_combine(pre[j], seg[j], static_cast<float>(nvalid) * sg.w2[j]) : St{nan, nan, nan};
            s_slot[j][lane] = make_float4(agg[j].p, agg[j].a, agg[j].b, 0.f);
        }
    }
    cluster_arrive_release();
    if (chained && warp == 0) {
        // the entering state of a chained call, taken while the cluster's
        // other parts reach the barrier (read by every warp after the CTA
        // barrier below)
        St x[V];
        chain_take(A, bs * A.C + c, cvalid, x);
#pragma unroll
        for (int j = 0; j < V; ++j) s_in_chain[j][lane] = x[j];
    }
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
                                   static_cast<float>(PT) * sg.w2[j]);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) s_x[j][lane] = xs[j];
    }
    __syncthreads();
    // summary of every token from the chunk start to this warp's segment
    St z[V];
#pragma unroll
    for (int j = 0; j < V; ++j) z[j] = st_combine(s_x[j][lane], pre[j], static_cast<float>(pre_len) * sg.w2[j]);
    St chunk_sum[V];   // the last part's warp W-1: summary of the whole chunk
    if (warp == W - 1 && q == last) {
#pragma unroll
        for (int j = 0; j < V; ++j)
            chunk_sum[j] = st_combine(s_x[j][lane], agg[j], static_cast<float>(part_len) * sg.w2[j]);
    }

    // -------- the entering state from here on --------
    const int64_t lanes = A.B * A.C;
    St sin[V];
    if (chained) {
        // the previous call of the chain published it (taken by warp 0 at
        // the cluster barrier above); no wait for that kernel's end
#pragma unroll
        for (int j = 0; j < V; ++j) sin[j] = s_in_chain[j][lane];
    } else {
        if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
        for (int j = 0; j < V; ++j) {
            sin[j] = st_identity();
            if (A.s_in != nullptr && cvalid) {
                const int64_t li = bs * A.C + c + j;
                sin[j] = St{A.s_in[2 * lanes + li] * kLog2e, A.s_in[li], A.s_in[lanes + li]};
            }
        }
    }
    // every CTA has read state_in (and its remote reads are done) once all
    // arrive here; the last part writes state_out after that (and, in a
    // chain, overwrites the words every part has read by then)
    cluster_arrive_release();
    if (warp == W - 1 && q == last) {
        cluster_wait_acquire();
        St so[V];
#pragma unroll
        for (int j = 0; j < V; ++j)
            so[j] = ok ? st_combine(sin[j], chunk_sum[j], static_cast<float>(A.T) * sg.w2[j]) : St{nan, nan, nan};
        if (A.s_out != nullptr && cvalid) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const int64_t li = bs * A.C + c + j;
                A.s_out[li] = so[j].a;
                A.s_out[lanes + li] = so[j].b;
                A.s_out[2 * lanes + li] = so[j].p * kLn2;
            }
        }
        if (A.chain != nullptr) {
            // release: state_out before the word (the next call writes
            // state_out only after it has read the word)
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            if (cvalid) {
#pragma unroll
                for (int j = 0; j < V; ++j)
                    st_word(A.chain + bs * A.C + c + j, so[j], word_tag(A.chain_out, kKindChain));
            }
        }
    }

    // ---- pass 2: outputs from the segment's start state, then one store per warp ----
    if (A.y != nullptr && nvalid > 0) {
        if (cvalid) {
            if (ok) {
                St st[V];
#pragma unroll
                for (int j = 0; j < V; ++j) st[j] = st_combine(sin[j], z[j], static_cast<float>(t_seg) * sg.w2[j]);
                const unsigned char* rrow = vrow + G::TILE;
                if (full_part) stream_pass2<IO, GATE, LS, true>(krow, vrow, rrow, nvalid, sg, st);
                else stream_pass2<IO, GATE, LS, false>(krow, vrow, rrow, nvalid, sg, st);
            } else {
                // a copy that did not land: NaN outputs, never stale values
                const float out[2] = {nan, nan};
                for (int i = 0; i < nvalid; ++i) Vec<IO, V>::store(reinterpret_cast<IO*>(vrow + i * ROW), out);
            }
        }
        // the warp's rows were written through the generic proxy; the TMA
        // store reads them through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&ty, smem + G::TILE + warp * LS * ROW, x0, static_cast<int>(A.t0 + t_seg),
                         static_cast<int>(bs));
            bulk_commit_group();
        }
    }
    if (!ok && threadIdx.x == 0) {
        if (A.hdr != nullptr) record_timeout(A, q * A.nLB + lb);
        // let the copy land before the CTA's shared memory is released
        mbar_wait(&full, 0u, kCopyWaitNs);
    }
    // the stores must have read shared memory before the CTA exits
    if (lane == 0 && A.y != nullptr && nvalid > 0) bulk_wait_group_read0();
    if (!(warp == W - 1 && q == last)) cluster_wait_acquire();
    // a chained call has not waited for the previous kernel: one CTA waits
    // for it before exiting, so the grid still ends after the previous one
    // (the stream's kernels finish in order) while every other CTA frees
    // its SM slot for the next call at once
    if (chained && blockIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace wkv
