// wkv_part.cuh -- part kernel: few lane blocks, sequences cut along T.
//
// With few lane blocks (one or a few long sequences) the lane-resident kernel
// leaves most SMs idle, and each of its CTAs walks its chunks one after the
// other.  Here every lane block is cut along T into parts of PT = W*LS tokens,
// and a part is small enough to sit in shared memory whole, so it is read from
// HBM once:
//
//   load     one TMA copy per array (k, v, and r when gated) brings the part's
//            PT x CB tile into a shared-memory buffer, and two bulk copies
//            the channels' w and u; with several buffers the next parts'
//            copies overlap this part's arithmetic.
//   pass 0/1 warp s computes the summary of its LS-token segment (same
//            fixed-scale fast path and exact running-max fallback as the
//            other kernels; the per-token exponentials stay in registers).
//   prefix   every warp folds the summaries of the segments before its own.
//            Warp W-1 also forms the part's summary, publishes it, and finds
//            the state entering the part by decoupled look-back over the
//            parts before it (one slot per part and channel, holding the
//            part's summary and later its inclusive state; each lane walks
//            its own channels), then publishes the state after the part.
//   pass 2   each warp's start state is the entering state followed by its
//            prefix; outputs as in the other kernels.
//
// Parts are claimed in order from the workspace's ticket counter (part-major:
// all first parts, then all second parts, ...), so a part only waits on parts
// that running CTAs have claimed, and the CTA count does not matter for
// progress.  Without a workspace (a single part per lane block) the CTAs take
// parts with a fixed stride instead.
#pragma once

#include "wkv_segment.cuh"

namespace wkv {

template <typename IO, int V, bool GATE, int W, int LS, int NB>
struct PartGeometry {
    static constexpr int CB = 32 * V;
    static constexpr int PT = W * LS;
    static constexpr int NARR = GATE ? 3 : 2;
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = PT * ROW;
    // w, u of the part's channels follow the tiles (bulk copies), and for a
    // first part the initial state's a, b, p
    static constexpr uint32_t PARAM = 5 * CB * sizeof(float);
    static constexpr uint32_t PART = NARR * TILE + PARAM;
    static constexpr uint32_t SMEM = NB * PART;
    static constexpr int THREADS = W * 32;
};

template <typename IO, int V, bool GATE, int W, int LS, int NB>
__device__ __forceinline__ void part_issue(const CUtensorMap* tk, const CUtensorMap* tv, const CUtensorMap* tr,
                                           const ChunkArgs& A, unsigned char* buf, uint64_t* bar, int64_t part) {
    using G = PartGeometry<IO, V, GATE, W, LS, NB>;
    const int64_t q = part / A.nLB, lb = part % A.nLB;
    const int x = static_cast<int>((lb % A.nCB) * G::CB);
    const int y = static_cast<int>(q * G::PT);
    const int z = static_cast<int>(lb / A.nCB);
    // channels of this block inside C: a multiple of 4, because C is
    const uint32_t pbytes = static_cast<uint32_t>(min(static_cast<int64_t>(G::CB), A.C - x)) * 4u;
    float* prm = reinterpret_cast<float*>(buf + G::NARR * G::TILE);
    // the buffer was last read through the generic proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const bool first = q == 0 && A.s_in != nullptr;
    mbar_expect_tx(bar, G::NARR * G::TILE + (first ? 5u : 2u) * pbytes);
    tma_load_3d(buf, tk, x, y, z, bar);
    tma_load_3d(buf + G::TILE, tv, x, y, z, bar);
    if (GATE) tma_load_3d(buf + 2 * G::TILE, tr, x, y, z, bar);
    bulk_load(prm, A.w + x, pbytes, bar);
    bulk_load(prm + G::CB, A.u + x, pbytes, bar);
    if (first) {
        const int64_t lanes = A.B * A.C;
        const float* si = A.s_in + z * A.C + x;
        bulk_load(prm + 2 * G::CB, si, pbytes, bar);
        bulk_load(prm + 3 * G::CB, si + lanes, pbytes, bar);
        bulk_load(prm + 4 * G::CB, si + 2 * lanes, pbytes, bar);
    }
}

// Look-back of one part, run by one warp; every lane walks back on its own
// V channels.  Part slots hold one word per channel that the part's own
// summary (kKindAgg) and later its inclusive state (kKindInc) overwrite, so
// a reader sees either; each round reads WIN slots in one round trip and
// walks them nearest first: an inclusive state ends the walk, a summary is
// folded in and the walk goes on, anything else waits for the next round.
// The start of the sequence stands for an inclusive state (sin).  Returns
// false (x NaN) if the wait limit passed first.
template <int V, int PT, int WIN>
__device__ __forceinline__ bool part_lookback(const ChunkArgs& A, int64_t lb, int64_t q, uint32_t epoch,
                                              const float* w2, const St* sin, St* x, int lane) {
    constexpr int CB = 32 * V;
    St acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = st_identity();
    int64_t cur = q - 1;
    float span = 0.f;
    const uint32_t tag_agg = word_tag(epoch, kKindAgg), tag_inc = word_tag(epoch, kKindInc);
    const uint64_t t0 = global_ns();
    unsigned sleep_ns = 32;
    for (;;) {
        Word wv[WIN][V];
#pragma unroll
        for (int l = 0; l < WIN; ++l) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                wv[l][j] = cur - l >= 0 ? ld_word(A.aggw + ((cur - l) * A.nLB + lb) * CB + lane * V + j)
                                        : Word{0.f, 0.f, 0.f, 0u};
            }
        }
        bool progressed = false;
#pragma unroll
        for (int l = 0; l < WIN; ++l) {
            if (cur < 0) {
#pragma unroll
                for (int j = 0; j < V; ++j) x[j] = st_combine(sin[j], acc[j], span * w2[j]);
                return true;
            }
            bool inc = true, agg = true;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                inc = inc && wv[l][j].tag == tag_inc;
                agg = agg && wv[l][j].tag == tag_agg;
            }
            if (inc) {
#pragma unroll
                for (int j = 0; j < V; ++j) x[j] = st_combine(word_state(wv[l][j]), acc[j], span * w2[j]);
                return true;
            }
            if (!agg) break;
#pragma unroll
            for (int j = 0; j < V; ++j) acc[j] = st_combine(word_state(wv[l][j]), acc[j], span * w2[j]);
            span += static_cast<float>(PT);
            --cur;
            progressed = true;
        }
        if (!progressed) {
            if (global_ns() - t0 > A.wait_limit_ns) {
                const float nan = __int_as_float(0x7fc00000);
#pragma unroll
                for (int j = 0; j < V; ++j) x[j] = St{nan, nan, nan};
                return false;
            }
            __nanosleep(sleep_ns);
            if (sleep_ns < 256) sleep_ns <<= 1;
        }
    }
}

// Warp W-1's share of a part: publish the part's summary, find the state
// entering the part by look-back, publish the state after it (or write
// state_out after the last part), and leave the entering state in
// x[j*32 + lane].
template <int V, int PT, int WIN>
__device__ __forceinline__ void part_scan(const ChunkArgs& A, int64_t part, uint32_t epoch, bool cvalid, float w20,
                                          float w21, St agg0, St agg1, int part_len, const float* prm, St* x) {
    static_assert(V == 2, "channel pairs");
    constexpr int CB = 32 * V;
    const int lane = threadIdx.x & 31;
    const int64_t q = part / A.nLB, lb = part % A.nLB;
    const int64_t bs = lb / A.nCB;
    const int64_t c = (lb % A.nCB) * CB + lane * V;
    const int64_t lanes = A.B * A.C;
    const float w2[V] = {w20, w21};
    const St agg[V] = {agg0, agg1};
    // The sequence's initial state, copied into the part's buffer with its
    // tiles.  Only the first part's look-back reaches the start: a first
    // part publishes its inclusive state and never a summary, so every later
    // walk ends at an inclusive state.  The copy lands before the part
    // publishes anything; the last part, which may overwrite the state in
    // place (state_out == state_in), writes only after seeing a chain of
    // inclusive states that starts there.
    St sin[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        sin[j] = st_identity();
        if (q == 0 && A.s_in != nullptr && cvalid) {
            const int o = lane * V + j;
            sin[j] = St{prm[4 * CB + o] * kLog2e, prm[2 * CB + o], prm[3 * CB + o]};
        }
    }
    const bool has_next = q + 1 < A.nchunks;
    Word* slot = A.aggw + part * CB;
    if (has_next && q > 0) publish<V>(slot, agg, epoch, kKindAgg, lane);
    St xs[V];
    if (!part_lookback<V, PT, WIN>(A, lb, q, epoch, w2, sin, xs, lane) && A.hdr != nullptr)
        record_timeout(A, part);
    St inc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        x[j * 32 + lane] = xs[j];
        inc[j] = st_combine(xs[j], agg[j], static_cast<float>(part_len) * w2[j]);
    }
    if (has_next) {
        publish<V>(slot, inc, epoch, kKindInc, lane);
    } else if (A.s_out != nullptr && cvalid) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int64_t li = bs * A.C + c + j;
            A.s_out[li] = inc[j].a;
            A.s_out[lanes + li] = inc[j].b;
            A.s_out[2 * lanes + li] = inc[j].p * kLn2;
        }
    }
}

template <typename IO, int V, bool GATE, int W, int LS, int NB, int MINB, int PWIN, bool CACHE>
__global__ void __launch_bounds__(W * 32, MINB)
part_forward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tr, const ChunkArgs A) {
    using G = PartGeometry<IO, V, GATE, W, LS, NB>;
    constexpr int CB = G::CB;
    constexpr int PT = G::PT;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[NB];
    __shared__ int64_t s_part[NB];      // part whose copy each buffer holds (>= units: none)
    __shared__ St s_seg[W][V][32];      // segment summaries of the current part
    __shared__ St s_x[V][32];           // state entering the current part
    __shared__ uint32_t s_epoch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool ticket = A.hdr != nullptr;
    int64_t stride_next = blockIdx.x;   // thread 0 only, without a workspace
    auto claim = [&]() -> int64_t {
        if (ticket) return static_cast<int64_t>(atomicAdd(&A.hdr->ticket, 1u));
        const int64_t t = stride_next;
        stride_next += gridDim.x;
        return t;
    };
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (GATE) prefetch_tensormap(&tr);
    }
    pdl_begin();
    if (threadIdx.x == 0) {
        for (int b = 0; b < NB; ++b) mbar_init(&full[b], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_epoch = ticket ? ld_relaxed_u32(&A.hdr->epoch) : 0u;
        for (int b = 0; b < NB; ++b) {
            const int64_t t = claim();
            s_part[b] = t;
            if (t < A.units) part_issue<IO, V, GATE, W, LS, NB>(&tk, &tv, &tr, A, smem + b * G::PART, &full[b], t);
        }
    }
    __syncthreads();
    const uint32_t epoch = s_epoch;

    for (uint32_t i = 0;; ++i) {
        const int bi = static_cast<int>(i % NB);
        const int64_t part = s_part[bi];
        if (part >= A.units) break;
        const int64_t q = part / A.nLB, lb = part % A.nLB;
        const int64_t bs = lb / A.nCB;
        const int64_t c = (lb % A.nCB) * CB + lane * V;
        const bool full_part = (q + 1) * PT <= A.T;
        const int part_len = full_part ? PT : static_cast<int>(A.T - q * PT);
        SegCtx<V, LS> cx;
        const unsigned char* stage = smem + bi * G::PART;
        const bool got = mbar_wait(&full[bi], (i / NB) & 1u, kCopyWaitNs);
        St seg[V];
        if (got) {
            if (full_part) seg_pass01<IO, V, GATE, W, LS, true, true, CACHE>(A, q, bs, c, stage, cx, seg);
            else seg_pass01<IO, V, GATE, W, LS, false, true, CACHE>(A, q, bs, c, stage, cx, seg);
#pragma unroll
            for (int j = 0; j < V; ++j) s_seg[warp][j][lane] = seg[j];
        }
        // every thread takes the same branch: a copy that did not land ends
        // the CTA's work
        if (!__syncthreads_and(got)) {
            if (threadIdx.x == 0) {
                if (ticket) record_timeout(A, part);
                // let copies still in flight land before the CTA exits
                for (int b = 0; b < NB; ++b) {
                    const uint32_t k = i + static_cast<uint32_t>((b - bi + NB) % NB);
                    if (s_part[b] < A.units) mbar_wait(&full[b], (k / NB) & 1u, kCopyWaitNs);
                }
            }
            break;
        }
        // prefix of the segments before this warp's own (from the empty state)
        St pre[V];
        int pre_len = 0;
#pragma unroll
        for (int j = 0; j < V; ++j) pre[j] = st_identity();
        for (int sg = 0; sg < warp; ++sg) {
            const int len = full_part ? LS : max(0, min(LS, part_len - sg * LS));
#pragma unroll
            for (int j = 0; j < V; ++j) pre[j] = st_combine(pre[j], s_seg[sg][j][lane], static_cast<float>(len) * cx.w2[j]);
            pre_len += len;
        }
        if (warp == W - 1) {
            St agg[V];
#pragma unroll
            for (int j = 0; j < V; ++j) agg[j] = st_combine(pre[j], seg[j], static_cast<float>(cx.nvalid) * cx.w2[j]);
            part_scan<V, PT, PWIN>(A, part, epoch, cx.cvalid, cx.w2[0], cx.w2[1], agg[0], agg[1], part_len,
                                  reinterpret_cast<const float*>(stage + G::NARR * G::TILE), &s_x[0][0]);
        }
        __syncthreads();
        if (cx.nvalid > 0 && cx.cvalid && A.y != nullptr) {
            St st[V];
#pragma unroll
            for (int j = 0; j < V; ++j) st[j] = st_combine(s_x[j][lane], pre[j], static_cast<float>(pre_len) * cx.w2[j]);
            if (full_part) seg_pass2<IO, V, GATE, W, LS, true, CACHE>(A, stage, cx, st);
            else seg_pass2<IO, V, GATE, W, LS, false, CACHE>(A, stage, cx, st);
        }
        // buffer bi, s_seg and s_x are free again
        __syncthreads();
        if (threadIdx.x == 0) {
            const int64_t t = claim();
            s_part[bi] = t;
            if (t < A.units) part_issue<IO, V, GATE, W, LS, NB>(&tk, &tv, &tr, A, smem + bi * G::PART, &full[bi], t);
        }
        if (NB == 1) __syncthreads();
    }
    if (ticket && threadIdx.x == 0) finish_launch(A, gridDim.x);
}

}  // namespace wkv
