// wkv_lane.cuh -- lane-resident chunked forward kernel.
//
// Each CTA owns lane blocks (CB = 32*V channels of one sequence) and walks
// their chunks in order, so the state carried from one chunk to the next
// stays in the CTA.  To balance the work, CTA g takes an equal share of the
// lane-major (lane block, chunk) order: at most the head of its last lane
// block and the tail of its first one are partial, and the head's end state
// is handed to the next CTA as one 16-byte word per channel (see LaneRange).
// It is the path when there are at least as many lane blocks as SMs; the
// look-back kernels split single sequences across CTAs otherwise.
//
// Warps 0..W-1 compute, warp W is the producer.  Per chunk of TT = W*LS
// tokens: the producer streams the k, v, r tiles into a ring of S shared-
// memory stages with TMA; warp s runs pass 0/1 over its LS-token segment
// (same fixed-scale fast path and exact running-max fallback as the other
// kernels), the W segment summaries meet in shared memory (one named barrier
// per chunk), each warp folds the carried state with the summaries before
// its own to get its segment's start state, warp W-1 also forms the state
// after the chunk for the next one, and pass 2 writes the outputs.  The
// compute warps release a stage with an mbarrier the producer waits on.
#pragma once

#include "wkv_segment.cuh"

namespace wkv {

template <typename IO, int V, bool GATE, int W, int LS, int S>
struct LaneGeometry {
    static constexpr int CB = 32 * V;
    static constexpr int TT = W * LS;
    static constexpr int NARR = GATE ? 3 : 2;
    static constexpr int ROW = CB * static_cast<int>(sizeof(IO));
    static constexpr uint32_t TILE = TT * ROW;
    static constexpr uint32_t STAGE = NARR * TILE + 5 * CB * sizeof(float);  // tiles + unused param area
    static constexpr uint32_t SMEM = S * STAGE;
    static constexpr int THREADS = (W + 1) * 32;
};

// The contiguous range [s, e) of the lane-major (lane block, chunk) order a
// CTA owns, as work items in processing order: the head of its last lane
// block (chunks from 0, ending inside the block; its end state is handed to
// the next CTA), then whole lane blocks, then the tail of its first lane
// block (starting inside the block from the state the previous CTA handed
// over).  With at least as many lane blocks as CTAs every range spans a lane
// block boundary, so a CTA has at most one head and one tail and no hand-off
// depends on another.  `whole` (no workspace to hand states through) rounds
// every range to whole lane blocks: CTA g takes lane blocks
// [g*nLB/G, (g+1)*nLB/G), and no range has a head or a tail.
struct LaneRange {
    int64_t nc;            // chunks per lane block
    int64_t f0, nfull;     // whole lane blocks [f0, f0 + nfull)
    int64_t lb_head, head_end, lb_tail, tail_begin;
    bool head, tail;
    int count;

    __device__ __forceinline__ void init(int64_t nLB, int64_t nchunks, int64_t g, int64_t G, bool whole) {
        nc = nchunks;
        const int64_t U = nLB * nchunks;
        const int64_t s = whole ? (g * nLB / G) * nchunks : g * U / G;
        const int64_t e = whole ? ((g + 1) * nLB / G) * nchunks : (g + 1) * U / G;
        tail = s % nc != 0;
        lb_tail = s / nc;
        tail_begin = s % nc;
        head = e % nc != 0;
        lb_head = e / nc;
        head_end = e % nc;
        f0 = (s + nc - 1) / nc;
        nfull = e / nc - f0;
        if (nfull < 0) nfull = 0;
        count = static_cast<int>(nfull) + (head ? 1 : 0) + (tail ? 1 : 0);
    }
    // item i: lane block, chunk range [c0, c1), whether its start state comes
    // from the previous CTA and whether its end state goes to the next one
    __device__ __forceinline__ void item(int i, int64_t& lb, int64_t& c0, int64_t& c1, bool& from_prev,
                                         bool& to_next) const {
        from_prev = false;
        to_next = false;
        if (head) {
            if (i == 0) {
                lb = lb_head;
                c0 = 0;
                c1 = head_end;
                to_next = true;
                return;
            }
            --i;
        }
        if (i < nfull) {
            lb = f0 + i;
            c0 = 0;
            c1 = nc;
            return;
        }
        lb = lb_tail;
        c0 = tail_begin;
        c1 = nc;
        from_prev = true;
    }
    // item i in the order of the reverse mode, which walks chunks from the
    // last to the first: the tail of the first lane block (it starts from
    // the end of the sequence; its reverse state at tail_begin goes to the
    // previous CTA), then whole lane blocks, then the head of the last one
    // (it starts from the reverse state the next CTA hands over).
    __device__ __forceinline__ void item_back(int i, int64_t& lb, int64_t& c0, int64_t& c1, bool& to_prev,
                                              bool& from_next) const {
        to_prev = false;
        from_next = false;
        if (tail) {
            if (i == 0) {
                lb = lb_tail;
                c0 = tail_begin;
                c1 = nc;
                to_prev = true;
                return;
            }
            --i;
        }
        if (i < nfull) {
            lb = f0 + i;
            c0 = 0;
            c1 = nc;
            return;
        }
        lb = lb_head;
        c0 = 0;
        c1 = head_end;
        from_next = true;
    }
};

// State entering work item i (called by one warp, once per item): the
// sequence's initial state, or the state the previous CTA handed over
// (waited for with a time bound; NaN and a recorded error on expiry).
// The call's arguments come as values (not the argument block by reference),
// so the kernel's arguments stay in the constant bank.
template <int V>
__device__ __noinline__ void lane_entry_state(const float* s_in, int64_t B, int64_t C, int64_t nCB,
                                              const Word* incw, WsHeader* hdr, uint64_t limit_ns,
                                              const LaneRange& R, int i, uint32_t epoch, St* out) {
    constexpr int CB = 32 * V;
    const int lane = threadIdx.x & 31;
    const int64_t lanes = B * C;
    int64_t lb, c0, c1;
    bool from_prev, to_next;
    R.item(i, lb, c0, c1, from_prev, to_next);
    const int64_t cb = (lb % nCB) * CB + lane * V;
    if (!from_prev) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            out[j] = st_identity();
            if (s_in != nullptr && cb + j < C) {
                const int64_t li = (lb / nCB) * C + cb + j;
                out[j] = St{s_in[2 * lanes + li] * kLog2e, s_in[li], s_in[lanes + li]};
            }
        }
        return;
    }
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

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads that also ANDs a flag over them, so
// every participating thread takes the same branch afterwards.
__device__ __forceinline__ bool named_sync_and(int id, int threads, bool flag) {
    uint32_t all;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(all)
        : "r"(static_cast<uint32_t>(flag)), "r"(id), "r"(threads)
        : "memory");
    return all != 0;
}

// CKPT: checkpoint sweep for the reverse mode instead of outputs: no pass 2,
// and the state entering every chunk (and the one after the sequence) goes
// to A.ckpt.
template <typename IO, int V, bool GATE, int W, int LS, int S, int MINB = 2, bool CKPT = false>
__global__ void __launch_bounds__(LaneGeometry<IO, V, GATE, W, LS, S>::THREADS, MINB)
lane_forward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tr, const ChunkArgs A) {
    using G = LaneGeometry<IO, V, GATE, W, LS, S>;
    constexpr int CB = G::CB;
    constexpr int TT = G::TT;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[S], empty[S];
    __shared__ St s_seg[2][W][V][32];   // segment summaries, double-buffered by chunk parity
    __shared__ St s_carry[2][V][32];    // state at the start of a chunk, double-buffered
    __shared__ LaneRange s_range;       // this CTA's share of the chunk order
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (GATE) prefetch_tensormap(&tr);
    }
    pdl_begin();
    if (threadIdx.x == 0) {
        s_range.init(A.nLB, A.nchunks, blockIdx.x, gridDim.x, A.hdr == nullptr);
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], W);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == W) {
        // ---------------- producer ----------------
        if (lane == 0) {
            const LaneRange& R = s_range;
            uint32_t it = 0;
            for (int item = 0; item < R.count; ++item) {
                int64_t lb, c0, c1;
                bool from_prev, to_next;
                R.item(item, lb, c0, c1, from_prev, to_next);
                const int x = static_cast<int>((lb % A.nCB) * CB);
                const int z = static_cast<int>(lb / A.nCB);
                for (int64_t chunk = c0; chunk < c1; ++chunk, ++it) {
                    const int s = static_cast<int>(it % S);
                    if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1u, A.wait_limit_ns))
                        return;  // the compute warps stopped; they time out on full[] as well
                    unsigned char* st = smem + s * G::STAGE;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_expect_tx(&full[s], G::NARR * G::TILE);
                    const int y = static_cast<int>(chunk * TT);
                    tma_load_3d(st, &tk, x, y, z, &full[s]);
                    tma_load_3d(st + G::TILE, &tv, x, y, z, &full[s]);
                    if (GATE) tma_load_3d(st + 2 * G::TILE, &tr, x, y, z, &full[s]);
                }
            }
        }
        return;
    }

    // ---------------- compute ----------------
    // Shared buffers alternate with the parity of the running chunk count it
    // (continuous across work items).  The state entering a work item is
    // written by warp W-1 where it would otherwise write the carried state,
    // so every slot is written and read in the same barrier order.
    const int64_t lanes = A.B * A.C;
    const uint32_t epoch = A.hdr != nullptr ? ld_relaxed_u32(&A.hdr->epoch) : 0u;
    const LaneRange& R = s_range;
    bool ok = true;
    if (warp == W - 1 && R.count > 0) {
        St x0[V];
        lane_entry_state<V>(A.s_in, A.B, A.C, A.nCB, A.incw, A.hdr, A.wait_limit_ns, R, 0, epoch, x0);
#pragma unroll
        for (int j = 0; j < V; ++j) s_carry[0][j][lane] = x0[j];
    }
    uint32_t it = 0;
    for (int item = 0; item < R.count && ok; ++item) {
        int64_t lb, c0, c1;
        bool from_prev, to_next;
        R.item(item, lb, c0, c1, from_prev, to_next);
        const int64_t b = lb / A.nCB;
        const int64_t c = (lb % A.nCB) * CB + lane * V;
        SegCtx<V, LS> cx;
        cx.cvalid = c < A.C;
        {
            float wv[V], uv[V];
#pragma unroll
            for (int j = 0; j < V; ++j) {
                wv[j] = cx.cvalid ? __ldg(A.w + c + j) : 1.f;
                uv[j] = cx.cvalid ? __ldg(A.u + c + j) : 0.f;
            }
            set_params<V, LS>(cx, wv, uv);
        }
        for (int64_t chunk = c0; chunk < c1; ++chunk, ++it) {
            const int s = static_cast<int>(it % S);
            const int par = static_cast<int>(it & 1u);
            const bool got = mbar_wait(&full[s], (it / S) & 1u, kCopyWaitNs);
            const unsigned char* stage = smem + s * G::STAGE;
            const bool full_chunk = (chunk + 1) * TT <= A.T;
            St seg[V];
            if (got) {
                if (full_chunk) seg_pass01<IO, V, GATE, W, LS, true, false>(A, chunk, b, c, stage, cx, seg);
                else seg_pass01<IO, V, GATE, W, LS, false, false>(A, chunk, b, c, stage, cx, seg);
#pragma unroll
                for (int j = 0; j < V; ++j) s_seg[par][warp][j][lane] = seg[j];
            }
            // a copy that did not land stops every compute warp together
            if (!named_sync_and(1, W * 32, got)) {
                if (threadIdx.x == 0 && A.hdr != nullptr) record_timeout(A, -1);
                ok = false;
                break;
            }
            if (CKPT && warp == 0) {
                St* dst = A.ckpt + (chunk * A.nLB + lb) * CB + lane * V;
#pragma unroll
                for (int j = 0; j < V; ++j) dst[j] = s_carry[par][j][lane];
            }
            // start state of this warp's segment: carried state, then the
            // segments before this one
            // rows of this chunk (all TT but in a sequence's last, partial chunk)
            const int chunk_rows = full_chunk ? TT : static_cast<int>(A.T - chunk * TT);
            St st[V];
#pragma unroll
            for (int j = 0; j < V; ++j) st[j] = s_carry[par][j][lane];
            float seglen[V];
#pragma unroll
            for (int j = 0; j < V; ++j) seglen[j] = static_cast<float>(LS) * cx.w2[j];
            for (int sg = 0; sg < warp; ++sg) {
                // segments before this one are full unless the chunk is short
                if (!full_chunk) {
                    const int len = max(0, min(LS, chunk_rows - sg * LS));
#pragma unroll
                    for (int j = 0; j < V; ++j) seglen[j] = static_cast<float>(len) * cx.w2[j];
                }
#pragma unroll
                for (int j = 0; j < V; ++j) st[j] = st_combine(st[j], s_seg[par][sg][j][lane], seglen[j]);
            }
            if (warp == W - 1) {
                // state after the chunk: this warp's start, then its own segment
                St nx[V];
#pragma unroll
                for (int j = 0; j < V; ++j) nx[j] = st_combine(st[j], seg[j], static_cast<float>(cx.nvalid) * cx.w2[j]);
                if (CKPT && chunk == A.nchunks - 1) {
                    St* dst = A.ckpt + (A.nchunks * A.nLB + lb) * CB + lane * V;
#pragma unroll
                    for (int j = 0; j < V; ++j) dst[j] = nx[j];
                }
                if (chunk == c1 - 1) {
                    if (to_next) {
                        publish<V>(A.incw + lb * CB, nx, epoch, kKindInc, lane);
                    } else if (A.s_out != nullptr && cx.cvalid) {
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            const int64_t li = b * A.C + c + j;
                            A.s_out[li] = nx[j].a;
                            A.s_out[lanes + li] = nx[j].b;
                            A.s_out[2 * lanes + li] = nx[j].p * kLn2;
                        }
                    }
                    if (item + 1 < R.count)
                        lane_entry_state<V>(A.s_in, A.B, A.C, A.nCB, A.incw, A.hdr, A.wait_limit_ns, R, item + 1,
                                            epoch, nx);
                }
#pragma unroll
                for (int j = 0; j < V; ++j) s_carry[par ^ 1][j][lane] = nx[j];
            }
            if (!CKPT && cx.nvalid > 0 && cx.cvalid && A.y != nullptr) {
                if (full_chunk) seg_pass2<IO, V, GATE, W, LS, true>(A, stage, cx, st);
                else seg_pass2<IO, V, GATE, W, LS, false>(A, stage, cx, st);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    if (threadIdx.x == 0 && A.hdr != nullptr) finish_launch(A, gridDim.x);
}

}  // namespace wkv
