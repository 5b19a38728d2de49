// wkv_lane.cuh -- lane-resident chunked forward kernel.
//
// Each CTA owns whole lane blocks (CB = 32*V channels of one sequence) and
// walks their chunks in order, so the state carried from one chunk to the
// next never leaves the CTA: no workspace and no waiting on other CTAs.  It
// is the path when there are enough lane blocks to fill every CTA slot of
// the GPU; the look-back kernels split the sequence across CTAs otherwise.
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

#include "wkv_chunk_ws.cuh"

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

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <typename IO, int V, bool GATE, int W, int LS, int S>
__global__ void __launch_bounds__(LaneGeometry<IO, V, GATE, W, LS, S>::THREADS, 2)
lane_forward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tr, const ChunkArgs A) {
    using G = LaneGeometry<IO, V, GATE, W, LS, S>;
    constexpr int CB = G::CB;
    constexpr int TT = G::TT;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[S], empty[S];
    __shared__ St s_seg[2][W][V][32];   // segment summaries, double-buffered by chunk parity
    __shared__ St s_carry[2][V][32];    // state at the start of a chunk, double-buffered
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
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
            int64_t it = 0;
            for (int64_t lb = blockIdx.x; lb < A.nLB; lb += gridDim.x) {
                const int x = static_cast<int>((lb % A.nCB) * CB);
                const int z = static_cast<int>(lb / A.nCB);
                for (int64_t chunk = 0; chunk < A.nchunks; ++chunk, ++it) {
                    const int s = static_cast<int>(it % S);
                    if (it >= S && !mbar_wait(&empty[s], static_cast<uint32_t>(((it / S) - 1) & 1), A.wait_limit_ns))
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
    // (continuous across lane blocks).  The state entering a lane block is
    // written by warp W-1 where it would otherwise write the carried state,
    // so every slot is written and read in the same barrier order.
    const int64_t lanes = A.B * A.C;
    auto initial_state = [&](int64_t lbx, int j) -> St {
        if (lbx >= A.nLB) return st_identity();
        const int64_t cc = (lbx % A.nCB) * CB + lane * V + j;
        if (A.s_in == nullptr || cc >= A.C) return st_identity();
        const int64_t li = (lbx / A.nCB) * A.C + cc;
        return St{A.s_in[2 * lanes + li] * kLog2e, A.s_in[li], A.s_in[lanes + li]};
    };
    if (warp == W - 1 && static_cast<int64_t>(blockIdx.x) < A.nLB) {
#pragma unroll
        for (int j = 0; j < V; ++j) s_carry[0][j][lane] = initial_state(blockIdx.x, j);
    }
    int64_t it = 0;
    for (int64_t lb = blockIdx.x; lb < A.nLB; lb += gridDim.x) {
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
        for (int64_t chunk = 0; chunk < A.nchunks; ++chunk, ++it) {
            const int s = static_cast<int>(it % S);
            const int par = static_cast<int>(it & 1);
            if (!mbar_wait(&full[s], static_cast<uint32_t>((it / S) & 1), A.wait_limit_ns)) {
                if (threadIdx.x == 0 && A.hdr != nullptr) record_timeout(A, -1);
                return;
            }
            const unsigned char* stage = smem + s * G::STAGE;
            const int64_t unit = chunk * A.nLB + lb;
            const bool full_chunk = (chunk + 1) * TT <= A.T;
            St seg[V];
            if (full_chunk) seg_pass01<IO, V, GATE, W, LS, true, false>(A, unit, stage, cx, seg);
            else seg_pass01<IO, V, GATE, W, LS, false, false>(A, unit, stage, cx, seg);
#pragma unroll
            for (int j = 0; j < V; ++j) s_seg[par][warp][j][lane] = seg[j];
            named_sync(1, W * 32);
            // start state of this warp's segment: carried state, then the
            // segments before this one
            const int64_t chunk_rows = min(static_cast<int64_t>(TT), A.T - chunk * TT);
            St st[V];
#pragma unroll
            for (int j = 0; j < V; ++j) st[j] = s_carry[par][j][lane];
            for (int sg = 0; sg < warp; ++sg) {
                const int len = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), chunk_rows - sg * LS)));
#pragma unroll
                for (int j = 0; j < V; ++j) st[j] = st_combine(st[j], s_seg[par][sg][j][lane], static_cast<float>(len) * cx.w2[j]);
            }
            if (warp == W - 1) {
                // state after the chunk: this warp's start, then its own segment
                const bool last = chunk == A.nchunks - 1;
                for (int j = 0; j < V; ++j) {
                    const St nx = st_combine(st[j], seg[j], static_cast<float>(cx.nvalid) * cx.w2[j]);
                    s_carry[par ^ 1][j][lane] = last ? initial_state(lb + gridDim.x, j) : nx;
                    if (last && A.s_out != nullptr && cx.cvalid) {
                        const int64_t li = b * A.C + c + j;
                        A.s_out[li] = nx.a;
                        A.s_out[lanes + li] = nx.b;
                        A.s_out[2 * lanes + li] = nx.p * kLn2;
                    }
                }
            }
            if (cx.nvalid > 0 && cx.cvalid) {
                if (full_chunk) seg_pass2<IO, V, GATE, W, LS, true>(A, stage, cx, st);
                else seg_pass2<IO, V, GATE, W, LS, false>(A, stage, cx, st);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
}

}  // namespace wkv
