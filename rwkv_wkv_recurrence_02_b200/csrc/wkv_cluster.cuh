// wkv_cluster.cuh -- cluster kernel: few lane blocks, short sequences.
//
// A call with fewer lane blocks than SMs and at most CL parts of PT = W*LS
// tokens per sequence (one chunk of a long stream, say) runs as one thread
// block cluster per lane block, one CTA per part.  The scan that
// "並列学習の定式化" says the parallel mode performs (here an associative
// combination of segment summaries) then needs no global memory at all:
//
//   load     one TMA copy per array brings the CTA's PT x CB tile into shared
//            memory, with bulk copies of the channels' w, u (and for the
//            first part the initial state).
//   pass 0/1 warp s computes the summary of its LS-token segment, as in the
//            other kernels.
//   publish  warp W-1 folds the segment summaries into the part's summary
//            and leaves it in a shared-memory slot; the first part leaves
//            its inclusive state (initial state followed by the part).
//   barrier  one cluster barrier (release / acquire) makes every slot of the
//            cluster visible to every CTA of it.
//   prefix   warp W-1 of part q reads the slots of parts 0..q-1 through
//            distributed shared memory and folds them: the state entering
//            its part.  The cluster's last part writes state_out.
//   pass 2   outputs from each warp's start state.
//
// A second cluster barrier, split into an arrive after the remote reads and
// a wait before the exit, keeps every CTA's slot alive while others may read
// it.  No CTA waits on another cluster, and the hardware schedules a
// cluster's CTAs together, so progress needs no ticket order.  Every thread
// reaches both barriers on every path.
#pragma once

#include "wkv_part.cuh"

namespace wkv {

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// A state held in another CTA's shared memory: (p, a, b) of a float4 slot.
__device__ __forceinline__ St ld_cluster_state(const float4* local, uint32_t rank) {
    uint32_t addr;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(local)), "r"(rank));
    float4 s;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(s.x), "=f"(s.y), "=f"(s.z), "=f"(s.w)
                 : "r"(addr)
                 : "memory");
    return St{s.x, s.y, s.z};
}

template <typename IO, int V, bool GATE, int W, int LS, int MINB>
__global__ void __launch_bounds__(W * 32, MINB)
cluster_forward_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ CUtensorMap tr, const ChunkArgs A) {
    static_assert(V == 2, "channel pairs");
    using G = PartGeometry<IO, V, GATE, W, LS, 1>;
    constexpr int CB = G::CB;
    constexpr int PT = G::PT;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ __align__(8) uint64_t full;
    __shared__ St s_seg[W][V][32];          // segment summaries of the part
    __shared__ __align__(16) float4 s_slot[V][32];   // what later parts of the cluster read
    __shared__ St s_x[V][32];               // state entering the part
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = cluster_ctarank();    // part index along T
    const int64_t last = static_cast<int64_t>(cluster_nctarank()) - 1;
    const int64_t lb = cluster_id_x();      // lane block
    const int64_t part = q * A.nLB + lb;    // the part kernel's numbering (part-major)
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (GATE) prefetch_tensormap(&tr);
    }
    pdl_begin();
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        part_issue<IO, V, GATE, W, LS, 1>(&tk, &tv, &tr, A, smem, &full, part);
    }
    __syncthreads();

    const int64_t bs = lb / A.nCB;
    const int64_t c = (lb % A.nCB) * CB + lane * V;
    const bool full_part = (q + 1) * PT <= A.T;
    const int part_len = full_part ? PT : static_cast<int>(A.T - q * PT);
    SegCtx<V, LS> cx;
    const bool got = mbar_wait(&full, 0u, kCopyWaitNs);
    St seg[V];
    if (got) {
        if (full_part) seg_pass01<IO, V, GATE, W, LS, true, true, true, true>(A, q, bs, c, smem, cx, seg);
        else seg_pass01<IO, V, GATE, W, LS, false, true, true, true>(A, q, bs, c, smem, cx, seg);
#pragma unroll
        for (int j = 0; j < V; ++j) s_seg[warp][j][lane] = seg[j];
    }
    // every thread takes the same branch below
    const bool ok = __syncthreads_and(got);
    const float nan = __int_as_float(0x7fc00000);

    // prefix of the segments before this warp's own (from the empty state)
    St pre[V];
    int pre_len = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) pre[j] = st_identity();
    St agg[V];
    if (ok) {
        for (int sg = 0; sg < warp; ++sg) {
            const int len = full_part ? LS : max(0, min(LS, part_len - sg * LS));
#pragma unroll
            for (int j = 0; j < V; ++j)
                pre[j] = st_combine(pre[j], s_seg[sg][j][lane], static_cast<float>(len) * cx.w2[j]);
            pre_len += len;
        }
    }
    if (warp == W - 1) {
        const float* prm = reinterpret_cast<const float*>(smem + G::NARR * G::TILE);
#pragma unroll
        for (int j = 0; j < V; ++j) {
            St slot{nan, nan, nan};
            if (ok) {
                agg[j] = st_combine(pre[j], seg[j], static_cast<float>(cx.nvalid) * cx.w2[j]);
                slot = agg[j];
                if (q == 0) {
                    // the sequence's initial state, copied with the tiles
                    St sin = st_identity();
                    if (A.s_in != nullptr && cx.cvalid) {
                        const int o = lane * V + j;
                        sin = St{prm[4 * CB + o] * kLog2e, prm[2 * CB + o], prm[3 * CB + o]};
                    }
                    s_x[j][lane] = sin;
                    slot = st_combine(sin, agg[j], static_cast<float>(part_len) * cx.w2[j]);
                }
            } else if (q == 0) {
                s_x[j][lane] = slot;
            }
            s_slot[j][lane] = make_float4(slot.p, slot.a, slot.b, 0.f);
            if (q == 0) agg[j] = slot;   // rank 0: the inclusive state
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();

    if (warp == W - 1) {
        St x[V];
#pragma unroll
        for (int j = 0; j < V; ++j) x[j] = St{nan, nan, nan};
        if (q > 0 && ok) {
            // rank 0 holds the inclusive state of part 0; parts 1..q-1 are full
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = ld_cluster_state(&s_slot[j][lane], 0u);
            for (int64_t r = 1; r < q; ++r) {
#pragma unroll
                for (int j = 0; j < V; ++j)
                    x[j] = st_combine(x[j], ld_cluster_state(&s_slot[j][lane], static_cast<uint32_t>(r)),
                                      static_cast<float>(PT) * cx.w2[j]);
            }
        }
        if (q > 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) s_x[j][lane] = x[j];
        }
        if (q == last && A.s_out != nullptr && c < A.C) {
            const int64_t lanes = A.B * A.C;
#pragma unroll
            for (int j = 0; j < V; ++j) {
                // rank 0's agg already is its inclusive state
                const St inc = !ok ? St{nan, nan, nan}
                                   : (q == 0 ? agg[j] : st_combine(x[j], agg[j], static_cast<float>(part_len) * cx.w2[j]));
                const int64_t li = bs * A.C + c + j;
                A.s_out[li] = inc.a;
                A.s_out[lanes + li] = inc.b;
                A.s_out[2 * lanes + li] = inc.p * kLn2;
            }
        }
    }
    // this CTA reads no other CTA's shared memory from here on
    cluster_arrive_relaxed();
    __syncthreads();
    if (ok && cx.nvalid > 0 && cx.cvalid && A.y != nullptr) {
        St st[V];
#pragma unroll
        for (int j = 0; j < V; ++j) st[j] = st_combine(s_x[j][lane], pre[j], static_cast<float>(pre_len) * cx.w2[j]);
        if (full_part) seg_pass2<IO, V, GATE, W, LS, true, true>(A, smem, cx, st);
        else seg_pass2<IO, V, GATE, W, LS, false, true>(A, smem, cx, st);
    }
    if (!ok && threadIdx.x == 0) {
        if (A.hdr != nullptr) record_timeout(A, part);
        // let the copy land before the CTA's shared memory is released
        mbar_wait(&full, 0u, kCopyWaitNs);
    }
    cluster_wait_acquire();
}

}  // namespace wkv
