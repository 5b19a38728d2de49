// wkv_chunk.cuh -- chunked associative-scan forward kernel.
//
// The recurrence of "リカレント定式化" is linear in the state with a constant
// per-channel factor e^-w, so a run of tokens has a summary (the state it
// reaches from the empty state) and summaries compose associatively: this is
// the scan that "並列学習の定式化" says the parallel mode performs.
//
// Work split.  A unit is one CTA: CB = 32*V channels of one sequence b times a
// chunk of TT = W*LS tokens.  Warp s of the CTA owns segment s of the chunk
// (LS consecutive tokens); lane l owns V consecutive channels, so every row
// access of a warp is one contiguous 32*V-element run.  Inputs go straight
// from HBM into registers and are read exactly once.
//
// Per unit:
//   pass 0  per segment: max/min of k and the running-max exponent q.
//   pass 1  per segment summary.  Fast path: every token of the segment is
//           scaled by one fixed reference (its largest k), so each token costs
//           one ex2 and the sums are plain FMAs; the per-token exponentials
//           are kept in registers for pass 2.  If the keys of a segment span
//           too wide a range for one reference, the segment takes the exact
//           running-max recurrence instead.
//   scan    segment summaries are combined through shared memory (each warp
//           folds the summaries before it).  Warp W-1 folds all of them into
//           the chunk summary, publishes it, and finds the state at the start
//           of the chunk by decoupled look-back over the chunks before it
//           (their published summaries or inclusive states), then publishes
//           the inclusive state for the chunks after it.
//   pass 2  outputs of each segment from its start state: fast path reuses the
//           cached exponentials (one more ex2 for the gate, one rcp); the
//           exact path walks the running-max recurrence.
//
// Cross-CTA waits are bounded in time; on expiry the kernel records an error
// in the workspace and writes NaN for the affected outputs instead of waiting.
#pragma once

#include "wkv_common.cuh"

namespace wkv {

constexpr uint32_t kStatusAgg = 1;  // chunk summary published
constexpr uint32_t kStatusInc = 2;  // inclusive state (state after the chunk) published
constexpr uint32_t kErrTimeout = 1;

// First 256 bytes of a workspace.
struct WsHeader {
    uint32_t epoch;     // launch counter: status words carry it, so no reset is needed between calls
    uint32_t done;      // CTAs finished in the current launch
    uint32_t error;     // kErrTimeout bits, sticky until the workspace is re-initialised
    uint32_t err_unit;  // a unit that hit the error
};

struct ChunkArgs {
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const void* r;
    const float* s_in;
    void* y;
    float* s_out;
    int64_t B, T, C;
    int64_t nCB;        // channel blocks per sequence
    int64_t nLB;        // lane blocks = B * nCB
    int64_t nchunks;    // ceil(T / TT)
    int64_t units;      // nLB * nchunks
    WsHeader* hdr;      // null when nchunks == 1
    unsigned long long* status;  // [units]  (epoch << 32) | kind
    float* agg;         // [units][3][CB]  chunk summaries
    float* inc;         // [units][3][CB]  states after each chunk
    int64_t unit_offset;
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Spin (with backoff) until the status word of a chunk carries this launch's
// epoch and a non-zero kind.  Gives up after `limit_ns` of wall time or 2^26
// polls and returns 0.
__device__ __noinline__ unsigned long long wait_status(const unsigned long long* addr, uint32_t epoch,
                                                      uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    unsigned sleep_ns = 32;
    for (uint32_t it = 0; it < (1u << 26); ++it) {
        const unsigned long long s = ld_acquire_u64(addr);
        if (static_cast<uint32_t>(s >> 32) == epoch && (s & 3ull) != 0ull) return s;
        if ((it & 7u) == 7u && global_ns() - t0 > limit_ns) return 0ull;
        __nanosleep(sleep_ns);
        if (sleep_ns < 512) sleep_ns <<= 1;
    }
    return 0ull;
}

template <int V>
__device__ __forceinline__ void publish(float* dst, const St* val, unsigned long long* status,
                                        uint32_t epoch, uint32_t kind, int lane) {
    constexpr int CB = 32 * V;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        __stcg(dst + 0 * CB + lane * V + j, val[j].p);
        __stcg(dst + 1 * CB + lane * V + j, val[j].a);
        __stcg(dst + 2 * CB + lane * V + j, val[j].b);
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_u64(status, (static_cast<unsigned long long>(epoch) << 32) | kind);
}

template <int V>
__device__ __forceinline__ void fetch(const float* src, St* val, int lane) {
    constexpr int CB = 32 * V;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        val[j].p = __ldcg(src + 0 * CB + lane * V + j);
        val[j].a = __ldcg(src + 1 * CB + lane * V + j);
        val[j].b = __ldcg(src + 2 * CB + lane * V + j);
    }
}

// Decoupled look-back, run by one warp: the state at the start of `chunk`
// for this lane block.  `sin` is the state before chunk 0.
template <int V, int TT>
__device__ __forceinline__ void lookback(const ChunkArgs& A, int64_t chunk, int64_t lb, uint32_t epoch,
                                      const float* w2, const St* sin, St* x, int lane) {
    constexpr int CB = 32 * V;
    St acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = st_identity();
    int64_t span = 0;  // tokens summarised by acc (between the found state and `chunk`)
    for (int64_t c = chunk - 1;; --c) {
        if (c < 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = st_combine(sin[j], acc[j], static_cast<float>(span) * w2[j]);
            return;
        }
        const int64_t uj = c * A.nLB + lb;
        unsigned long long s = 0ull;
        if (lane == 0) s = wait_status(A.status + uj, epoch, A.wait_limit_ns);
        s = __shfl_sync(0xffffffffu, s, 0);
        if (s == 0ull) {
            if (lane == 0) {
                atomicOr(&A.hdr->error, kErrTimeout);
                atomicExch(&A.hdr->err_unit, static_cast<uint32_t>(chunk * A.nLB + lb));
            }
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = St{__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                                  __int_as_float(0x7fc00000)};
            return;
        }
        // every lane re-reads the (now ready) word with acquire semantics, so
        // its own payload loads below are ordered after the producer's stores
        s = ld_acquire_u64(A.status + uj);
        const uint32_t kind = static_cast<uint32_t>(s & 3ull);
        St g[V];
        fetch<V>((kind == kStatusInc ? A.inc : A.agg) + uj * 3 * CB, g, lane);
        if (kind == kStatusInc) {
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = st_combine(g[j], acc[j], static_cast<float>(span) * w2[j]);
            return;
        }
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = st_combine(g[j], acc[j], static_cast<float>(span) * w2[j]);
        span += TT;
    }
}

// Thresholds of the fixed-reference fast path, in base-2 exponent units.
// Segment keys: with M = max k, every per-token factor 2^(k-M) and the bonus
// term 2^(u+k-M) stay within [2^-96, 2^96]; values flushed to zero (< 2^-126)
// are then < 2^-30 of the current token's own term.
constexpr float kFastSpan = 96.f;
// Start state against the segment: every term, rescaled to R = max(M, p),
// stays >= 2^-100 times the current token's term.
constexpr float kFastState = 100.f;

template <typename IO, int V, bool GATE, int W, int LS, bool FULL>
__device__ __forceinline__ void chunk_body(const ChunkArgs& A, St (&s_agg)[W][V][32], St (&s_x)[V][32]) {
    constexpr int CB = 32 * V;
    constexpr int TT = W * LS;
    using Ld = Vec<IO, V>;
    using Lf = Vec<float, V>;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t unit = A.unit_offset + blockIdx.x;
    const int64_t chunk = unit / A.nLB;
    const int64_t lb = unit % A.nLB;
    const int64_t b = lb / A.nCB;
    const int64_t c = (lb % A.nCB) * CB + lane * V;
    const bool cvalid = c < A.C;
    const int64_t T = A.T, C = A.C;
    const int64_t lanes = A.B * C;
    const int64_t t_seg = chunk * TT + static_cast<int64_t>(warp) * LS;
    const int64_t chunk_rows = min(static_cast<int64_t>(TT), T - chunk * TT);
    const int nvalid = FULL ? LS : static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), T - t_seg)));
    const bool need_ws = A.nchunks > 1;

    uint32_t epoch = 0;
    if (need_ws && warp == W - 1) {
        if (lane == 0) epoch = ld_relaxed_u32(&A.hdr->epoch);
        epoch = __shfl_sync(0xffffffffu, epoch, 0);
    }

    // ---- per-channel parameters (base 2) ----
    float w2[V], u2[V], dk[V], eu[V];
    {
        typename Lf::raw wr{}, ur{};
        if (cvalid) {
            wr = Lf::load(A.w + c);
            ur = Lf::load(A.u + c);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            w2[j] = cvalid ? Lf::get(wr, j) * kLog2e : 1.f;
            u2[j] = cvalid ? Lf::get(ur, j) * kLog2e : 0.f;
            dk[j] = ex2(-w2[j]);
            eu[j] = ex2(u2[j]);
        }
    }

    // ---- loads: LS rows x V channels of k, v, r ----
    const int64_t base = (b * T + t_seg) * C + c;
    const IO* kp = static_cast<const IO*>(A.k) + base;
    const IO* vp = static_cast<const IO*>(A.v) + base;
    const IO* rp = GATE ? static_cast<const IO*>(A.r) + base : nullptr;
    typename Ld::raw kr[LS], vr[LS], rr[LS];
#pragma unroll
    for (int i = 0; i < LS; ++i) {
        if (cvalid && (FULL || i < nvalid)) {
            kr[i] = Ld::load(kp + i * C);
            vr[i] = Ld::load(vp + i * C);
            if (GATE) rr[i] = Ld::load(rp + i * C);
        } else {
            kr[i] = typename Ld::raw{};
            vr[i] = typename Ld::raw{};
            rr[i] = typename Ld::raw{};
        }
    }

    // ---- pass 0: key range and running-max exponent of the segment ----
    float kf[LS][V];
    float kmax[V], kmin[V], q[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        kmax[j] = -3.0e38f;
        kmin[j] = 3.0e38f;
        q[j] = kFreshP2;
    }
#pragma unroll
    for (int i = 0; i < LS; ++i) {
        if (FULL || i < nvalid) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float k2 = Ld::get(kr[i], j) * kLog2e;
                kf[i][j] = k2;
                kmax[j] = fmaxf(kmax[j], k2);
                kmin[j] = fminf(kmin[j], k2);
                q[j] = fmaxf(q[j] - w2[j], k2);
            }
        }
    }
    bool fast1 = true;
#pragma unroll
    for (int j = 0; j < V; ++j) fast1 = fast1 && (kmax[j] - kmin[j] + fabsf(u2[j]) <= kFastSpan);

    // ---- pass 1: segment summary ----
    St seg[V];
    if (nvalid == 0) {
#pragma unroll
        for (int j = 0; j < V; ++j) seg[j] = st_identity();
    } else if (fast1) {
        float n[V], db[V];
#pragma unroll
        for (int j = 0; j < V; ++j) n[j] = db[j] = 0.f;
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float ek = ex2(kf[i][j] - kmax[j]);
                    kf[i][j] = ek;
                    n[j] = fmaf(n[j], dk[j], ek * Ld::get(vr[i], j));
                    db[j] = fmaf(db[j], dk[j], ek);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float s = ex2(kmax[j] - q[j]);
            seg[j] = St{q[j], n[j] * s, db[j] * s};
        }
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) seg[j] = st_identity();
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float vv = Ld::get(vr[i], j);
                    const float pd = seg[j].p - w2[j];
                    const float d2 = pd - kf[i][j];
                    const float e = ex2(-fabsf(d2));
                    if (d2 >= 0.f) {
                        seg[j].a = fmaf(e, vv, seg[j].a);
                        seg[j].b += e;
                        seg[j].p = pd;
                    } else {
                        seg[j].a = fmaf(e, seg[j].a, vv);
                        seg[j].b = fmaf(e, seg[j].b, 1.f);
                        seg[j].p = kf[i][j];
                    }
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) s_agg[warp][j][lane] = seg[j];
    __syncthreads();

    // ---- scan over the segments of this chunk ----
    St lp[V];  // summary of segments 0..warp-1
#pragma unroll
    for (int j = 0; j < V; ++j) lp[j] = st_identity();
    for (int s = 0; s < warp; ++s) {
        const int len = FULL ? LS : static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), chunk_rows - s * LS)));
#pragma unroll
        for (int j = 0; j < V; ++j) lp[j] = st_combine(lp[j], s_agg[s][j][lane], static_cast<float>(len) * w2[j]);
    }
    if (warp == W - 1) {
        St agg[V], sin[V], x[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            agg[j] = st_combine(lp[j], seg[j], static_cast<float>(nvalid) * w2[j]);
            if (A.s_in != nullptr && cvalid) {
                const int64_t li = b * C + c + j;
                sin[j] = St{A.s_in[2 * lanes + li] * kLog2e, A.s_in[li], A.s_in[lanes + li]};
            } else {
                sin[j] = st_identity();
            }
        }
        const bool last = chunk == A.nchunks - 1;
        const int64_t uoff = unit * 3 * CB;
        if (chunk == 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = sin[j];
        } else {
            if (!last) publish<V>(A.agg + uoff, agg, A.status + unit, epoch, kStatusAgg, lane);
            lookback<V, TT>(A, chunk, lb, epoch, w2, sin, x, lane);
        }
        St incl[V];
#pragma unroll
        for (int j = 0; j < V; ++j) incl[j] = st_combine(x[j], agg[j], static_cast<float>(chunk_rows) * w2[j]);
        if (need_ws && !last) publish<V>(A.inc + uoff, incl, A.status + unit, epoch, kStatusInc, lane);
        if (last && A.s_out != nullptr && cvalid) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const int64_t li = b * C + c + j;
                A.s_out[li] = incl[j].a;
                A.s_out[lanes + li] = incl[j].b;
                A.s_out[2 * lanes + li] = incl[j].p * kLn2;
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) s_x[j][lane] = x[j];
        if (need_ws && lane == 0) {
            const uint32_t before = atomicAdd(&A.hdr->done, 1u);
            if (before == static_cast<uint32_t>(A.units - 1)) {
                // every CTA of this launch has read the epoch; start the next one
                A.hdr->done = 0u;
                __threadfence();
                atomicAdd(&A.hdr->epoch, 1u);
            }
        }
    }
    __syncthreads();
    if (nvalid == 0 || !cvalid) return;

    // ---- pass 2: outputs of this segment ----
    St st[V];
#pragma unroll
    for (int j = 0; j < V; ++j)
        st[j] = st_combine(s_x[j][lane], lp[j], static_cast<float>(warp * LS) * w2[j]);
    bool fast2 = fast1;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const bool near = st[j].p >= kmax[j] - kFastState;
        const bool negligible = st[j].p < kmax[j] - 1.5f * kFastState && st[j].b <= 16777216.f;
        fast2 = fast2 && (st[j].p - kmin[j] + fabsf(u2[j]) <= kFastState) && (near || negligible);
    }
    IO* yp = static_cast<IO*>(A.y) + base;
    if (fast2) {
        float n[V], db[V], sl[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float R = fmaxf(kmax[j], st[j].p);
            sl[j] = ex2(kmax[j] - R);
            const float ss = ex2(st[j].p - R);
            n[j] = st[j].a * ss;
            db[j] = st[j].b * ss;
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
                float out[V];
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float ek = kf[i][j] * sl[j];
                    const float ekv = ek * Ld::get(vr[i], j);
                    const float num = fmaf(eu[j], ekv, n[j]);
                    float den = fmaf(eu[j], ek, db[j]);
                    if (GATE) den *= gate_den(Ld::get(rr[i], j));
                    out[j] = num * rcp(den);
                    n[j] = fmaf(n[j], dk[j], ekv);
                    db[j] = fmaf(db[j], dk[j], ek);
                }
                Ld::store(yp + i * C, out);
            }
        }
    } else {
        if (fast1) {
            // pass 1 replaced the keys by their exponentials: read them again
#pragma unroll
            for (int i = 0; i < LS; ++i) {
                if (FULL || i < nvalid) {
                    const auto kk = Ld::load(kp + i * C);
#pragma unroll
                    for (int j = 0; j < V; ++j) kf[i][j] = Ld::get(kk, j) * kLog2e;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
                float out[V];
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float gd = GATE ? gate_den(Ld::get(rr[i], j)) : 1.f;
                    out[j] = lane_token(st[j].a, st[j].b, st[j].p, w2[j], u2[j], kf[i][j],
                                        Ld::get(vr[i], j), gd, 1.f);
                }
                Ld::store(yp + i * C, out);
            }
        }
    }
}

template <typename IO, int V, bool GATE, int W, int LS>
__global__ void __launch_bounds__(W * 32)
chunk_forward_kernel(const ChunkArgs A) {
    __shared__ St s_agg[W][V][32];
    __shared__ St s_x[V][32];
    constexpr int TT = W * LS;
    const int64_t unit = A.unit_offset + blockIdx.x;
    const int64_t chunk = unit / A.nLB;
    if ((chunk + 1) * TT <= A.T)
        chunk_body<IO, V, GATE, W, LS, true>(A, s_agg, s_x);
    else
        chunk_body<IO, V, GATE, W, LS, false>(A, s_agg, s_x);
}

}  // namespace wkv
