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
// Cross-chunk protocol: every published state is a 16-byte word per channel
// carrying the launch epoch and its kind, so readers validate what they read
// without flags or fences.  Cross-CTA waits are bounded in time; on expiry the
// kernel records an error in the workspace and writes NaN for the affected
// outputs instead of waiting.
#pragma once

#include <cuda.h>

#include "wkv_common.cuh"

namespace wkv {

constexpr uint32_t kKindAgg = 1;  // chunk summary (from the empty state)
constexpr uint32_t kKindInc = 2;  // inclusive state (state after the chunk)
constexpr uint32_t kKindChain = 3; // state a call of a chunk chain leaves (epoch: position in the chain)
constexpr uint32_t kErrTimeout = 1;
// Limit of a wait for this CTA's own TMA copies to land.  Unlike the waits on
// other CTAs it does not follow the configurable limit: a CTA must not exit
// while a copy into its shared memory is still in flight.
constexpr uint64_t kCopyWaitNs = 2000000000ull;

// First 256 bytes of a workspace.
struct WsHeader {
    uint32_t epoch;     // launch counter: words carry it, so no reset is needed between calls
    uint32_t done;      // CTAs finished in the current launch
    uint32_t error;     // kErrTimeout bits, sticky until the workspace is re-initialised
    uint32_t err_unit;  // a unit that hit the error
    uint32_t ticket;    // next unit to claim (part and register-load look-back kernels)
};

// One published state of one channel, (p, a, b) as is, plus a tag = (launch
// epoch mod 2^30) << 2 | kind.  Written and read as one aligned 16-byte
// access, so a reader sees either the whole word or none of it and needs no
// separate flag or fence.
struct alignas(16) Word {
    float p, a, b;
    uint32_t tag;
};

__device__ __forceinline__ uint32_t word_tag(uint32_t epoch, uint32_t kind) { return (epoch << 2) | kind; }

struct ChunkArgs {
    const float* w;
    const float* u;
    const void* k;
    const void* v;
    const void* r;
    const float* s_in;
    void* y;            // null: only the state is wanted (no pass 2, no output)
    float* s_out;
    int64_t B, T, C;
    int64_t nCB;        // channel blocks per sequence
    int64_t nLB;        // lane blocks = B * nCB
    int64_t nchunks;    // ceil(T / TT)
    int64_t units;      // nLB * nchunks
    WsHeader* hdr;      // null when nchunks == 1
    Word* aggw;         // [units][CB] chunk summaries
    Word* incw;         // [units][CB] states after each chunk
    St* ckpt;           // lane-resident kernel only, or null: [nchunks + 1][nLB][CB] base-2 states
                        // entering each chunk, the last one the state after the sequence
    uint64_t wait_limit_ns;
    uint32_t early;     // stream kernel: inputs may be read before the previous kernel of the stream ends
    // stream kernel, chunk chains: [B * C] words the state after the call is
    // published to (null: none), the position in the chain whose word holds
    // the entering state (0: the chain's first call reads s_in), and the
    // position the published words carry
    Word* chain;
    uint32_t chain_in, chain_out;
    // stream kernel: first token of the launch within the arrays (the
    // arrays' own T is the tensor maps'; this launch covers T tokens)
    int64_t t0;
};

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

__device__ __forceinline__ void st_word(Word* dst, St s, uint32_t tag) {
    asm volatile("st.relaxed.gpu.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(__float_as_uint(s.p)),
                 "r"(__float_as_uint(s.a)), "r"(__float_as_uint(s.b)), "r"(tag)
                 : "memory");
}

__device__ __forceinline__ Word ld_word(const Word* src) {
    uint32_t p, a, b, t;
    asm volatile("ld.relaxed.gpu.global.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(p), "=r"(a), "=r"(b), "=r"(t)
                 : "l"(src)
                 : "memory");
    return Word{__uint_as_float(p), __uint_as_float(a), __uint_as_float(b), t};
}

__device__ __forceinline__ St word_state(const Word& w) { return St{w.p, w.a, w.b}; }

// Each lane publishes the words of its own V channels.
template <int V>
__device__ __forceinline__ void publish(Word* dst, const St* val, uint32_t epoch, uint32_t kind, int lane) {
#pragma unroll
    for (int j = 0; j < V; ++j) st_word(dst + lane * V + j, val[j], word_tag(epoch, kind));
}

// Windowed decoupled look-back state, kept by the warp that looks back for
// one unit: `acc` summarises the chunks already folded (from chunk `cur`+1
// up to the unit), `span` their token count, `x` the result once `done`.
template <int V>
struct LookState {
    St acc[V];
    St x[V];
    int64_t cur;
    int64_t span;
    bool done;
};

constexpr int kWin = 4;

// One round of the look-back: every lane reads the summary and inclusive
// words of its own channels for chunks cur, cur-1, ..., cur-WIN+1 (one
// round trip), then the warp walks them nearest first.  A chunk counts as
// published only if every lane saw its word with this launch's epoch, so all
// lanes take the same path with data they observed themselves.  The walk
// stops at the first inclusive state (or at the start of the sequence, where
// `sin` takes its place) and otherwise folds summaries into acc.  Returns
// true if it made progress.
template <int V, int TT, int WIN = kWin>
__device__ __forceinline__ bool lookback_round(const ChunkArgs& A, int64_t lb, uint32_t epoch, const float* w2,
                                               const St* sin, LookState<V>& L, int lane) {
    constexpr int CB = 32 * V;
    Word wi[WIN][V], wa[WIN][V];
#pragma unroll
    for (int l = 0; l < WIN; ++l) {
        const int64_t c = L.cur - l;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            if (c >= 0) {
                const int64_t off = (c * A.nLB + lb) * CB + lane * V + j;
                wi[l][j] = ld_word(A.incw + off);
                wa[l][j] = ld_word(A.aggw + off);
            } else {
                wi[l][j] = Word{0.f, 0.f, 0.f, 0u};
                wa[l][j] = Word{0.f, 0.f, 0.f, 0u};
            }
        }
    }
    bool progressed = false;
#pragma unroll
    for (int l = 0; l < WIN; ++l) {
        if (L.cur < 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) L.x[j] = st_combine(sin[j], L.acc[j], static_cast<float>(L.span) * w2[j]);
            L.done = true;
            return true;
        }
        bool inc = true, agg = true;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            inc = inc && wi[l][j].tag == word_tag(epoch, kKindInc);
            agg = agg && wa[l][j].tag == word_tag(epoch, kKindAgg);
        }
        if (__all_sync(0xffffffffu, inc)) {
#pragma unroll
            for (int j = 0; j < V; ++j)
                L.x[j] = st_combine(word_state(wi[l][j]), L.acc[j], static_cast<float>(L.span) * w2[j]);
            L.done = true;
            return true;
        }
        if (!__all_sync(0xffffffffu, agg)) return progressed;
#pragma unroll
        for (int j = 0; j < V; ++j)
            L.acc[j] = st_combine(word_state(wa[l][j]), L.acc[j], static_cast<float>(L.span) * w2[j]);
        L.span += TT;
        L.cur -= 1;
        progressed = true;
    }
    return progressed;
}

// Blocking look-back: rounds with backoff until the start state is known or
// `limit_ns` passes (then x is NaN and the function returns false).
template <int V, int TT, int WIN = kWin>
__device__ __forceinline__ bool lookback_finish(const ChunkArgs& A, int64_t lb, uint32_t epoch, const float* w2,
                                                const St* sin, LookState<V>& L, int lane) {
    const uint64_t t0 = global_ns();
    unsigned sleep_ns = 32;
    while (!L.done) {
        if (!lookback_round<V, TT, WIN>(A, lb, epoch, w2, sin, L, lane)) {
            if (global_ns() - t0 > A.wait_limit_ns) {
                const float nan = __int_as_float(0x7fc00000);
#pragma unroll
                for (int j = 0; j < V; ++j) L.x[j] = St{nan, nan, nan};
                return false;
            }
            __nanosleep(sleep_ns);
            if (sleep_ns < 256) sleep_ns <<= 1;
        }
    }
    return true;
}

template <int V>
__device__ __forceinline__ void look_init(LookState<V>& L, int64_t chunk) {
#pragma unroll
    for (int j = 0; j < V; ++j) L.acc[j] = st_identity();
    L.cur = chunk - 1;
    L.span = 0;
    L.done = false;
}

__device__ __forceinline__ void record_timeout(const ChunkArgs& A, int64_t unit) {
    atomicOr(&A.hdr->error, kErrTimeout);
    atomicExch(&A.hdr->err_unit, static_cast<uint32_t>(unit));
}

// Thresholds of the fixed-reference fast path, in base-2 exponent units.
// Segment keys: with M = max k, every per-token factor 2^(k-M) and the bonus
// term 2^(u+k-M) stay within [2^-96, 2^96]; values flushed to zero (< 2^-126)
// are then < 2^-30 of the current token's own term.
constexpr float kFastSpan = 96.f;
// Start state against the segment: every term, rescaled to R = max(M, p),
// stays >= 2^-100 times the current token's term.
constexpr float kFastState = 100.f;

// One unit (CB channels of one sequence x one chunk of TT tokens), run by
// the whole CTA.  SMEM selects where the rows come from: false = straight
// from global memory into registers (all loads issued up front); true = a
// shared-memory stage that a TMA copy filled (rows read as they are used).
// `stage` points at the stage's k tile; v and r tiles follow it.
template <typename IO, int V, bool GATE, int W, int LS, bool FULL, bool SMEM>
__device__ __forceinline__ void unit_body(const ChunkArgs& A, int64_t unit, uint32_t epoch,
                                          const unsigned char* stage, St (&s_agg)[W][V][32],
                                          St (&s_x)[V][32]) {
    constexpr int CB = 32 * V;
    constexpr int TT = W * LS;
    constexpr int ROW = CB * static_cast<int>(sizeof(IO));     // bytes of one tile row
    constexpr int TILE = TT * ROW;
    using Ld = Vec<IO, V>;
    using Lf = Vec<float, V>;
    using Raw = typename Ld::raw;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
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

    // ---- row access ----
    const int64_t base = (b * T + t_seg) * C + c;
    const IO* kp = static_cast<const IO*>(A.k) + base;
    const IO* vp = static_cast<const IO*>(A.v) + base;
    const IO* rp = GATE ? static_cast<const IO*>(A.r) + base : nullptr;
    const unsigned char* srow = stage + warp * LS * ROW + lane * V * static_cast<int>(sizeof(IO));
    Raw kr[LS], vr[LS], rr[LS];
    if constexpr (!SMEM) {
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (cvalid && (FULL || i < nvalid)) {
                kr[i] = Ld::load(kp + i * C);
                vr[i] = Ld::load(vp + i * C);
                if (GATE) rr[i] = Ld::load(rp + i * C);
            } else {
                kr[i] = Raw{};
                vr[i] = Raw{};
                rr[i] = Raw{};
            }
        }
    }
    auto krow = [&](int i) -> Raw {
        if constexpr (SMEM) return *reinterpret_cast<const Raw*>(srow + i * ROW);
        else return kr[i];
    };
    auto vrow = [&](int i) -> Raw {
        if constexpr (SMEM) return *reinterpret_cast<const Raw*>(srow + TILE + i * ROW);
        else return vr[i];
    };
    auto rrow = [&](int i) -> Raw {
        if constexpr (SMEM) return *reinterpret_cast<const Raw*>(srow + 2 * TILE + i * ROW);
        else return rr[i];
    };

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
            const Raw kk = krow(i);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float k2 = Ld::get(kk, j) * kLog2e;
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
                const Raw vv = vrow(i);
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float ek = ex2(kf[i][j] - kmax[j]);
                    kf[i][j] = ek;
                    n[j] = fmaf(n[j], dk[j], ek * Ld::get(vv, j));
                    db[j] = fmaf(db[j], dk[j], ek);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float sc = ex2(kmax[j] - q[j]);
            seg[j] = St{q[j], n[j] * sc, db[j] * sc};
        }
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) seg[j] = st_identity();
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
                const Raw vr_ = vrow(i);
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float vv = Ld::get(vr_, j);
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
    for (int sg = 0; sg < warp; ++sg) {
        const int len = FULL ? LS : static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(LS), chunk_rows - sg * LS)));
#pragma unroll
        for (int j = 0; j < V; ++j) lp[j] = st_combine(lp[j], s_agg[sg][j][lane], static_cast<float>(len) * w2[j]);
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
        const int64_t uoff = unit * CB;
        if (chunk == 0) {
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = sin[j];
        } else {
            if (!last) publish<V>(A.aggw + uoff, agg, epoch, kKindAgg, lane);
            LookState<V> L;
            look_init<V>(L, chunk);
            if (!lookback_finish<V, TT>(A, lb, epoch, w2, sin, L, lane) && lane == 0) record_timeout(A, unit);
#pragma unroll
            for (int j = 0; j < V; ++j) x[j] = L.x[j];
        }
        St incl[V];
#pragma unroll
        for (int j = 0; j < V; ++j) incl[j] = st_combine(x[j], agg[j], static_cast<float>(chunk_rows) * w2[j]);
        if (need_ws && !last) publish<V>(A.incw + uoff, incl, epoch, kKindInc, lane);
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
    }
    __syncthreads();
    if (nvalid == 0 || !cvalid || A.y == nullptr) return;

    // ---- pass 2: outputs of this segment (none when only the state is wanted) ----
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
                const Raw vv = vrow(i);
                Raw rv{};
                if (GATE) rv = rrow(i);
                float out[V];
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float ek = kf[i][j] * sl[j];
                    const float ekv = ek * Ld::get(vv, j);
                    const float num = fmaf(eu[j], ekv, n[j]);
                    float den = fmaf(eu[j], ek, db[j]);
                    if (GATE) den *= gate_den(Ld::get(rv, j));
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
                    Raw kk;
                    if constexpr (SMEM) kk = krow(i);
                    else kk = Ld::load(kp + i * C);
#pragma unroll
                    for (int j = 0; j < V; ++j) kf[i][j] = Ld::get(kk, j) * kLog2e;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < LS; ++i) {
            if (FULL || i < nvalid) {
                const Raw vv = vrow(i);
                Raw rv{};
                if (GATE) rv = rrow(i);
                float out[V];
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const float gd = GATE ? gate_den(Ld::get(rv, j)) : 1.f;
                    out[j] = lane_token(st[j].a, st[j].b, st[j].p, w2[j], u2[j], kf[i][j], Ld::get(vv, j), gd,
                                        1.f);
                }
                Ld::store(yp + i * C, out);
            }
        }
    }
}

// Last CTA of a launch (by the count of finished CTAs) starts the next
// launch's epoch and resets the counters.  Every CTA read the epoch before
// it counted itself, so no CTA of this launch can see the new value.
__device__ __forceinline__ void finish_launch(const ChunkArgs& A, uint32_t ctas) {
    const uint32_t before = atomicAdd(&A.hdr->done, 1u);
    if (before == ctas - 1u) {
        A.hdr->done = 0u;
        A.hdr->ticket = 0u;
        __threadfence();
        atomicAdd(&A.hdr->epoch, 1u);
    }
}

// One unit per CTA, rows loaded from global memory into registers.  Takes
// any alignment that the vector width allows.  With a workspace, a CTA
// claims its unit from the workspace's ticket counter, so units are taken in
// chunk-major order whatever order the hardware starts the CTAs in: a unit
// only waits on units of earlier chunks, which CTAs already running hold.
template <typename IO, int V, bool GATE, int W, int LS>
__global__ void __launch_bounds__(W * 32)
chunk_forward_kernel(const ChunkArgs A) {
    __shared__ St s_agg[W][V][32];
    __shared__ St s_x[V][32];
    __shared__ uint32_t s_epoch;
    __shared__ int64_t s_unit;
    constexpr int TT = W * LS;
    const bool need_ws = A.nchunks > 1;
    if (threadIdx.x == 0) {
        s_epoch = need_ws ? ld_relaxed_u32(&A.hdr->epoch) : 0u;
        s_unit = need_ws ? static_cast<int64_t>(atomicAdd(&A.hdr->ticket, 1u)) : static_cast<int64_t>(blockIdx.x);
    }
    __syncthreads();
    const uint32_t epoch = s_epoch;
    const int64_t unit = s_unit;
    const int64_t chunk = unit / A.nLB;
    if ((chunk + 1) * TT <= A.T)
        unit_body<IO, V, GATE, W, LS, true, false>(A, unit, epoch, nullptr, s_agg, s_x);
    else
        unit_body<IO, V, GATE, W, LS, false, false>(A, unit, epoch, nullptr, s_agg, s_x);
    if (need_ws && threadIdx.x == 0) finish_launch(A, static_cast<uint32_t>(A.units));
}

// ---------------------------------------------------------------------------
// persistent kernel: TMA tiles into a shared-memory ring, one unit per turn
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for a phase of an mbarrier; false after `limit_ns` (or 2^26 polls).
// The common case (phase already complete) stays inline; the polling loop
// is out of line.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 26); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u && global_ns() - t0 > limit_ns) return false;
    }
    return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, limit_ns);
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace wkv
