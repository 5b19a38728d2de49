// wkv5_tc.cuh -- the matrix-state WKV in blocks of tokens on the tensor cores
// (tcgen05, kind::tf32, accumulators in tensor memory).
//
// Same operator as wkv5.cuh (the reading of the article "RWKVアーキテクチャ
// 徹底解説", "RWKVバージョンの進化 / v4からv7まで"): per head an N x N state S,
//   y_t[j] = sum_i r_t[i] ( S[i][j] + u[i] k_t[i] v_t[j] ),
//   S[i][j] <- e^{-w_t[i]} S[i][j] + k_t[i] v_t[j].
// Over a block of L tokens entered with state S0, with Lam_t[i] the sum of
// the block's decay rates before token t (Lam_0 = 0, Lam_L the block's
// total), the outputs and the state after the block are the same sums
// regrouped into matrix products:
//
//   y_t  = sum_i r_t[i] e^{-Lam_t[i]} S0[i][:]                     (inter)
//        + sum_{s<t} A[t][s] v_s + (sum_i r_t[i] u[i] k_t[i]) v_t  (intra)
//   A[t][s] = sum_i r_t[i] e^{-(Lam_t - Lam_m)[i]} k_s[i] e^{(Lam_{s+1} - Lam_m)[i]}
//   S_L  = e^{-Lam_L} S0 + sum_s (k_s e^{-(Lam_L - Lam_{s+1})}) (x) v_s
//
// with any reference m; m is the block's middle token.  Every factor is
// formed in fp32 and each product of two factors that the sums keep has
// exponent -(Lam_t - Lam_{s+1}) <= 0.  The factors themselves stay finite
// while every |Lam_t - Lam_m| <= kTcSpan, so a window of 64 tokens is cut
// into blocks of 64, 16, 4 or 1 tokens: the longest for which that holds on
// every channel (always 64 for decays up to 1.8 per token; a block of one
// token is exact for any decay).  A block of fewer tokens leaves the rest of
// the 64-row tiles zero.
//
// One CTA of 256 threads per (sequence, head), N = 64, bf16 r, k, v, y.
// Per block, five 64 x 64 products on the tensor cores, M = N = 64, K = 64
// in 8 steps of 8, operands fp32 in shared memory read as tf32, K-major,
// no swizzle:
//   batch 1:  D_A  = R~ K~^T          (scores before masking)
//             D_Y  = R~ S0'           (inter outputs)
//             D_S  = hi(K^)^T V       (state increment)
//   batch 2:  D_Y += mask(D_A) V      (intra outputs and the bonus diagonal)
//             D_S += lo(K^)^T V
// R~ = r e^{-(Lam_t - Lam_m)} already carries the inter factor but for a
// per-channel e^{-Lam_m}, which goes into the state instead: S0' =
// diag(e^{-Lam_m}) S0, so R~ S0' = sum_i r_t[i] e^{-Lam_t[i]} S0[i][:].
// K^ = k e^{-(Lam_L - Lam_{s+1})} is split into hi + lo (hi: the 19 bits tf32
// keeps, lo: the rest), so the state increment keeps fp32 accuracy (v is
// bf16, exact in tf32); the outputs take the tf32 products (errors of order
// 1e-3 of the output scale, below the bf16 output's own rounding).  The state
// S stays fp32 in registers: the M = 64 accumulator layout puts row 16q + l
// in lane l of tensor-memory lane quarter q; warps q and q + 4 read that
// quarter, the first columns [0, 32), the second [32, 64), with the
// 16-lane x 256-bit load shape, in which thread l holds rows l / 4 and
// l / 4 + 8 of the 16 and, of every 8 columns, columns 2 (l % 4) and
// 2 (l % 4) + 1: 16 entries of S per thread.
// One thread issues the MMAs; tcgen05.commit arrives on an mbarrier that the
// others wait on (bounded).  A window's r, k, v come by TMA into one stage,
// refilled once the window's last block has read it; per-token decays come
// by TMA into the staged state's tile, which is free from the last block's
// first batch of products until the next window's stage 1 writes it (the
// decays are read before that; a window cut into blocks shorter than 64
// tokens reads them from global memory instead).  So two CTAs fit per SM
// (112.8 KB of shared memory, at most 128 registers).  Tensor memory: 3
// accumulators of 64 columns, 256 columns allocated per CTA.
#pragma once

#include <cuda_bf16.h>

#include "wkv5.cuh"
#include "wkv_chunk.cuh"

namespace wkv {

// Operand tile layout (K-major, no swizzle), in 16-byte slots: a core matrix
// is 8 rows of one slot each; the two core matrices of an 8-wide k step sit
// kTcLbo slots apart, 8-row groups kTcSbo slots apart, k steps kTcKs slots
// apart.  The odd offsets (9, 17, 138: one slot of padding per core matrix
// pair, two per k step) put the 8 slots a warp touches when it writes one
// row across 32 consecutive k, or 8 rows of one slot, in 8 different bank
// groups, so the staging stores do not conflict.
constexpr uint32_t kTcLbo = 9, kTcSbo = 17, kTcKs = 138;
constexpr uint32_t kTcTile = (7 * kTcKs + 8 * kTcSbo) * 16;   // one fp32 operand tile (17632 bytes)
constexpr uint32_t kTcTiles = 5 * kTcTile;          // R~, K~, hi(K^)^T, V^T, S0'^T
// Staging ring: a window's r, k, v (bf16) and, with per-token decays, w (fp32)
// as 64 tokens x 64 channels, brought by TMA one window ahead.
struct TcStage {
    static constexpr uint32_t IO = 64 * 64 * 2;                   // one bf16 array
    static constexpr uint32_t BYTES = 3 * IO;                     // r, k, v of a window
    static constexpr int MINB = 2;                                // CTAs per SM
    static constexpr uint32_t BASE = (kTcTiles + 127u) & ~127u;   // the stage, 128-byte aligned
    static constexpr uint32_t SMEM = BASE + BYTES;                // tiles, then the stage
    static_assert(64 * 64 * 4 <= kTcTile, "a window's decays fit the state's tile");
};
constexpr uint32_t kTcCols = 256;                   // tensor memory columns allocated
constexpr float kTcSpan = 60.f;                     // bound of |Lam_t - Lam_m| (natural units)
constexpr int kTcThreads = 256;                     // 8 warps: 2 per lane quarter of tensor memory

// Byte offset of element (row, k) of a 64 x 64 fp32 operand tile.
__host__ __device__ __forceinline__ uint32_t tc_off(int row, int k) {
    const uint32_t slot = static_cast<uint32_t>(k >> 3) * kTcKs + static_cast<uint32_t>(row >> 3) * kTcSbo +
                          static_cast<uint32_t>((k >> 2) & 1) * kTcLbo + static_cast<uint32_t>(row & 7);
    return slot * 16u + static_cast<uint32_t>(k & 3) * 4u;
}

// Shared-memory matrix descriptor of one k step of such a tile.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(kTcLbo) << 16;       // leading byte offset (16-byte units)
    d |= static_cast<uint64_t>(kTcSbo) << 32;       // stride byte offset (16-byte units)
    d |= static_cast<uint64_t>(1u) << 46;           // descriptor version of this generation
    return d;                                       // base offset 0, no swizzle
}

// Instruction descriptor: D fp32, A and B tf32, both K-major, N = 64, M = 64.
constexpr uint32_t kTcIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((64u >> 3) << 17) | ((64u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(kTcIdesc), "r"(acc)
        : "memory");
}

// D (+)= A B^T over K = 64: A, B 64 x 64 tiles (rows x k) at shared addresses a, b.
__device__ __forceinline__ void tc_gemm(uint32_t d, uint32_t a, uint32_t b, bool accumulate) {
#pragma unroll
    for (int s = 0; s < 8; ++s)
        tc_mma(d, tc_desc(a + kTcKs * 16u * s), tc_desc(b + kTcKs * 16u * s), (accumulate || s > 0) ? 1u : 0u);
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 accumulator rows (lanes 0..15 of the warp's lane quarter) x 32 columns
// from taddr's column (warp-wide, 16-lane x 256-bit shape, 4 repeats):
// x[4 g + 2 h + e] = row l / 4 + 8 h, column 8 g + 2 (l % 4) + e.
__device__ __forceinline__ void tc_ld16x32(uint32_t taddr, float* x) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int q = 0; q < 16; ++q) x[q] = __uint_as_float(r[q]);
}

__device__ __forceinline__ void tc_st(unsigned char* tile, int row, int k, float x) {
    *reinterpret_cast<float*>(tile + tc_off(row, k)) = x;
}
// two consecutive k (k even) of one row: half a slot
__device__ __forceinline__ void tc_st2(unsigned char* tile, int row, int k, float a, float b) {
    *reinterpret_cast<float2*>(tile + tc_off(row, k)) = make_float2(a, b);
}
// four consecutive k (k % 4 == 0) of one row: one slot
__device__ __forceinline__ void tc_st4(unsigned char* tile, int row, int k, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(tile + tc_off(row, k)) = make_float4(a, b, c, d);
}

// Longest block (64, 16, 4 or 1 tokens) whose blocks keep |Lam_t - Lam_m|
// within kTcSpan for this channel over the window's n tokens, m the middle
// token of each block (a block of bl tokens: m = bl / 2, the last block may
// be shorter).  rate(t): the channel's decay rate at token t of the window.
template <typename Rate>
__device__ __forceinline__ int tc_block_len(int n, Rate rate) {
    const int cand[3] = {64, 16, 4};
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        const int L = cand[c];
        bool ok = true;
        for (int b0 = 0; b0 < n && ok; b0 += L) {
            const int bl = n - b0 < L ? n - b0 : L, mid = bl / 2;
            float first = 0.f, second = 0.f;   // decay before and after the middle
            for (int t = 0; t < bl; ++t) {
                if (t < mid) first += rate(b0 + t);
                else second += rate(b0 + t);
            }
            ok = first <= kTcSpan && second <= kTcSpan;
        }
        if (ok) return L;
    }
    return 1;
}

template <bool PERTOK>
__global__ void __launch_bounds__(kTcThreads, TcStage::MINB)
    wkv5_tc_kernel(const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tw, const Wkv5Args A) {
    using SG = TcStage;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* RT = smem;                  // R~ [t][i]; after batch 1: lo(K^)^T [i][s]
    unsigned char* KT = smem + kTcTile;        // K~ [s][i]; after batch 1: the masked scores [t][s]
    unsigned char* KH = smem + 2 * kTcTile;    // hi(K^)^T [i][s]
    unsigned char* VT = smem + 3 * kTcTile;    // V^T [j][s]
    unsigned char* ST = smem + 4 * kTcTile;    // S0'^T [j][i] = e^{-Lam_m[i]} S0[i][j]; per-token decays [t][i]
    __shared__ __align__(8) uint64_t bar[2], full[2];   // full[0]: r, k, v; full[1]: the decays
    __shared__ uint32_t tslot;
    __shared__ float s_u[64], s_eend[64], s_emid[64];
    __shared__ float s_wq[PERTOK ? 4 : 1][64];   // per-token decays: sums over the window's quarters

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // staging: channel ci, tokens [16 qq, 16 qq + 16) of a block
    const int ci = tid & 63, qq = tid >> 6;
    // accumulators: warp w reads lane quarter w % 4 (rows 16 (w % 4) .. + 15)
    // and columns [c0, c0 + 32); this thread holds rows R0 + 8 h and, of
    // every 8 columns from c0, columns 2 (lane % 4) + e
    const int R0 = 16 * (warp & 3) + (lane >> 2);
    const int c0 = 32 * (warp >> 2);
    const int cl = 2 * (lane & 3);
    const int64_t bh = blockIdx.x, b = bh / A.H, h = bh % A.H;
    const int64_t T = A.T, C = A.C;
    const int64_t ch0 = h * 64;
    __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(A.y);
    const float nan = __int_as_float(0x7fc00000);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // TMA of window wi's r, k, v into the stage, and of its decays into the
    // state's tile
    auto fetch = [&](int64_t wi) {
        unsigned char* st = smem + SG::BASE;
        mbar_expect_tx(&full[0], SG::BYTES);
        const int x = static_cast<int>(ch0), y = static_cast<int>(wi * 64), z = static_cast<int>(b);
        tma_load_3d(st, &tr, x, y, z, &full[0]);
        tma_load_3d(st + SG::IO, &tk, x, y, z, &full[0]);
        tma_load_3d(st + 2 * SG::IO, &tv, x, y, z, &full[0]);
    };
    auto fetch_w = [&](int64_t wi) {
        mbar_expect_tx(&full[1], 64u * 64u * 4u);
        tma_load_3d(ST, &tw, static_cast<int>(ch0), static_cast<int>(wi * 64), static_cast<int>(b), &full[1]);
    };
    if (tid == 0) {
        prefetch_tensormap(&tr);
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (PERTOK) prefetch_tensormap(&tw);
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fetch(0);
        if (PERTOK) fetch_w(0);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tslot)),
                     "r"(kTcCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid < 64) s_u[tid] = A.u[ch0 + tid];
    // the state this thread owns: S[4 g + 2 hh + e] = S[R0 + 8 hh][c0 + 8 g + cl + e]
    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) S[j] = 0.f;
    if (A.s_in != nullptr) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float* src = A.s_in + (bh * 64 + R0 + 8 * hh) * 64 + c0 + cl;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const float2 x = *reinterpret_cast<const float2*>(src + 8 * g);
                S[4 * g + 2 * hh] = x.x;
                S[4 * g + 2 * hh + 1] = x.y;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tslot;
    // the accumulators (lane 0, column base of the allocation + offset); the
    // loads add this warp's lane quarter and column half
    const uint32_t tA = tbase, tY = tbase + 64, tS = tbase + 128;
    const uint32_t lane_off = (static_cast<uint32_t>(32 * (warp & 3)) << 16) + static_cast<uint32_t>(c0);
    const uint32_t aRT = smem_u32(RT), aKT = smem_u32(KT), aKH = smem_u32(KH), aVT = smem_u32(VT),
                   aST = smem_u32(ST);
    uint32_t phase = 0;
    bool ok = true;
    // windows whose copies were started / waited for (r, k, v; the decays)
    int64_t issued = 1, consumed = 0, issued_w = PERTOK ? 1 : 0, consumed_w = 0;

    const float wc = PERTOK ? 0.f : A.w[ch0 + ci];
    // per-channel decays: the factors of consecutive tokens differ by e^{-+w}
    const float dec1 = PERTOK ? 1.f : ex2(-wc * kLog2e), inc1 = PERTOK ? 1.f : ex2(wc * kLog2e);
    for (int64_t w0 = 0; w0 < T && ok; w0 += 64) {
        const int wn = static_cast<int>(T - w0 < 64 ? T - w0 : 64);
        const int64_t wi = w0 / 64;
        const uint32_t spar = static_cast<uint32_t>(wi & 1);
        {
            bool got = mbar_wait(&full[0], spar, kCopyWaitNs);
            if (PERTOK) got = mbar_wait(&full[1], spar, kCopyWaitNs) && got;
            ok = __syncthreads_and(got);
        }
        if (!ok) break;
        consumed = wi + 1;
        consumed_w = PERTOK ? wi + 1 : 0;
        const unsigned char* st = smem + SG::BASE;
        const __nv_bfloat16* sr = reinterpret_cast<const __nv_bfloat16*>(st);
        const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(st + SG::IO);
        const __nv_bfloat16* sv = reinterpret_cast<const __nv_bfloat16*>(st + 2 * SG::IO);
        const float* sw = reinterpret_cast<const float*>(ST);
        const float* gw = PERTOK ? A.w + (b * T + w0) * C + ch0 + ci : nullptr;
        // ---- block length for this window (the shortest any channel needs) ----
        auto rate_s = [&](int t) -> float { return PERTOK ? sw[t * 64 + ci] : wc; };
        int lm;
        // a full window with per-token decays: each of a channel's four
        // threads sums its quarter of the window once; blocks of 64 tokens
        // need only the sums of the two halves, and the block's cumulative
        // decays follow from the quarters
        bool quarters = false;
        float wq[4] = {0.f, 0.f, 0.f, 0.f};
        if (PERTOK && wn == 64) {
            float part = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) part += sw[(16 * qq + q) * 64 + ci];
            s_wq[PERTOK ? qq : 0][ci] = part;
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 4; ++q) wq[q] = s_wq[PERTOK ? q : 0][ci];
            quarters = wq[0] + wq[1] <= kTcSpan && wq[2] + wq[3] <= kTcSpan;
        }
        if (PERTOK) {
            lm = quarters ? 64 : tc_block_len(wn, rate_s);
        } else {
            // a constant rate: the longest half of a block (of bl tokens, the
            // last one possibly shorter) is ceil(bl / 2) tokens
            auto fits = [&](int L) { const int bl = wn < L ? wn : L; return ((bl + 1) / 2) * wc <= kTcSpan; };
            lm = fits(64) ? 64 : fits(16) ? 16 : fits(4) ? 4 : 1;
        }
        const int L = !__syncthreads_or(lm < 64) ? 64 : !__syncthreads_or(lm < 16) ? 16
                    : !__syncthreads_or(lm < 4)  ? 4  : 1;
        // In a block of more than one token no factor is clamped, so the
        // state-increment factor follows from the intra one:
        // e^{-(Lam_L - Lam_{t+1})} = e^{Lam_{t+1} - Lam_m} e^{-(Lam_L - Lam_m)}.
        // (The inter factor e^{-Lam_t} = e^{Lam_m - Lam_t} e^{-Lam_m} holds in
        // every block: in a block of one token both sides are 1.)
        const bool tame = L > 1;
        // the decays: from the state's tile while it still holds them (a
        // window of one block: its stage 1 reads them before it writes the
        // state), else from global memory
        const bool rate_smem = L == 64;
        auto rate = [&](int t) -> float {
            return PERTOK ? (rate_smem ? sw[t * 64 + ci] : __ldg(gw + static_cast<int64_t>(t) * C)) : wc;
        };

        for (int b0 = 0; b0 < wn && ok; b0 += L) {
            const int bl = wn - b0 < L ? wn - b0 : L;   // tokens of this block
            const int mid = bl / 2;                     // the reference token
            const int64_t t0 = w0 + b0;
            const bool last_block = b0 + L >= wn;
            // ---- stage 1: decays and the operand tiles ----
            // Lam at the middle and at the end of the block, and at this
            // thread's first row, for channel ci
            float lam_mid = 0.f, lam_end = 0.f, lam_row = 0.f;
            if (PERTOK && quarters && L == 64) {
                lam_mid = wq[0] + wq[1];
                lam_end = lam_mid + (wq[2] + wq[3]);
                for (int q = 0; q < 4; ++q)
                    if (q < qq) lam_row += wq[q];
            } else if (PERTOK) {
                for (int t = 0; t < bl; ++t) {
                    if (t == mid) lam_mid = lam_end;
                    if (t == 16 * qq) lam_row = lam_end;
                    lam_end += rate(b0 + t);
                }
                if (16 * qq >= bl) lam_row = lam_end;
            } else {
                lam_mid = static_cast<float>(mid) * wc;
                lam_end = static_cast<float>(bl) * wc;
                lam_row = static_cast<float>(min(16 * qq, bl)) * wc;
            }
            const float emid = ex2(-lam_mid * kLog2e), erest = ex2(-(lam_end - lam_mid) * kLog2e);
            if (qq == 0) {
                s_eend[ci] = ex2(-lam_end * kLog2e);
                s_emid[ci] = emid;
            }
            // per-token decays (one CTA per SM, registers to spare): lo(K^)
            // is kept from here to stage 3; per-channel decays form it again
            float klo[PERTOK ? 16 : 1];
            {
                float khq[4], vq[4];
                float lam = lam_row;
                // per-channel decays in a block of more than one token: the
                // factors of the thread's first token, then products
                float er = 1.f, ek = 1.f;
                if (!PERTOK && tame) {
                    const float t1 = static_cast<float>(16 * qq);
                    er = ex2((lam_mid - t1 * wc) * kLog2e);
                    ek = ex2(((t1 + 1.f) * wc - lam_mid) * kLog2e);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int t = 16 * qq + q;
                    float rt = 0.f, kt = 0.f, kh_full = 0.f, v = 0.f;
                    if (t < bl) {
                        const int e = (b0 + t) * 64 + ci;   // window row b0 + t, channel ci
                        const float r = __bfloat162float(sr[e]);
                        const float k = __bfloat162float(sk[e]);
                        v = __bfloat162float(sv[e]);
                        float fr, fk, fg;
                        if (!PERTOK && tame) {
                            fr = er;
                            fk = ek;
                            fg = ek * erest;
                            er *= dec1;
                            ek *= inc1;
                        } else {
                            float lt, lt1;
                            if (PERTOK) {
                                lt = lam;
                                lam += rate(b0 + t);
                                lt1 = lam;
                            } else {
                                lt = static_cast<float>(t) * wc;
                                lt1 = static_cast<float>(t + 1) * wc;
                            }
                            fr = ex2(fminf(lam_mid - lt, kTcSpan) * kLog2e);
                            fk = ex2(fminf(lt1 - lam_mid, kTcSpan) * kLog2e);
                            fg = tame ? fk * erest : ex2(-(lam_end - lt1) * kLog2e);
                        }
                        rt = r * fr;
                        kt = k * fk;
                        kh_full = k * fg;
                    }
                    // row t across 32 channels: one word per lane, no bank conflict
                    tc_st(RT, t, ci, rt);
                    tc_st(KT, t, ci, kt);
                    khq[q & 3] = __uint_as_float(__float_as_uint(kh_full) & 0xFFFFE000u);   // the bits tf32 keeps
                    if constexpr (PERTOK) klo[q] = kh_full - khq[q & 3];
                    vq[q & 3] = v;
                    if ((q & 3) == 3) {
                        // channel ci's row, four tokens: one slot per lane
                        tc_st4(KH, ci, t - 3, khq[0], khq[1], khq[2], khq[3]);
                        tc_st4(VT, ci, t - 3, vq[0], vq[1], vq[2], vq[3]);
                    }
                }
            }
            // S0'^T for the inter product: this thread's entries of S, times
            // e^{-Lam_m} of their row's channel
            __syncthreads();   // s_emid
            {
                const float em[2] = {s_emid[R0], s_emid[R0 + 8]};
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            tc_st(ST, c0 + 8 * g + cl + e, R0 + 8 * hh, S[4 * g + 2 * hh + e] * em[hh]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // ---- batch 1 ----
            if (tid == 0) {
                tc_gemm(tA, aRT, aKT, false);
                tc_gemm(tY, aRT, aST, false);
                tc_gemm(tS, aKH, aVT, false);
                tc_commit(&bar[0]);
            }
            ok = __syncthreads_and(mbar_wait(&bar[0], phase, kCopyWaitNs));
            tc_fence_after();
            // the products have read the state's tile: the next window's
            // decays go there now
            if (PERTOK && last_block && ok && w0 + 64 < T) {
                if (tid == 0) fetch_w(wi + 1);
                issued_w = wi + 2;
            }
            // ---- stage 3: masked scores, lo(K^)^T ----
            {
                // the bonus diagonal of rows R0 and R0 + 8 where this warp's
                // column half holds them: sum over the head's channels of
                // r u k, from the staged inputs of the token, split over the
                // four threads of a row (16 channels each, the quarters
                // rotated by row so that the 8 rows of a load do not share
                // banks) and summed by two shuffles
                float dg[2] = {0.f, 0.f};
                if ((warp & 3) / 2 == warp / 4) {
                    const int part = ((lane & 3) + (lane >> 2)) & 3;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = R0 + 8 * hh;
                        if (row < bl) {
                            const uint4* r8 = reinterpret_cast<const uint4*>(sr + (b0 + row) * 64 + 16 * part);
                            const uint4* k8 = reinterpret_cast<const uint4*>(sk + (b0 + row) * 64 + 16 * part);
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
                                const uint4 rv = r8[c], kv = k8[c];
                                const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int ch = 16 * part + 8 * c + 2 * e;
                                    const float r0 = __uint_as_float(rw[e] << 16), r1 = __uint_as_float(rw[e] & 0xffff0000u);
                                    const float k0 = __uint_as_float(kw[e] << 16), k1 = __uint_as_float(kw[e] & 0xffff0000u);
                                    dg[hh] = fmaf(r0 * s_u[ch], k0, dg[hh]);
                                    dg[hh] = fmaf(r1 * s_u[ch + 1], k1, dg[hh]);
                                }
                            }
                        }
                        dg[hh] += __shfl_xor_sync(0xffffffffu, dg[hh], 1);
                        dg[hh] += __shfl_xor_sync(0xffffffffu, dg[hh], 2);
                    }
                }
                float a[16];
                tc_ld16x32(lane_off + tA, a);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = R0 + 8 * hh;
                        float m[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int sc = c0 + 8 * g + cl + e;
                            m[e] = sc < row ? a[4 * g + 2 * hh + e] : (sc == row ? dg[hh] : 0.f);
                        }
                        tc_st2(KT, row, c0 + 8 * g + cl, m[0], m[1]);
                    }
                }
            }
            if constexpr (PERTOK) {
#pragma unroll
                for (int q = 0; q < 16; q += 4) tc_st4(RT, ci, 16 * qq + q, klo[q], klo[q + 1], klo[q + 2], klo[q + 3]);
            } else {
                // lo(K^) of this thread's channel and tokens, formed again
                // exactly as in stage 1, into R~'s tile (free after batch 1)
                float lo[16];
                float lam = lam_row;
                float ek = 1.f;
                if (!PERTOK && tame) ek = ex2(((static_cast<float>(16 * qq) + 1.f) * wc - lam_mid) * kLog2e);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int t = 16 * qq + q;
                    lo[q] = 0.f;
                    if (t < bl) {
                        const float k = __bfloat162float(sk[(b0 + t) * 64 + ci]);
                        float fg;
                        if (!PERTOK && tame) {
                            fg = ek * erest;
                            ek *= inc1;
                        } else {
                            float lt1;
                            if (PERTOK) {
                                lam += rate(b0 + t);
                                lt1 = lam;
                            } else {
                                lt1 = static_cast<float>(t + 1) * wc;
                            }
                            fg = tame ? ex2(fminf(lt1 - lam_mid, kTcSpan) * kLog2e) * erest
                                      : ex2(-(lam_end - lt1) * kLog2e);
                        }
                        const float kh_full = k * fg;
                        lo[q] = kh_full - __uint_as_float(__float_as_uint(kh_full) & 0xFFFFE000u);
                    }
                }
#pragma unroll
                for (int q = 0; q < 16; q += 4) tc_st4(RT, ci, 16 * qq + q, lo[q], lo[q + 1], lo[q + 2], lo[q + 3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // one stage: the window's inputs are read (stage 1 and the lines
            // above of its last block); the next window's copy starts now
            if (last_block && w0 + 64 < T) {
                if (tid == 0) fetch(wi + 1);
                issued = wi + 2;
            }
            // ---- batch 2 ----
            if (tid == 0 && ok) {
                tc_gemm(tY, aKT, aVT, true);
                tc_gemm(tS, aRT, aVT, true);
                tc_commit(&bar[1]);
            }
            ok = __syncthreads_and(ok && mbar_wait(&bar[1], phase, kCopyWaitNs));
            tc_fence_after();
            // ---- stage 5: outputs, state ----
            {
                float x[16];
                tc_ld16x32(lane_off + tY, x);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = R0 + 8 * hh;
                    if (row < bl) {
                        __nv_bfloat16* dst = yg + (b * T + t0 + row) * C + ch0 + c0 + cl;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const __nv_bfloat162 p = __floats2bfloat162_rn(ok ? x[4 * g + 2 * hh] : nan,
                                                                           ok ? x[4 * g + 2 * hh + 1] : nan);
                            *reinterpret_cast<__nv_bfloat162*>(dst + 8 * g) = p;
                        }
                    }
                }
                tc_ld16x32(lane_off + tS, x);
                const float dec[2] = {s_eend[R0], s_eend[R0 + 8]};
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = 4 * g + 2 * hh + e;
                            S[j] = ok ? fmaf(dec[hh], S[j], x[j]) : nan;
                        }
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            phase ^= 1u;
        }
    }
    // a wait that failed leaves copies started but not waited for: they
    // must land before this CTA's shared memory is released
    if (tid == 0) {
        for (int64_t w = consumed; w < issued; ++w) mbar_wait(&full[0], static_cast<uint32_t>(w & 1), kCopyWaitNs);
        for (int64_t w = consumed_w; w < issued_w; ++w) mbar_wait(&full[1], static_cast<uint32_t>(w & 1), kCopyWaitNs);
    }
    if (A.s_out != nullptr) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float* dst = A.s_out + (bh * 64 + R0 + 8 * hh) * 64 + c0 + cl;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                *reinterpret_cast<float2*>(dst + 8 * g) =
                    ok ? make_float2(S[4 * g + 2 * hh], S[4 * g + 2 * hh + 1]) : make_float2(nan, nan);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTcCols) : "memory");
    }
}

}  // namespace wkv
