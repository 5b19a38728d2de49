// wkv_api.cu -- the C ABI of libwkv.so (declared in include/wkv.h).
//
// Host side only: argument validation, kernel selection and launches.  Every
// step of the operator runs in the kernels of wkv_seq.cuh, wkv_chunk.cuh and
// wkv_step.cuh; there is no host fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/wkv.h"
#include "wkv_chunk.cuh"
#include "wkv_lane.cuh"
#include "wkv_part.cuh"
#include "wkv_cluster.cuh"
#include "wkv_stream.cuh"
#include "wkv_backward.cuh"
#include "wkv_seq.cuh"
#include "wkv_step.cuh"
#include "wkv_shift.cuh"
#include "wkv5.cuh"
#include "wkv5_tc.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";

constexpr int64_t kMaxElems = int64_t(1) << 62;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};

// Register-load look-back kernel: W compute warps per CTA, LS tokens per warp
// segment, TT = W * LS = 64 tokens per chunk.  The workspace is sized for the
// smallest unit any kernel publishes words for (64 tokens here and in the
// part kernel).
constexpr int kW = 8;
constexpr int kLS = 8;
constexpr int kMinTT = kW * kLS;
// Lane-resident kernel: compute warps, tokens per warp segment, ring depth
// and CTAs per SM of the forward, per I/O type.  bf16 tiles are half as
// large, so its CTAs carry more compute warps in the same shared memory,
// which is what hides the recurrence's latency.
template <typename IO>
struct LaneCfg {
    static constexpr int W = 4, LS = 16, S = 3, MINB = 2;
};
template <>
struct LaneCfg<float> {
    static constexpr int W = 4, LS = 16, S = 2, MINB = 2;
};
// tokens per chunk of the lane-resident forward
inline int lane_tt(int dtype) {
    return dtype == WKV_F32 ? LaneCfg<float>::W * LaneCfg<float>::LS
                            : LaneCfg<__nv_bfloat16>::W * LaneCfg<__nv_bfloat16>::LS;
}
// The checkpoint sweep of the backward: 64-token chunks, the chunks the
// reverse walk takes.
constexpr int kLaneW = 4;
constexpr int kLaneLS = 16;
// Part kernel: compute warps and tokens per warp segment (64-token parts),
// four CTAs per SM.  It runs when there are fewer 64-channel lane blocks
// than SMs; the lane-resident kernel from there on.
constexpr int kPartW = 4;
constexpr int kPartLS = 16;
constexpr int kPartMinBlocks = 4;
// look-back window (parts per round trip) and whether pass 1 keeps its
// exponentials in registers for pass 2
constexpr int kPartWin = 1;
constexpr bool kPartCache = true;
// Cluster kernel: 4 compute warps x 32-token segments (128-token parts), at
// most 8 parts (a portable cluster) per sequence, four CTAs per SM.  It runs
// instead of the part kernel when every sequence fits one cluster.
constexpr int kClusterW = 4;
constexpr int kClusterLS = 32;
constexpr int kClusterPT = kClusterW * kClusterLS;
constexpr int kClusterMax = 8;
constexpr int kClusterMinBlocks = 4;
// Stream kernel: 8 compute warps x LS-token segments (32 for bfloat16, 16 for
// float32: 32 registers of k either way), one CTA per part, at most 8 parts
// (a portable cluster) per call.
constexpr int kStreamW = 8;
constexpr int kStreamMax = 8;
// A longer call with few lane blocks runs as a chain of stream launches of
// this many parts each, the state handed on through the workspace.
constexpr int64_t kStreamLongParts = 4;
constexpr int64_t kStreamLongMinLB = 48;
template <typename IO>
constexpr int stream_ls() { return sizeof(IO) == 2 ? 32 : 16; }
constexpr int64_t stream_pt(int dtype) { return kStreamW * (dtype == WKV_BF16 ? 32 : 16); }
// Sequences at most this long take the sequential kernel.
constexpr int64_t kSeqMaxT = 16;
// Limit of every wait on another CTA's result: 1 s, or WKV_WAIT_LIMIT_NS (read
// once per process; used by the tests to make waits run out on purpose).
// Waits for a CTA's own TMA copies have a fixed limit (kCopyWaitNs).
uint64_t wait_limit_ns() {
    static const uint64_t v = []() -> uint64_t {
        const char* e = std::getenv("WKV_WAIT_LIMIT_NS");
        if (e != nullptr && *e != '\0') {
            char* end = nullptr;
            const unsigned long long x = std::strtoull(e, &end, 10);
            if (end != e) return x;
        }
        return 1000000000ull;
    }();
    return v;
}

int record_cuda(cudaError_t e) {
    if (e == cudaSuccess) return WKV_OK;
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return WKV_ERR_CUDA;
}

int check_launch() { return record_cuda(cudaPeekAtLastError()); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// [p, p+bytes) intersects [q, q+qbytes)?
bool overlaps(const void* p, size_t bytes, const void* q, size_t qbytes) {
    if (p == nullptr || q == nullptr || bytes == 0 || qbytes == 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qbytes && b < a + bytes;
}

bool mul_ok(int64_t a, int64_t b, int64_t c, int64_t* out) {
    if (a < 0 || b < 0 || c < 0) return false;
    __int128 p = static_cast<__int128>(a) * b * c;
    if (p >= kMaxElems) return false;
    *out = static_cast<int64_t>(p);
    return true;
}

size_t elem_bytes(int dtype) { return dtype == WKV_BF16 ? 2 : 4; }

struct ChunkGeom {
    int64_t nCB, nLB, nchunks, units;
    size_t aggw_off, incw_off, bytes;
};

ChunkGeom chunk_geom(int64_t B, int64_t T, int64_t C, int V, int TT) {
    ChunkGeom g{};
    const int64_t CB = 32 * V;
    g.nCB = (C + CB - 1) / CB;
    g.nLB = B * g.nCB;
    g.nchunks = (T + TT - 1) / TT;
    g.units = g.nLB * g.nchunks;
    if (g.nchunks <= 1) return g;  // no cross-CTA exchange, no workspace
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    // header, then one 16-byte word per channel per chunk for the chunk
    // summaries and for the inclusive states
    g.aggw_off = 256;
    g.incw_off = g.aggw_off + up(size_t(g.units) * CB * sizeof(wkv::Word));
    g.bytes = g.incw_off + up(size_t(g.units) * CB * sizeof(wkv::Word));
    return g;
}

bool use_sequential(int64_t T) { return T <= kSeqMaxT; }

// Chunk chains (WKV_FLAG_CHAIN_BEGIN / WKV_FLAG_CHAIN_NEXT): per workspace,
// the call that published last, so that the next call of the chain knows
// which position's word to wait for.  A call without a matching record
// starts a new chain.
struct ChainRec {
    const void* ws = nullptr;
    const float* state = nullptr;   // that call's state_out
    int64_t B = 0, C = 0;
    int dtype = -1;
    uint32_t next = 0;              // position tag of the words it published
};
constexpr int kChainSlots = 32;
std::mutex g_chain_mutex;
ChainRec g_chain[kChainSlots];
int g_chain_evict = 0;

// Positions of a chain's published words cycle through 1 .. 2^30 - 1 (a
// word's tag holds 30 bits of position; 0 marks a chain's first call).
constexpr uint32_t kChainPosMax = (1u << 30) - 1u;
uint32_t chain_advance(uint32_t p, int64_t n) {
    return static_cast<uint32_t>((static_cast<uint64_t>(p) + static_cast<uint64_t>(n) - 1u) % kChainPosMax) + 1u;
}

// Any call that uses a workspace outside a chain ends the workspace's chain.
void chain_forget(const void* ws) {
    if (ws == nullptr) return;
    std::lock_guard<std::mutex> lock(g_chain_mutex);
    for (ChainRec& r : g_chain)
        if (r.ws == ws) r = ChainRec{};
}

// Position whose words hold this call's entering state (0: none, the call
// reads state_in), and the record of this call, which publishes `count`
// positions (one per launch), for the next one.
uint32_t chain_enter(const void* ws, bool next, const float* state_in, const float* state_out, int64_t B, int64_t C,
                     int dtype, int64_t count) {
    std::lock_guard<std::mutex> lock(g_chain_mutex);
    ChainRec* rec = nullptr;
    for (ChainRec& r : g_chain)
        if (r.ws == ws) rec = &r;
    uint32_t in = 0;
    if (rec != nullptr && next && state_in != nullptr && rec->state == state_in && rec->B == B && rec->C == C &&
        rec->dtype == dtype)
        in = rec->next;
    if (rec == nullptr) {
        for (ChainRec& r : g_chain)
            if (r.ws == nullptr && rec == nullptr) rec = &r;
    }
    if (rec == nullptr) {
        // every slot in use: end the oldest-placed chain (its next call starts over)
        rec = &g_chain[g_chain_evict];
        g_chain_evict = (g_chain_evict + 1) % kChainSlots;
    }
    *rec = ChainRec{ws, state_out, B, C, dtype, chain_advance(in, count)};
    return in;
}

int forced_kernel();

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

// Vector width 2 needs an even C and every row base aligned to 2 elements.
int pick_vec(int64_t C, int dtype, const void* const* io, int nio, const float* const* f32, int nf) {
    if (C % 2 != 0) return 1;
    const size_t eb = elem_bytes(dtype);
    for (int i = 0; i < nio; ++i)
        if (io[i] && !aligned(io[i], 2 * eb)) return 1;
    for (int i = 0; i < nf; ++i)
        if (f32[i] && !aligned(f32[i], 8)) return 1;
    return 2;
}

template <typename IO, int V, bool GATE>
void launch_seq(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const void* k,
                const void* v, const void* r, const float* s_in, void* y, float* s_out,
                cudaStream_t st) {
    const int64_t groups = B * (C / V);
    const int threads = 256;
    const int64_t blocks = (groups + threads - 1) / threads;
    wkv::seq_forward_kernel<IO, V, GATE><<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        B, T, C, w, u, static_cast<const IO*>(k), static_cast<const IO*>(v),
        static_cast<const IO*>(r), s_in, static_cast<IO*>(y), s_out);
}

template <typename IO, int V, bool GATE>
void launch_chunk(const wkv::ChunkArgs& a, int64_t grid, cudaStream_t st) {
    wkv::chunk_forward_kernel<IO, V, GATE, kW, kLS><<<static_cast<unsigned>(grid), kW * 32, 0, st>>>(a);
}

// ---- TMA path ----------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 3-D map over a (B, T, C) array: box = CB channels x TT tokens x 1 sequence.
// Coordinates past T or C read as zeros.
// promo: the L2 sector promotion of the copies (256 bytes unless given).
bool encode_map(CUtensorMap* m, const void* ptr, int dtype, int64_t B, int64_t T, int64_t C, int CB, int TT,
                CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t eb = elem_bytes(dtype);
    const cuuint64_t dims[3] = {cuuint64_t(C), cuuint64_t(T), cuuint64_t(B)};
    const cuuint64_t strides[2] = {cuuint64_t(C) * eb, cuuint64_t(T) * cuuint64_t(C) * eb};
    const cuuint32_t box[3] = {cuuint32_t(CB), cuuint32_t(TT), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, dtype == WKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// TMA needs 16-byte aligned bases and row strides, and coordinates in int32.
bool tma_eligible(int V, int dtype, int64_t B, int64_t T, int64_t C, const void* k, const void* v, const void* r,
                  const float* w, const float* u, const float* s_in) {
    // w, u and the initial state travel as bulk copies of whole rows
    if (C % 4 != 0 || !aligned(w, 16) || !aligned(u, 16) || (s_in && !aligned(s_in, 16))) return false;
    if (V != 2) return false;
    const int64_t eb = static_cast<int64_t>(elem_bytes(dtype));
    if ((C * eb) % 16 != 0) return false;
    if (B >= (int64_t(1) << 31) || T >= (int64_t(1) << 31) || C >= (int64_t(1) << 31)) return false;
    if (!aligned(k, 16) || !aligned(v, 16) || (r && !aligned(r, 16))) return false;
    return encode_fn() != nullptr;
}

// The cluster kernel takes the call: TMA-eligible, vectorisable, and every
// sequence within one cluster of parts.
bool fits_cluster(int dtype, int64_t B, int64_t T, int64_t C, const void* k, const void* v, const void* r,
                  const float* w, const float* u, const float* s_in, const void* y, const float* s_out) {
    if (T <= kSeqMaxT || (T + kClusterPT - 1) / kClusterPT > kClusterMax) return false;
    if (C % 2 != 0 || !aligned(y, 2 * elem_bytes(dtype)) || (s_out && !aligned(s_out, 8))) return false;
    const int64_t nLB = B * ((C + 63) / 64);
    if (nLB * ((T + kClusterPT - 1) / kClusterPT) > 0x7fffffffLL) return false;
    return tma_eligible(2, dtype, B, T, C, k, v, r, w, u, s_in);
}

// Kernel choice: 0 = automatic; the environment variable WKV_FORWARD_KERNEL
// (seq | chunk | part | lane | cluster | stream) forces one, for ablation
// measurements: chunk = register-load look-back kernel, part = part kernel,
// lane = lane-resident kernel, each even where another would run; cluster /
// stream = cluster or stream kernel wherever every sequence fits one cluster.
int forced_kernel() {
    static int f = []() {
        const char* e = std::getenv("WKV_FORWARD_KERNEL");
        if (e == nullptr) return 0;
        if (std::strcmp(e, "seq") == 0) return 1;
        if (std::strcmp(e, "chunk") == 0) return 2;
        if (std::strcmp(e, "part") == 0) return 5;
        if (std::strcmp(e, "lane") == 0) return 6;
        if (std::strcmp(e, "cluster") == 0) return 7;
        if (std::strcmp(e, "stream") == 0) return 8;
        return 0;
    }();
    return f;
}

// Launch of a TMA kernel with programmatic stream serialization: its CTAs
// may be scheduled while the previous kernel of the stream drains; the
// kernel waits for that kernel (griddepcontrol.wait) before its first
// global memory access.
template <typename... P>
int launch_pdl(void (*kern)(P...), int64_t grid, int threads, uint32_t smem, cudaStream_t st,
               const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tr, const wkv::ChunkArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, kern, tk, tv, tr, a));
}

// Lane-resident kernel: each CTA owns whole lane blocks; grid = min(lane
// blocks, resident capacity).
template <typename IO, bool GATE, int W, int LS, int STAGES, int MINB, bool CKPT = false>
int launch_lane(wkv::ChunkArgs a, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t st) {
    using G = wkv::LaneGeometry<IO, 2, GATE, W, LS, STAGES>;
    auto kern = wkv::lane_forward_kernel<IO, 2, GATE, W, LS, STAGES, MINB, CKPT>;
    static int capacity[kMaxDevices] = {0};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (capacity[dev] == 0) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        int per_sm = 0;
        rc = record_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, G::THREADS, G::SMEM));
        if (rc != WKV_OK) return rc;
        // a configuration that fits no SM is an error, not one CTA per SM
        if (per_sm <= 0) return record_cuda(cudaErrorLaunchOutOfResources);
        capacity[dev] = per_sm * sm_count();
    }
    CUtensorMap tk, tv, tr;
    // CTAs that split lane blocks read neighbouring lane blocks' rows at
    // different times: L2 fetches of a row's width (128 bytes for bfloat16)
    // waste no DRAM bandwidth on bytes evicted before their CTA reads them
    const CUtensorMapL2promotion promo =
        G::ROW >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
    if (!encode_map(&tk, a.k, dtype, a.B, a.T, a.C, G::CB, G::TT, promo) ||
        !encode_map(&tv, a.v, dtype, a.B, a.T, a.C, G::CB, G::TT, promo))
        return WKV_ERR_CUDA;
    if (GATE) {
        if (!encode_map(&tr, a.r, dtype, a.B, a.T, a.C, G::CB, G::TT, promo)) return WKV_ERR_CUDA;
    } else {
        tr = tv;
    }
    const int64_t grid = a.nLB < capacity[dev] ? a.nLB : capacity[dev];
    // fewer CTAs than lane blocks: equal shares of the chunk order, with one
    // state handed between neighbouring CTAs through the workspace.  Without
    // an adequate workspace (the forward only) every CTA takes whole lane
    // blocks instead (no hand-off; shares differ by up to one lane block).
    const bool ws_adequate = workspace != nullptr && workspace_bytes >= 256 + size_t(a.nLB) * G::CB * sizeof(wkv::Word) &&
                             (CKPT || workspace_bytes >= wkv_forward_workspace_bytes(a.B, a.T, a.C, dtype));
    if (grid < a.nLB && a.nchunks > 1 && (CKPT || ws_adequate)) {
        if (!ws_adequate) return WKV_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
        a.hdr = reinterpret_cast<wkv::WsHeader*>(workspace);
        a.incw = reinterpret_cast<wkv::Word*>(static_cast<char*>(workspace) + 256);
    } else {
        a.hdr = nullptr;
        a.incw = nullptr;
    }
    a.aggw = nullptr;
    return launch_pdl(kern, grid, G::THREADS, G::SMEM, st, tk, tv, tr, a);
}

// Part kernel: lane blocks cut into parts along T, claimed in order from the
// workspace's ticket counter; grid = min(parts, resident capacity).
template <typename IO, bool GATE, int NB>
int launch_part(wkv::ChunkArgs a, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t st) {
    using G = wkv::PartGeometry<IO, 2, GATE, kPartW, kPartLS, NB>;
    auto kern = wkv::part_forward_kernel<IO, 2, GATE, kPartW, kPartLS, NB, kPartMinBlocks, kPartWin, kPartCache>;
    static int capacity[kMaxDevices] = {0};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (capacity[dev] == 0) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        int per_sm = 0;
        rc = record_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, G::THREADS, G::SMEM));
        if (rc != WKV_OK) return rc;
        // a configuration that fits no SM is an error, not one CTA per SM
        if (per_sm <= 0) return record_cuda(cudaErrorLaunchOutOfResources);
        capacity[dev] = per_sm * sm_count();
    }
    const ChunkGeom g = chunk_geom(a.B, a.T, a.C, 2, G::PT);
    a.nCB = g.nCB;
    a.nLB = g.nLB;
    a.nchunks = g.nchunks;
    a.units = g.units;
    if (g.nchunks > 1) {
        if (workspace == nullptr) return WKV_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
        if (workspace_bytes < g.bytes || workspace_bytes < wkv_forward_workspace_bytes(a.B, a.T, a.C, dtype))
            return WKV_ERR_WORKSPACE;
        char* ws = static_cast<char*>(workspace);
        a.hdr = reinterpret_cast<wkv::WsHeader*>(ws);
        a.aggw = reinterpret_cast<wkv::Word*>(ws + g.aggw_off);
        a.incw = reinterpret_cast<wkv::Word*>(ws + g.incw_off);
    } else {
        a.hdr = nullptr;
        a.aggw = nullptr;
        a.incw = nullptr;
    }
    CUtensorMap tk, tv, tr;
    if (!encode_map(&tk, a.k, dtype, a.B, a.T, a.C, G::CB, G::PT) ||
        !encode_map(&tv, a.v, dtype, a.B, a.T, a.C, G::CB, G::PT))
        return WKV_ERR_CUDA;
    if (GATE) {
        if (!encode_map(&tr, a.r, dtype, a.B, a.T, a.C, G::CB, G::PT)) return WKV_ERR_CUDA;
    } else {
        tr = tv;
    }
    const int64_t grid = a.units < capacity[dev] ? a.units : capacity[dev];
    return launch_pdl(kern, grid, G::THREADS, G::SMEM, st, tk, tv, tr, a);
}

// Cluster kernel: one cluster of ceil(T / PT) CTAs per lane block, one CTA
// per part; needs no workspace (a workspace given only receives a failed
// copy's error flag).
template <typename IO, bool GATE>
int launch_cluster(wkv::ChunkArgs a, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t st) {
    using G = wkv::PartGeometry<IO, 2, GATE, kClusterW, kClusterLS, 1>;
    auto kern = wkv::cluster_forward_kernel<IO, 2, GATE, kClusterW, kClusterLS, kClusterMinBlocks>;
    static bool ready[kMaxDevices] = {false};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (!ready[dev]) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        ready[dev] = true;
    }
    const ChunkGeom g = chunk_geom(a.B, a.T, a.C, 2, G::PT);
    if (g.nchunks < 1 || g.nchunks > kClusterMax || g.units > 0x7fffffffLL) return WKV_ERR_SHAPE;
    a.nCB = g.nCB;
    a.nLB = g.nLB;
    a.nchunks = g.nchunks;
    a.units = g.units;
    a.hdr = workspace != nullptr && aligned(workspace, 256) && workspace_bytes >= sizeof(wkv::WsHeader)
                ? reinterpret_cast<wkv::WsHeader*>(workspace)
                : nullptr;
    a.aggw = nullptr;
    a.incw = nullptr;
    CUtensorMap tk, tv, tr;
    if (!encode_map(&tk, a.k, dtype, a.B, a.T, a.C, G::CB, G::PT) ||
        !encode_map(&tv, a.v, dtype, a.B, a.T, a.C, G::CB, G::PT))
        return WKV_ERR_CUDA;
    if (GATE) {
        if (!encode_map(&tr, a.r, dtype, a.B, a.T, a.C, G::CB, G::PT)) return WKV_ERR_CUDA;
    } else {
        tr = tv;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(g.units));
    cfg.blockDim = dim3(G::THREADS);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(g.nchunks);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return record_cuda(cudaLaunchKernelEx(&cfg, kern, tk, tv, tr, a));
}

template <typename IO>
int dispatch_cluster(bool gate, const wkv::ChunkArgs& a, int dtype, void* ws, size_t ws_bytes, cudaStream_t st) {
    return gate ? launch_cluster<IO, true>(a, dtype, ws, ws_bytes, st)
                : launch_cluster<IO, false>(a, dtype, ws, ws_bytes, st);
}

// Stream kernel: one cluster of ceil(T / PT) CTAs per lane block.  With
// tc > 0 the call runs as a chain of launches of tc tokens each (the last
// one shorter), the state handed from launch to launch through a.chain's
// words: launch i waits for position a.chain_in advanced i times.
template <typename IO, bool GATE>
int launch_stream(wkv::ChunkArgs a, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t st,
                  int64_t tc = 0) {
    constexpr int LS = stream_ls<IO>();
    using G = wkv::StreamGeometry<IO, GATE, kStreamW, LS>;
    auto kern = wkv::stream_forward_kernel<IO, GATE, kStreamW, LS, 3>;
    static bool ready[kMaxDevices] = {false};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (!ready[dev]) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        ready[dev] = true;
    }
    const int64_t T = a.T;
    const int64_t per = tc > 0 ? tc : T;
    if (per < 1 || (per + G::PT - 1) / G::PT > kStreamMax || (tc > 0 && a.chain == nullptr)) return WKV_ERR_SHAPE;
    {
        const ChunkGeom g = chunk_geom(a.B, per, a.C, 2, G::PT);
        if (g.units > 0x7fffffffLL) return WKV_ERR_SHAPE;
    }
    a.hdr = workspace != nullptr && aligned(workspace, 256) && workspace_bytes >= sizeof(wkv::WsHeader)
                ? reinterpret_cast<wkv::WsHeader*>(workspace)
                : nullptr;
    a.aggw = nullptr;
    a.incw = nullptr;
    // tensor maps over the whole arrays; each launch addresses its rows by t0
    CUtensorMap tk, tv, tr, ty;
    if (!encode_map(&tk, a.k, dtype, a.B, T, a.C, G::CB, G::PT)) return WKV_ERR_CUDA;
    if (!encode_map(&tv, a.v, dtype, a.B, T, a.C, G::CB, G::PT)) return WKV_ERR_CUDA;
    if (GATE) {
        if (!encode_map(&tr, a.r, dtype, a.B, T, a.C, G::CB, G::PT)) return WKV_ERR_CUDA;
    } else {
        tr = tv;
    }
    // outputs: one box of a warp's LS rows (no y when only the state is wanted)
    if (a.y != nullptr) {
        if (!encode_map(&ty, a.y, dtype, a.B, T, a.C, G::CB, LS)) return WKV_ERR_CUDA;
    } else {
        ty = tv;
    }
    const int64_t n = (T + per - 1) / per;
    uint32_t pos = a.chain_in;
    for (int64_t i = 0; i < n; ++i) {
        wkv::ChunkArgs b = a;
        b.t0 = i * per;
        b.T = T - b.t0 < per ? T - b.t0 : per;
        const ChunkGeom g = chunk_geom(b.B, b.T, b.C, 2, G::PT);
        b.nCB = g.nCB;
        b.nLB = g.nLB;
        b.nchunks = g.nchunks;
        b.units = g.units;
        b.chain_in = pos;
        b.chain_out = chain_advance(pos, 1);
        pos = b.chain_out;
        if (i > 0) {
            b.s_in = nullptr;   // the entering state comes from the previous launch's words
            b.early = 1u;       // this call's inputs are not written by its own launches
        }
        if (i + 1 < n) b.s_out = nullptr;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(g.units));
        cfg.blockDim = dim3(G::THREADS);
        cfg.dynamicSmemBytes = G::SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(g.nchunks);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        rc = record_cuda(cudaLaunchKernelEx(&cfg, kern, tk, tv, tr, ty, b));
        if (rc != WKV_OK) return rc;
    }
    return WKV_OK;
}

template <typename IO>
int dispatch_stream(bool gate, const wkv::ChunkArgs& a, int dtype, void* ws, size_t ws_bytes, cudaStream_t st,
                    int64_t tc = 0) {
    return gate ? launch_stream<IO, true>(a, dtype, ws, ws_bytes, st, tc)
                : launch_stream<IO, false>(a, dtype, ws, ws_bytes, st, tc);
}

// Part buffers per CTA: as many as fit beside kPartMinBlocks CTAs per SM
// (up to three), at least one.
template <typename IO, bool GATE>
constexpr int part_buffers() {
    constexpr int budget = 225 * 1024 / kPartMinBlocks - 8 * 1024;   // static shared memory and slack
    constexpr int part = wkv::PartGeometry<IO, 2, GATE, kPartW, kPartLS, 1>::PART;
    return budget / part < 1 ? 1 : (budget / part > 3 ? 3 : budget / part);
}

template <typename IO>
int dispatch_part(bool gate, const wkv::ChunkArgs& a, int dtype, void* ws, size_t ws_bytes, cudaStream_t st) {
    return gate ? launch_part<IO, true, part_buffers<IO, true>()>(a, dtype, ws, ws_bytes, st)
                : launch_part<IO, false, part_buffers<IO, false>()>(a, dtype, ws, ws_bytes, st);
}

template <typename IO>
int dispatch_lane(bool gate, const wkv::ChunkArgs& a, int dtype, void* ws, size_t ws_bytes, cudaStream_t st) {
    using L = LaneCfg<IO>;
    return gate ? launch_lane<IO, true, L::W, L::LS, L::S, L::MINB>(a, dtype, ws, ws_bytes, st)
                : launch_lane<IO, false, L::W, L::LS, L::S, L::MINB>(a, dtype, ws, ws_bytes, st);
}

template <typename IO, int V>
void dispatch_forward(bool gate, bool seq, const wkv::ChunkArgs& a, int64_t grid, cudaStream_t st) {
    if (seq) {
        if (gate)
            launch_seq<IO, V, true>(a.B, a.T, a.C, a.w, a.u, a.k, a.v, a.r, a.s_in, a.y, a.s_out, st);
        else
            launch_seq<IO, V, false>(a.B, a.T, a.C, a.w, a.u, a.k, a.v, a.r, a.s_in, a.y, a.s_out, st);
    } else {
        if (gate)
            launch_chunk<IO, V, true>(a, grid, st);
        else
            launch_chunk<IO, V, false>(a, grid, st);
    }
}

template <typename IO, int V, bool GATE>
int launch_step(int64_t L, int64_t B, int64_t C, const float* w, const float* u, const void* k,
                 const void* v, const void* r, float* state, void* y, cudaStream_t st) {
    const int64_t total = L * B * (C / V);
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(threads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, wkv::step_kernel<IO, V, GATE>, L, B, C, w, u,
                                          static_cast<const IO*>(k), static_cast<const IO*>(v),
                                          static_cast<const IO*>(r), state, static_cast<IO*>(y)));
}

// Token shift: one thread per (sequence, kShiftTS tokens, V channels).
constexpr int kShiftTS = 8;

template <typename IO, int V>
int launch_shift(int64_t B, int64_t T, int64_t C, int nmix, const void* x, const float* mu, const void* x_prev,
                 void* out, void* x_last, cudaStream_t st) {
    const int64_t units = B * ((T + kShiftTS - 1) / kShiftTS) * (C / V);
    const int threads = 256;
    const int64_t blocks = (units + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return WKV_ERR_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(threads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, wkv::token_shift_kernel<IO, V, kShiftTS>, B, T, C, nmix,
                                          static_cast<const IO*>(x), mu, static_cast<const IO*>(x_prev),
                                          static_cast<IO*>(out), static_cast<IO*>(x_last)));
}

// Host-side checks of a forward call with T >= 1 and B, C >= 1: required
// pointers, alignment to the element types, and overlaps (y must be disjoint
// from every input and from state_out; state_out may equal state_in but
// overlap nothing else).
int forward_args(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u, const void* k,
                 const void* v, const void* r, const float* state_in, const void* y, const float* state_out) {
    const size_t eb = elem_bytes(dtype);
    const size_t io_bytes = size_t(B) * size_t(T) * size_t(C) * eb, st_bytes = size_t(B) * size_t(C) * 3 * 4,
                 p_bytes = size_t(C) * 4;
    if (!w || !u || !k || !v || !y) return WKV_ERR_NULLPTR;
    if (!aligned(w, 4) || !aligned(u, 4) || !aligned(k, eb) || !aligned(v, eb) || !aligned(y, eb) ||
        (r && !aligned(r, eb)) || (state_in && !aligned(state_in, 4)) || (state_out && !aligned(state_out, 4)))
        return WKV_ERR_ALIGN;
    const void* ins[] = {k, v, r};
    for (const void* p : ins)
        if (overlaps(y, io_bytes, p, io_bytes)) return WKV_ERR_ALIAS;
    if (overlaps(y, io_bytes, w, p_bytes) || overlaps(y, io_bytes, u, p_bytes) ||
        overlaps(y, io_bytes, state_in, st_bytes) || overlaps(y, io_bytes, state_out, st_bytes))
        return WKV_ERR_ALIAS;
    if (state_out) {
        for (const void* p : ins)
            if (overlaps(state_out, st_bytes, p, io_bytes)) return WKV_ERR_ALIAS;
        if (overlaps(state_out, st_bytes, w, p_bytes) || overlaps(state_out, st_bytes, u, p_bytes))
            return WKV_ERR_ALIAS;
        if (state_in && state_in != state_out && overlaps(state_out, st_bytes, state_in, st_bytes))
            return WKV_ERR_ALIAS;
    }
    return WKV_OK;
}

int run_forward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u, const void* k,
                const void* v, const void* r, const float* state_in, void* y, float* state_out, void* workspace,
                size_t workspace_bytes, unsigned flags, cudaStream_t stream);

}  // namespace

extern "C" {

int wkv_abi_version(void) { return 1; }

const char* wkv_strerror(int status) {
    switch (status) {
        case WKV_OK: return "success";
        case WKV_ERR_NULLPTR: return "a required pointer is NULL";
        case WKV_ERR_SHAPE: return "invalid size (negative, or element count beyond 2^62)";
        case WKV_ERR_DTYPE: return "unknown dtype (expected WKV_F32 or WKV_BF16)";
        case WKV_ERR_ALIGN: return "pointer not aligned to its element type (workspace: 256 bytes)";
        case WKV_ERR_ALIAS: return "an output buffer overlaps an input or another output";
        case WKV_ERR_CUDA: return "CUDA error (see wkv_last_cuda_error)";
        case WKV_ERR_TIMEOUT: return "a cross-block wait on the GPU gave up; affected outputs are NaN";
        case WKV_ERR_WORKSPACE: return "workspace missing or smaller than wkv_forward_workspace_bytes()";
        case WKV_ERR_SCRATCH: return "problem needs more scratch than wkv_forward_noalloc's built-in array";
        default: return "unknown wkv status";
    }
}

const char* wkv_last_cuda_error(void) { return g_last_cuda_error; }

size_t wkv_forward_workspace_bytes(int64_t B, int64_t T, int64_t C, int dtype) {
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n) || (dtype != WKV_F32 && dtype != WKV_BF16)) return 0;
    if (n == 0 || use_sequential(T)) return 0;
    // the larger of the two vector widths' layouts, so the size does not
    // depend on pointer alignment
    const size_t a = chunk_geom(B, T, C, 1, kMinTT).bytes, b = chunk_geom(B, T, C, 2, kMinTT).bytes;
    return a > b ? a : b;
}

int wkv_workspace_init(void* workspace, size_t bytes, cudaStream_t stream) {
    chain_forget(workspace);
    if (bytes == 0) return WKV_OK;
    if (workspace == nullptr) return WKV_ERR_NULLPTR;
    if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
    return record_cuda(cudaMemsetAsync(workspace, 0, bytes, stream));
}

int wkv_workspace_status(const void* workspace, cudaStream_t stream) {
    if (workspace == nullptr) return WKV_ERR_NULLPTR;
    if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
    int rc = record_cuda(cudaStreamSynchronize(stream));
    if (rc != WKV_OK) return rc;
    wkv::WsHeader h{};
    rc = record_cuda(cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost));
    if (rc != WKV_OK) return rc;
    return (h.error & wkv::kErrTimeout) ? WKV_ERR_TIMEOUT : WKV_OK;
}

int wkv_forward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                const void* k, const void* v, const void* r, const float* state_in, void* y,
                float* state_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return wkv_forward_ex(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out, workspace, workspace_bytes, 0u,
                          stream);
}

int wkv_forward_ex(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                   const void* k, const void* v, const void* r, const float* state_in, void* y,
                   float* state_out, void* workspace, size_t workspace_bytes, unsigned flags,
                   cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    if ((flags & ~unsigned(WKV_FLAG_INPUTS_READY | WKV_FLAG_CHAIN_BEGIN | WKV_FLAG_CHAIN_NEXT)) != 0 ||
        (flags & WKV_FLAG_CHAIN_BEGIN && flags & WKV_FLAG_CHAIN_NEXT))
        return WKV_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n)) return WKV_ERR_SHAPE;
    if (B == 0 || C == 0) return WKV_OK;
    const int64_t lanes = B * C;
    const size_t st_bytes = size_t(lanes) * 3 * 4;
    if (T == 0) {
        if (state_out == nullptr) return WKV_OK;
        if (!aligned(state_out, 4) || (state_in && !aligned(state_in, 4))) return WKV_ERR_ALIGN;
        if (state_in && state_in != state_out && overlaps(state_in, st_bytes, state_out, st_bytes))
            return WKV_ERR_ALIAS;
        if (state_in == state_out) return WKV_OK;
        wkv::copy_state_kernel<<<static_cast<unsigned>((lanes + 255) / 256), 256, 0, stream>>>(
            lanes, state_in, state_out);
        return check_launch();
    }
    const int vrc = forward_args(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out);
    if (vrc != WKV_OK) return vrc;
    return run_forward(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out, workspace, workspace_bytes, flags,
                       stream);
}

}  // extern "C"

namespace {

// Kernel choice and launch of a forward call whose arguments passed the host
// checks (B, C, T >= 1).  y == nullptr: only the state is wanted.
int run_forward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u, const void* k,
                const void* v, const void* r, const float* state_in, void* y, float* state_out, void* workspace,
                size_t workspace_bytes, unsigned flags, cudaStream_t stream) {
    const void* io[] = {k, v, r, y};
    const float* f32[] = {w, u, state_in, state_out};
    const int V = pick_vec(C, dtype, io, 4, f32, 4);
    const int force = forced_kernel();
    const bool seq = force == 1 || (force == 0 && use_sequential(T));
    if (seq) chain_forget(workspace);

    wkv::ChunkArgs a{};
    a.w = w;
    a.u = u;
    a.k = k;
    a.v = v;
    a.r = r;
    a.s_in = state_in;
    a.y = y;
    a.s_out = state_out;
    a.B = B;
    a.T = T;
    a.C = C;
    a.wait_limit_ns = wait_limit_ns();
    a.early = (flags & (WKV_FLAG_INPUTS_READY | WKV_FLAG_CHAIN_BEGIN | WKV_FLAG_CHAIN_NEXT)) ? 1u : 0u;
    a.chain = nullptr;
    a.chain_in = 0u;
    int64_t grid = 0;
    if (!seq) {
        const bool tma = force != 2 && tma_eligible(V, dtype, B, T, C, k, v, r, w, u, state_in);
        // at least one lane block per SM: CTAs walk whole sequences; fewer:
        // the part kernel cuts them along T.  The ticket counter is 32 bits.
        const int64_t nLB = B * ((C + 63) / 64);
        const int64_t nparts = nLB * ((T + kPartW * kPartLS - 1) / (kPartW * kPartLS));
        const bool part_ok = tma && nparts < (int64_t(1) << 31);
        // Every sequence within one cluster of parts: the cluster kernel needs
        // no workspace, so it serves calls that bring none (wkv_forward_noalloc
        // among them).  With a workspace the part kernel runs instead, which
        // measured a little faster on the streaming chunk.
        const bool cluster_ok = part_ok && (T + kClusterPT - 1) / kClusterPT <= kClusterMax;
        const bool ws_ok = workspace != nullptr && workspace_bytes >= wkv_forward_workspace_bytes(B, T, C, dtype);
        // Few lane blocks and a call that fits one cluster of stream-kernel
        // parts (a chunk of a carried stream): the stream kernel, which needs
        // no workspace and, with WKV_FLAG_INPUTS_READY, does everything but
        // the entering state's fold and the outputs before the previous
        // kernel of the stream ends.
        const int64_t spt = stream_pt(dtype);
        const size_t eb = elem_bytes(dtype);
        const size_t chain_bytes = size_t(B) * size_t(C) * sizeof(wkv::Word);
        const bool chain_ws = workspace != nullptr && aligned(workspace, 256) && workspace_bytes >= 256 + chain_bytes;
        const bool stream_io = part_ok && (y == nullptr || aligned(y, 16)) && (state_out == nullptr || aligned(state_out, 8));
        const bool stream_ok = stream_io && (T + spt - 1) / spt <= kStreamMax;
        // A longer call with room for the chain's words: a chain of stream
        // launches of kStreamLongParts parts each.  It beats the part
        // kernel's look-back when a launch fills the GPU and its tiles are
        // small: ungated bfloat16 with at least kStreamLongMinLB lane blocks
        // (measured: 1959 against 2144 us at B=1, T=262144, C=4096; but 369
        // against 159 us with 8 lane blocks, and slower for gated or float32
        // calls, whose tiles leave fewer CTAs per SM).
        const bool stream_long = stream_io && !stream_ok && chain_ws &&
                                 (force == 8 || (dtype == WKV_BF16 && r == nullptr && nLB >= kStreamLongMinLB));
        if ((stream_ok || stream_long) && (force == 8 || (force == 0 && nLB < sm_count()))) {
            const int64_t tc = stream_long ? kStreamLongParts * spt : 0;
            const int64_t launches = stream_long ? (T + tc - 1) / tc : 1;
            // a chain publishes each launch's end state at the start of the
            // workspace, right after its header
            const bool chain_call = (flags & (WKV_FLAG_CHAIN_BEGIN | WKV_FLAG_CHAIN_NEXT)) != 0;
            if ((chain_call && chain_ws) || stream_long) {
                a.chain = reinterpret_cast<wkv::Word*>(static_cast<char*>(workspace) + 256);
                if (chain_call) {
                    a.chain_in = chain_enter(workspace, (flags & WKV_FLAG_CHAIN_NEXT) != 0, state_in, state_out, B,
                                             C, dtype, launches);
                } else {
                    chain_forget(workspace);
                    a.chain_in = 0u;
                }
                if (a.chain_in == 0u) {
                    // a new chain: no word of an earlier one may look current
                    const int rc = record_cuda(cudaMemsetAsync(a.chain, 0, chain_bytes, stream));
                    if (rc != WKV_OK) {
                        chain_forget(workspace);
                        return rc;
                    }
                }
            } else {
                chain_forget(workspace);
            }
            const int rc = dtype == WKV_F32
                               ? dispatch_stream<float>(r != nullptr, a, dtype, workspace, workspace_bytes, stream, tc)
                               : dispatch_stream<__nv_bfloat16>(r != nullptr, a, dtype, workspace, workspace_bytes,
                                                                stream, tc);
            if (rc != WKV_OK) chain_forget(workspace);
            return rc;
        }
        chain_forget(workspace);
        if (cluster_ok && (force == 7 || (force == 0 && !ws_ok))) {
            return dtype == WKV_F32
                       ? dispatch_cluster<float>(r != nullptr, a, dtype, workspace, workspace_bytes, stream)
                       : dispatch_cluster<__nv_bfloat16>(r != nullptr, a, dtype, workspace, workspace_bytes, stream);
        }
        // No adequate workspace and no cluster fits: schedules that need no
        // scratch.  TMA-eligible calls take the lane-resident kernel over
        // whole lane blocks; any other layout walks the plain recurrence per
        // lane (the sequential kernel takes any T and any alignment).
        if (force == 0 && !ws_ok) {
            if (!tma) {
                if (B * (C / V) > int64_t(0x7fffffff) * 256) return WKV_ERR_SHAPE;
                if (dtype == WKV_F32) {
                    if (V == 2) dispatch_forward<float, 2>(r != nullptr, true, a, 0, stream);
                    else dispatch_forward<float, 1>(r != nullptr, true, a, 0, stream);
                } else {
                    if (V == 2) dispatch_forward<__nv_bfloat16, 2>(r != nullptr, true, a, 0, stream);
                    else dispatch_forward<__nv_bfloat16, 1>(r != nullptr, true, a, 0, stream);
                }
                return check_launch();
            }
            const ChunkGeom g = chunk_geom(B, T, C, 2, lane_tt(dtype));
            a.nCB = g.nCB;
            a.nLB = g.nLB;
            a.nchunks = g.nchunks;
            a.units = g.units;
            return dtype == WKV_F32 ? dispatch_lane<float>(r != nullptr, a, dtype, nullptr, 0, stream)
                                    : dispatch_lane<__nv_bfloat16>(r != nullptr, a, dtype, nullptr, 0, stream);
        }
        const bool part = part_ok && (force == 5 || (force == 0 && nLB < sm_count()));
        if (part) {
            a.nLB = nLB;
            return dtype == WKV_F32
                       ? dispatch_part<float>(r != nullptr, a, dtype, workspace, workspace_bytes, stream)
                       : dispatch_part<__nv_bfloat16>(r != nullptr, a, dtype, workspace, workspace_bytes, stream);
        }
        if (tma) {
            const ChunkGeom g = chunk_geom(B, T, C, 2, lane_tt(dtype));
            a.nCB = g.nCB;
            a.nLB = g.nLB;
            a.nchunks = g.nchunks;
            a.units = g.units;
            return dtype == WKV_F32
                       ? dispatch_lane<float>(r != nullptr, a, dtype, workspace, workspace_bytes, stream)
                       : dispatch_lane<__nv_bfloat16>(r != nullptr, a, dtype, workspace, workspace_bytes, stream);
        }
        const ChunkGeom g = chunk_geom(B, T, C, V, kW * kLS);
        a.nCB = g.nCB;
        a.nLB = g.nLB;
        a.nchunks = g.nchunks;
        a.units = g.units;
        grid = g.units;
        if (grid > 0x7fffffffLL) return WKV_ERR_SHAPE;
        if (g.bytes > 0) {
            if (workspace == nullptr) return WKV_ERR_WORKSPACE;
            if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
            if (workspace_bytes < wkv_forward_workspace_bytes(B, T, C, dtype)) return WKV_ERR_WORKSPACE;
            char* ws = static_cast<char*>(workspace);
            a.hdr = reinterpret_cast<wkv::WsHeader*>(ws);
            a.aggw = reinterpret_cast<wkv::Word*>(ws + g.aggw_off);
            a.incw = reinterpret_cast<wkv::Word*>(ws + g.incw_off);
        }
    }
    if (seq && B * (C / V) > int64_t(0x7fffffff) * 256) return WKV_ERR_SHAPE;
    if (dtype == WKV_F32) {
        if (V == 2) dispatch_forward<float, 2>(r != nullptr, seq, a, grid, stream);
        else dispatch_forward<float, 1>(r != nullptr, seq, a, grid, stream);
    } else {
        if (V == 2) dispatch_forward<__nv_bfloat16, 2>(r != nullptr, seq, a, grid, stream);
        else dispatch_forward<__nv_bfloat16, 1>(r != nullptr, seq, a, grid, stream);
    }
    return check_launch();
}

}  // namespace

extern "C" {

int wkv_state(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const void* k, const void* v,
              const float* state_in, float* state_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n)) return WKV_ERR_SHAPE;
    if (B == 0 || C == 0) return WKV_OK;
    if (state_out == nullptr) return WKV_ERR_NULLPTR;
    if (T == 0)   // the state passes through (the same as wkv_forward with T = 0)
        return wkv_forward(B, 0, C, dtype, nullptr, nullptr, nullptr, nullptr, nullptr, state_in, nullptr,
                           state_out, nullptr, 0, stream);
    if (!w || !k || !v) return WKV_ERR_NULLPTR;
    const size_t eb = elem_bytes(dtype);
    const size_t io_bytes = size_t(n) * eb, st_bytes = size_t(B) * size_t(C) * 3 * 4, p_bytes = size_t(C) * 4;
    if (!aligned(w, 4) || !aligned(k, eb) || !aligned(v, eb) || (state_in && !aligned(state_in, 4)) ||
        !aligned(state_out, 4))
        return WKV_ERR_ALIGN;
    if (overlaps(state_out, st_bytes, k, io_bytes) || overlaps(state_out, st_bytes, v, io_bytes) ||
        overlaps(state_out, st_bytes, w, p_bytes) ||
        (state_in && state_in != state_out && overlaps(state_out, st_bytes, state_in, st_bytes)))
        return WKV_ERR_ALIAS;
    // the state does not depend on u or on the gate: w stands in for u (any
    // finite row would do; it only steers the choice between two evaluations
    // of the same summary), no gate, no output
    return run_forward(B, T, C, dtype, w, w, k, v, nullptr, state_in, nullptr, state_out, workspace,
                       workspace_bytes, 0u, stream);
}

int wkv_state_combine(int64_t B, int64_t C, int n, const float* w, const int64_t* lens, const float* states,
                      const float* state_in, float* state_out, cudaStream_t stream) {
    int64_t lanes = 0;
    if (!mul_ok(B, C, 1, &lanes) || n < 0 || n > wkv::kCombineMax) return WKV_ERR_SHAPE;
    if (lanes == 0) return WKV_OK;
    if (state_out == nullptr || (n > 0 && (w == nullptr || lens == nullptr || states == nullptr)))
        return WKV_ERR_NULLPTR;
    wkv::CombineLens L{};
    for (int j = 0; j < n; ++j) {
        if (lens[j] < 0) return WKV_ERR_SHAPE;
        L.len[j] = lens[j];
    }
    if (!aligned(state_out, 4) || (w && !aligned(w, 4)) || (states && !aligned(states, 4)) ||
        (state_in && !aligned(state_in, 4)))
        return WKV_ERR_ALIGN;
    const size_t st_bytes = size_t(lanes) * 3 * 4;
    if (overlaps(state_out, st_bytes, states, st_bytes * size_t(n)) || overlaps(state_out, st_bytes, w, size_t(C) * 4) ||
        (state_in && state_in != state_out && overlaps(state_out, st_bytes, state_in, st_bytes)))
        return WKV_ERR_ALIAS;
    if ((lanes + 255) / 256 > 0x7fffffffLL) return WKV_ERR_SHAPE;
    if (n == 0)
        return wkv_forward(B, 0, C, WKV_F32, nullptr, nullptr, nullptr, nullptr, nullptr, state_in, nullptr,
                           state_out, nullptr, 0, stream);
    wkv::state_combine_kernel<<<static_cast<unsigned>((lanes + 255) / 256), 256, 0, stream>>>(
        B, C, n, w, L, states, state_in, state_out);
    return check_launch();
}

int wkv_step(int64_t L, int64_t B, int64_t C, int dtype, const float* w, const float* u,
             const void* k, const void* v, const void* r, float* state, void* y, cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(L, B, C, &n)) return WKV_ERR_SHAPE;
    if (n == 0) return WKV_OK;
    if (!w || !u || !k || !v || !state || !y) return WKV_ERR_NULLPTR;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(w, 4) || !aligned(u, 4) || !aligned(state, 4) || !aligned(k, eb) || !aligned(v, eb) ||
        !aligned(y, eb) || (r && !aligned(r, eb)))
        return WKV_ERR_ALIGN;
    const size_t io_bytes = size_t(n) * eb, st_bytes = size_t(n) * 3 * 4, p_bytes = size_t(L) * C * 4;
    const void* ins[] = {k, v, r};
    for (const void* p : ins)
        if (overlaps(y, io_bytes, p, io_bytes) || overlaps(state, st_bytes, p, io_bytes)) return WKV_ERR_ALIAS;
    if (overlaps(y, io_bytes, state, st_bytes) || overlaps(y, io_bytes, w, p_bytes) ||
        overlaps(y, io_bytes, u, p_bytes) || overlaps(state, st_bytes, w, p_bytes) ||
        overlaps(state, st_bytes, u, p_bytes))
        return WKV_ERR_ALIAS;
    const void* io[] = {k, v, r, y};
    const float* f32[] = {w, u, state};
    const int V = pick_vec(C, dtype, io, 4, f32, 3);
    if (L * B * (C / V) > int64_t(0x7fffffff) * 256) return WKV_ERR_SHAPE;
    const bool g = r != nullptr;
#define WKV_STEP(IO_, V_)                                                                  \
    (g ? launch_step<IO_, V_, true>(L, B, C, w, u, k, v, r, state, y, stream)              \
       : launch_step<IO_, V_, false>(L, B, C, w, u, k, v, r, state, y, stream))
    int rc;
    if (dtype == WKV_F32)
        rc = V == 2 ? WKV_STEP(float, 2) : WKV_STEP(float, 1);
    else
        rc = V == 2 ? WKV_STEP(__nv_bfloat16, 2) : WKV_STEP(__nv_bfloat16, 1);
#undef WKV_STEP
    return rc != WKV_OK ? rc : check_launch();
}

int wkv_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int nmix, const void* x, const float* mu,
                    const void* x_prev, void* out, void* x_last, cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n) || nmix < 1 || nmix > wkv::kShiftMaxMix || n > kMaxElems / nmix) return WKV_ERR_SHAPE;
    if (B == 0 || C == 0) return WKV_OK;
    const size_t eb = elem_bytes(dtype);
    const size_t lane_bytes = size_t(B) * C * eb, io_bytes = size_t(n) * eb;
    const size_t out_bytes = io_bytes * nmix, mu_bytes = size_t(nmix) * C * 4;
    if (!aligned(x, eb) || !aligned(mu, 4) || !aligned(out, eb) || !aligned(x_prev, eb) || !aligned(x_last, eb))
        return WKV_ERR_ALIGN;
    if (x_last && x_prev && x_last != x_prev && overlaps(x_last, lane_bytes, x_prev, lane_bytes))
        return WKV_ERR_ALIAS;
    if (T == 0) {
        if (x_last == nullptr || x_last == x_prev) return WKV_OK;
        if (x_prev == nullptr) return record_cuda(cudaMemsetAsync(x_last, 0, lane_bytes, stream));
        return record_cuda(cudaMemcpyAsync(x_last, x_prev, lane_bytes, cudaMemcpyDeviceToDevice, stream));
    }
    if (!x || !mu || !out) return WKV_ERR_NULLPTR;
    if (overlaps(out, out_bytes, x, io_bytes) || overlaps(out, out_bytes, mu, mu_bytes) ||
        overlaps(out, out_bytes, x_prev, lane_bytes) || overlaps(out, out_bytes, x_last, lane_bytes))
        return WKV_ERR_ALIAS;
    if (overlaps(x_last, lane_bytes, x, io_bytes) || overlaps(x_last, lane_bytes, mu, mu_bytes)) return WKV_ERR_ALIAS;
    // 16-byte accesses when every array and row allows them
    const int64_t vw = static_cast<int64_t>(16 / eb);
    const bool vec = C % vw == 0 && aligned(x, 16) && aligned(mu, 16) && aligned(out, 16) &&
                     (x_prev == nullptr || aligned(x_prev, 16)) && (x_last == nullptr || aligned(x_last, 16));
    int rc;
    if (dtype == WKV_F32)
        rc = vec ? launch_shift<float, 4>(B, T, C, nmix, x, mu, x_prev, out, x_last, stream)
                 : launch_shift<float, 1>(B, T, C, nmix, x, mu, x_prev, out, x_last, stream);
    else
        rc = vec ? launch_shift<__nv_bfloat16, 8>(B, T, C, nmix, x, mu, x_prev, out, x_last, stream)
                 : launch_shift<__nv_bfloat16, 1>(B, T, C, nmix, x, mu, x_prev, out, x_last, stream);
    return rc != WKV_OK ? rc : check_launch();
}

// ---------------------------------------------------------------------------
// Allocation-free variant of wkv_forward.  The chunked look-back kernel's
// cross-block scratch lives in this fixed device array instead of a caller
// workspace.  Host code cannot use the array's name as a device address, so
// the address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[WKV_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up on
// the first call per device, with that device current).
int noalloc_scratch(void** out) {
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        rc = record_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        if (rc != WKV_OK) return rc;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return WKV_OK;
}

// Scratch a call would use: the workspace wkv_forward takes for these sizes
// (its look-back and hand-off words), or 0 when wkv_forward needs none.
size_t noalloc_need(int64_t B, int64_t T, int64_t C, int dtype) {
    return wkv_forward_workspace_bytes(B, T, C, dtype);
}

}  // namespace

extern "C" {

size_t wkv_forward_noalloc_scratch_bytes(int64_t B, int64_t T, int64_t C, int dtype) {
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n) || n == 0 || (dtype != WKV_F32 && dtype != WKV_BF16)) return 0;
    return noalloc_need(B, T, C, dtype);
}

int wkv_forward_noalloc(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                        const void* k, const void* v, const void* r, const float* state_in, void* y,
                        float* state_out, cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n)) return WKV_ERR_SHAPE;
    const size_t need = (B == 0 || C == 0 || T == 0) ? 0 : noalloc_need(B, T, C, dtype);
    if (need > 0) {
        // argument errors first: nothing, not even the array, is written then
        const int vrc = forward_args(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out);
        if (vrc != WKV_OK) return vrc;
    }
    if (need == 0 || (fits_cluster(dtype, B, T, C, k, v, r, w, u, state_in, y, state_out) && forced_kernel() == 0)) {
        // nothing to do, or a call whose kernel needs no scratch (short
        // sequences, or one cluster of parts per sequence): the regular entry
        // point without a workspace does exactly that, and touches no array
        return wkv_forward(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out, nullptr, 0, stream);
    }
    if (need > WKV_NOALLOC_SCRATCH_BYTES) return WKV_ERR_SCRATCH;
    void* ws = nullptr;
    int rc = noalloc_scratch(&ws);
    if (rc != WKV_OK) return rc;
    // every call starts from a zeroed header and zeroed words: counters,
    // error word and epoch at 0, and no word left over from an earlier call
    rc = record_cuda(cudaMemsetAsync(ws, 0, need, stream));
    if (rc != WKV_OK) return rc;
    return wkv_forward(B, T, C, dtype, w, u, k, v, r, state_in, y, state_out, ws, need, stream);
}

int wkv_forward_noalloc_status(cudaStream_t stream) {
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    void* ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        ws = g_noalloc_ptr[dev];
    }
    // no call on this device has used the array yet: nothing can have failed
    if (ws == nullptr) return record_cuda(cudaStreamSynchronize(stream));
    return wkv_workspace_status(ws, stream);
}

}  // extern "C"


// ---------------------------------------------------------------------------
// reverse mode
// ---------------------------------------------------------------------------
namespace {

// Backward kernel: 8 compute warps x 8-token segments, the 64-token chunks
// of the checkpoint sweep.
constexpr int kBwdW = 8;
constexpr int kBwdLS = 8;
static_assert(kBwdW * kBwdLS == kLaneW * kLaneLS, "the backward walks the checkpoint sweep's chunks");

struct BwdLayout {
    int64_t nCB, nLB, nchunks;
    size_t ckpt_off, part_off, bytes;
};

// Workspace of wkv_backward: header, the checkpoint sweep's hand-off words,
// the checkpoints, the dw/du partials.
BwdLayout bwd_layout(int64_t B, int64_t T, int64_t C) {
    BwdLayout L{};
    constexpr int64_t CB = 64;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    L.nCB = (C + CB - 1) / CB;
    L.nLB = B * L.nCB;
    L.nchunks = (T + kBwdW * kBwdLS - 1) / (kBwdW * kBwdLS);
    L.ckpt_off = 256 + up(size_t(L.nLB) * CB * sizeof(wkv::Word));
    L.part_off = L.ckpt_off + up(size_t(L.nchunks + 1) * size_t(L.nLB) * CB * sizeof(wkv::St));
    L.bytes = L.part_off + up(2 * size_t(L.nLB) * CB * sizeof(float));
    return L;
}

// Reverse walk: CTAs take equal shares of the lane-major (lane block, chunk)
// order like the lane-resident forward kernel; grid = min(lane blocks,
// resident capacity), with one reverse state handed between neighbours
// through the workspace when a lane block is split.
template <typename IO, bool GATE, int S, int MAXREG>
int launch_backward(wkv::BwdArgs a, int dtype, void* workspace, cudaStream_t st) {
    using G = wkv::BwdGeometry<IO, GATE, kBwdW, kBwdLS, S>;
    auto kern = wkv::lane_backward_kernel<IO, GATE, kBwdW, kBwdLS, S, MAXREG>;
    static int capacity[kMaxDevices] = {0};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (capacity[dev] == 0) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        int per_sm = 0;
        rc = record_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, G::THREADS, G::SMEM));
        if (rc != WKV_OK) return rc;
        // a configuration that fits no SM is an error, not one CTA per SM
        if (per_sm <= 0) return record_cuda(cudaErrorLaunchOutOfResources);
        capacity[dev] = per_sm * sm_count();
    }
    const int64_t grid = a.nLB < capacity[dev] ? a.nLB : capacity[dev];
    if (grid < a.nLB && a.nchunks > 1) {
        a.hdr = reinterpret_cast<wkv::WsHeader*>(workspace);
        a.incw = reinterpret_cast<wkv::Word*>(static_cast<char*>(workspace) + 256);
    } else {
        a.hdr = nullptr;
        a.incw = nullptr;
    }
    // The walk visits neighbouring lane blocks at different times when CTAs
    // split them, so an L2 fetch wider than a tile row brings in bytes no CTA
    // reads before they are evicted: promote to the row's width (128 bytes
    // for bfloat16), not 256 bytes.
    const CUtensorMapL2promotion promo =
        G::ROW >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
    CUtensorMap tk, tv, tdy, tr;
    if (!encode_map(&tk, a.k, dtype, a.B, a.T, a.C, G::CB, G::TT, promo) ||
        !encode_map(&tv, a.v, dtype, a.B, a.T, a.C, G::CB, G::TT, promo) ||
        !encode_map(&tdy, a.dy, dtype, a.B, a.T, a.C, G::CB, G::TT, promo))
        return WKV_ERR_CUDA;
    if (GATE) {
        if (!encode_map(&tr, a.r, dtype, a.B, a.T, a.C, G::CB, G::TT, promo)) return WKV_ERR_CUDA;
    } else {
        tr = tk;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(G::THREADS);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, kern, tk, tv, tdy, tr, a));
}

template <typename IO>
int run_backward(const wkv::BwdArgs& b, wkv::ChunkArgs f, int dtype, void* ws, size_t ws_bytes, cudaStream_t st) {
    // checkpoint sweep (ring depth as in the forward), then the reverse walk
    constexpr int SF = sizeof(IO) == 4 ? 2 : 3;
    int rc = launch_lane<IO, false, kLaneW, kLaneLS, SF, 2, true>(f, dtype, ws, ws_bytes, st);
    if (rc != WKV_OK) return rc;
    rc = record_cuda(cudaMemsetAsync(b.part, 0, 2 * size_t(b.nLB) * 64 * sizeof(float), st));
    if (rc != WKV_OK) return rc;
    // three stages, one CTA (9 warps) per SM.  Registers: each of the SM's 4
    // sub-partitions holds 16K, and one of them carries 3 of the 9 warps, so
    // at most 168 per thread.  Two CTAs per SM would cap registers at 112,
    // and the spills cost more than the second CTA gains (measured on the
    // 14B-shaped layer: 1715 vs 1348 us).
    return b.r != nullptr ? launch_backward<IO, true, 3, 168>(b, dtype, ws, st)
                          : launch_backward<IO, false, 3, 168>(b, dtype, ws, st);
}

}  // namespace

extern "C" {

size_t wkv_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int dtype) {
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n) || (dtype != WKV_F32 && dtype != WKV_BF16)) return 0;
    if (n == 0) return 0;
    return bwd_layout(B, T, C).bytes;
}

int wkv_backward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                 const void* k, const void* v, const void* r, const float* state_in, const void* dy,
                 const float* dstate_out, void* dk, void* dv, void* dr, float* dw, float* du, float* dstate_in,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    chain_forget(workspace);
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n)) return WKV_ERR_SHAPE;
    if (C == 0) return WKV_OK;
    if (!dw || !du) return WKV_ERR_NULLPTR;
    const int64_t lanes = B * C;
    const size_t eb = elem_bytes(dtype);
    const size_t io_bytes = size_t(n) * eb, st_bytes = size_t(lanes) * 3 * 4, p_bytes = size_t(C) * 4;
    if (!aligned(dw, 4) || !aligned(du, 4)) return WKV_ERR_ALIGN;
    if (overlaps(dw, p_bytes, du, p_bytes)) return WKV_ERR_ALIAS;
    if (n == 0) {
        // no token: dw = du = 0, and the returned state's gradient passes through
        int rc = record_cuda(cudaMemsetAsync(dw, 0, p_bytes, stream));
        if (rc != WKV_OK) return rc;
        rc = record_cuda(cudaMemsetAsync(du, 0, p_bytes, stream));
        if (rc != WKV_OK || dstate_in == nullptr || lanes == 0) return rc;
        if (!aligned(dstate_in, 4) || (state_in && !aligned(state_in, 4)) || (dstate_out && !aligned(dstate_out, 4)))
            return WKV_ERR_ALIGN;
        wkv::bwd_passthrough_kernel<<<static_cast<unsigned>((lanes + 255) / 256), 256, 0, stream>>>(
            lanes, state_in, dstate_out, dstate_in);
        return check_launch();
    }
    if (!w || !u || !k || !v || !dy || !dk || !dv) return WKV_ERR_NULLPTR;
    if ((r == nullptr) != (dr == nullptr)) return WKV_ERR_NULLPTR;
    // TMA tiles and paired-channel stores: 16-byte aligned arrays, C a multiple of 4
    const void* arrs[] = {k, v, r, dy, dk, dv, dr, w, u, state_in, dstate_out, dstate_in};
    for (const void* p : arrs)
        if (p && !aligned(p, 16)) return WKV_ERR_ALIGN;
    if (C % 4 != 0 || (C * int64_t(eb)) % 16 != 0) return WKV_ERR_ALIGN;
    if (B >= (int64_t(1) << 31) || T >= (int64_t(1) << 31) || C >= (int64_t(1) << 31)) return WKV_ERR_SHAPE;
    // outputs overlap no input and no other output
    struct Span { const void* p; size_t n; };
    const Span ins[] = {{w, p_bytes}, {u, p_bytes}, {k, io_bytes}, {v, io_bytes}, {r, io_bytes},
                        {state_in, st_bytes}, {dy, io_bytes}, {dstate_out, st_bytes}};
    const Span outs[] = {{dk, io_bytes}, {dv, io_bytes}, {dr, io_bytes}, {dw, p_bytes}, {du, p_bytes},
                         {dstate_in, st_bytes}};
    for (const Span& o : outs) {
        for (const Span& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return WKV_ERR_ALIAS;
        for (const Span& o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return WKV_ERR_ALIAS;
    }
    const BwdLayout L = bwd_layout(B, T, C);
    if (workspace == nullptr || workspace_bytes < L.bytes) return WKV_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return WKV_ERR_ALIGN;
    char* ws = static_cast<char*>(workspace);
    if (L.nLB > 0x7fffffffLL) return WKV_ERR_SHAPE;
    if (encode_fn() == nullptr) return WKV_ERR_CUDA;   // no driver entry point for tensor maps

    wkv::ChunkArgs f{};
    f.w = w;
    f.u = u;
    f.k = k;
    f.v = v;
    f.s_in = state_in;
    f.B = B;
    f.T = T;
    f.C = C;
    f.nCB = L.nCB;
    f.nLB = L.nLB;
    f.nchunks = L.nchunks;
    f.units = L.nLB * L.nchunks;
    f.ckpt = reinterpret_cast<wkv::St*>(ws + L.ckpt_off);
    f.wait_limit_ns = wait_limit_ns();

    wkv::BwdArgs b{};
    b.w = w;
    b.u = u;
    b.k = k;
    b.v = v;
    b.r = r;
    b.dy = dy;
    b.s_in = state_in;
    b.ds_out = dstate_out;
    b.dk = dk;
    b.dv = dv;
    b.dr = dr;
    b.ds_in = dstate_in;
    b.ckpt = f.ckpt;
    b.part = reinterpret_cast<float*>(ws + L.part_off);
    b.B = B;
    b.T = T;
    b.C = C;
    b.nCB = L.nCB;
    b.nLB = L.nLB;
    b.nchunks = L.nchunks;
    b.wait_limit_ns = f.wait_limit_ns;
    if (B > 0) {
        const int rc = dtype == WKV_F32 ? run_backward<float>(b, f, dtype, workspace, workspace_bytes, stream)
                                        : run_backward<__nv_bfloat16>(b, f, dtype, workspace, workspace_bytes, stream);
        if (rc != WKV_OK) return rc;
    }
    wkv::bwd_reduce_kernel<<<static_cast<unsigned>((C + 255) / 256), 256, 0, stream>>>(b.part, B, C, L.nCB, dw, du);
    return check_launch();
}

}  // extern "C"


// ---------------------------------------------------------------------------
// multi-head matrix-state WKV (v5 / v6)
// ---------------------------------------------------------------------------
namespace {

constexpr int kWkv5TB = 32;

template <typename IO, int N, bool PERTOK>
int launch_wkv5(const wkv::Wkv5Args& a, cudaStream_t st) {
    using G = wkv::Wkv5Geometry<N, kWkv5TB>;
    auto kern = wkv::wkv5_forward_kernel<IO, N, kWkv5TB, PERTOK>;
    static bool ready[kMaxDevices] = {false};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (!ready[dev]) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
        if (rc != WKV_OK) return rc;
        ready[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.B * a.H));
    cfg.blockDim = dim3(G::THREADS);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, kern, a));
}

// Matrix-state WKV in blocks of tokens on the tensor cores: one CTA of 128
// threads per (sequence, head).
template <bool PERTOK>
int launch_wkv5_tc(const wkv::Wkv5Args& a, cudaStream_t st) {
    using SG = wkv::TcStage;
    auto kern = wkv::wkv5_tc_kernel<PERTOK>;
    static bool ready[kMaxDevices] = {false};
    int dev = 0;
    int rc = record_cuda(cudaGetDevice(&dev));
    if (rc != WKV_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    if (!ready[dev]) {
        rc = record_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SG::SMEM));
        if (rc != WKV_OK) return rc;
        // all of the unified L1 / shared memory as shared memory, so that two
        // CTAs fit on one SM
        rc = record_cuda(
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared));
        if (rc != WKV_OK) return rc;
        ready[dev] = true;
    }
    // windows of 64 tokens x one head's 64 channels
    CUtensorMap tr, tk, tv, tw;
    if (!encode_map(&tr, a.r, WKV_BF16, a.B, a.T, a.C, 64, 64) || !encode_map(&tk, a.k, WKV_BF16, a.B, a.T, a.C, 64, 64) ||
        !encode_map(&tv, a.v, WKV_BF16, a.B, a.T, a.C, 64, 64))
        return WKV_ERR_CUDA;
    if (PERTOK) {
        if (!encode_map(&tw, a.w, WKV_F32, a.B, a.T, a.C, 64, 64)) return WKV_ERR_CUDA;
    } else {
        tw = tk;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.B * a.H));
    cfg.blockDim = dim3(wkv::kTcThreads);
    cfg.dynamicSmemBytes = SG::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return record_cuda(cudaLaunchKernelEx(&cfg, kern, tr, tk, tv, tw, a));
}

// WKV5_KERNEL=recurrent keeps every shape on the CUDA-core recurrence; read
// once.
bool wkv5_recurrent_forced() {
    static const bool v = []() {
        const char* e = std::getenv("WKV5_KERNEL");
        return e != nullptr && std::strcmp(e, "recurrent") == 0;
    }();
    return v;
}

template <typename IO, int N>
int dispatch_wkv5(bool pertok, const wkv::Wkv5Args& a, cudaStream_t st) {
    return pertok ? launch_wkv5<IO, N, true>(a, st) : launch_wkv5<IO, N, false>(a, st);
}

}  // namespace

extern "C" {

int wkv5_forward(int64_t B, int64_t T, int64_t C, int64_t H, int dtype, const float* w, int w_per_token,
                 const float* u, const void* r, const void* k, const void* v, const float* state_in, void* y,
                 float* state_out, cudaStream_t stream) {
    if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_DTYPE;
    int64_t n = 0;
    if (!mul_ok(B, T, C, &n) || H <= 0 || C % H != 0) return WKV_ERR_SHAPE;
    const int64_t N = C / H;
    if (B == 0 || C == 0) return WKV_OK;
    if (N != 32 && N != 64) return WKV_ERR_SHAPE;
    if (B * H > 0x7fffffffLL) return WKV_ERR_SHAPE;
    const size_t st_bytes = size_t(B) * size_t(H) * size_t(N) * size_t(N) * 4;
    if (T == 0) {
        if (state_out == nullptr || state_out == state_in) return WKV_OK;
        if (!aligned(state_out, 4) || (state_in && !aligned(state_in, 4))) return WKV_ERR_ALIGN;
        if (state_in && overlaps(state_in, st_bytes, state_out, st_bytes)) return WKV_ERR_ALIAS;
        if (state_in) return record_cuda(cudaMemcpyAsync(state_out, state_in, st_bytes, cudaMemcpyDeviceToDevice, stream));
        return record_cuda(cudaMemsetAsync(state_out, 0, st_bytes, stream));
    }
    if (!w || !u || !r || !k || !v || !y) return WKV_ERR_NULLPTR;
    const size_t eb = elem_bytes(dtype);
    const size_t io_bytes = size_t(n) * eb, p_bytes = size_t(C) * 4;
    const size_t w_bytes = w_per_token ? size_t(n) * 4 : p_bytes;
    if (!aligned(w, 4) || !aligned(u, 4) || !aligned(r, eb) || !aligned(k, eb) || !aligned(v, eb) ||
        !aligned(y, eb) || (state_in && !aligned(state_in, 4)) || (state_out && !aligned(state_out, 4)))
        return WKV_ERR_ALIGN;
    struct Span { const void* p; size_t n; };
    const Span ins[] = {{w, w_bytes}, {u, p_bytes}, {r, io_bytes}, {k, io_bytes}, {v, io_bytes}};
    for (const Span& i : ins) {
        if (overlaps(y, io_bytes, i.p, i.n)) return WKV_ERR_ALIAS;
        if (state_out && overlaps(state_out, st_bytes, i.p, i.n)) return WKV_ERR_ALIAS;
    }
    if (overlaps(y, io_bytes, state_in, st_bytes) || overlaps(y, io_bytes, state_out, st_bytes)) return WKV_ERR_ALIAS;
    if (state_out && state_in && state_in != state_out && overlaps(state_out, st_bytes, state_in, st_bytes))
        return WKV_ERR_ALIAS;
    wkv::Wkv5Args a{};
    a.w = w;
    a.u = u;
    a.r = r;
    a.k = k;
    a.v = v;
    a.s_in = state_in;
    a.y = y;
    a.s_out = state_out;
    a.B = B;
    a.T = T;
    a.C = C;
    a.H = H;
    const bool pt = w_per_token != 0;
    int rc;
    // bf16 heads of 64 take the tensor-core blocks (their outputs carry tf32
    // products, within bf16's own rounding; the state keeps fp32 accuracy);
    // they read r, k, v, w by TMA and store y and the states 16 bytes at a
    // time.  float32 keeps the exact-fp32 recurrence.
    const bool tc = dtype == WKV_BF16 && N == 64 && aligned(y, 16) && (!state_in || aligned(state_in, 16)) &&
                    (!state_out || aligned(state_out, 16)) && aligned(r, 16) && aligned(k, 16) && aligned(v, 16) &&
                    (!pt || aligned(w, 16)) && T < (int64_t(1) << 31) && B < (int64_t(1) << 31) &&
                    encode_fn() != nullptr && !wkv5_recurrent_forced();
    if (tc)
        rc = pt ? launch_wkv5_tc<true>(a, stream) : launch_wkv5_tc<false>(a, stream);
    else if (dtype == WKV_F32)
        rc = N == 64 ? dispatch_wkv5<float, 64>(pt, a, stream) : dispatch_wkv5<float, 32>(pt, a, stream);
    else
        rc = N == 64 ? dispatch_wkv5<__nv_bfloat16, 64>(pt, a, stream) : dispatch_wkv5<__nv_bfloat16, 32>(pt, a, stream);
    return rc != WKV_OK ? rc : check_launch();
}

}  // extern "C"
