/*
 * wkv.h -- C ABI of libwkv.so, the sm_100a (B200) implementation of the RWKV-4
 * WKV time-mixing operator.
 *
 * The operator.  The article "RWKVアーキテクチャ徹底解説：Transformerに匹敵する
 * 線形アテンションRNN" (youngju.dev) defines, per channel c of a sequence
 * (section "コア計算", the explicit sum):
 *
 *   wkv_t = ( sum_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t}     )
 *
 * with a per-channel decay w = exp(decay) > 0 and bonus u.  Its block diagram
 * ("高レベル構造") gates the result, out_t = sigmoid(r_t) * wkv_t.  The same
 * article evaluates the sum as a recurrence over a (numerator, denominator,
 * running max) state ("リカレント定式化", "対数空間計算による数値安定性") in
 * two modes that give the same result: a parallel pass over a chunk and one
 * token at a time ("二重性：Transformerモード vs RNNモード").  The skill page
 * "rwkv-architecture" (agnxi.com) streams a long document through chunks while
 * carrying that state ("Process million-token sequences").
 *
 * Layouts (row-major, channel fastest, no padding):
 *   k, v, r, y : (B, T, C) in the dtype `dtype` (all four the same)
 *   w, u       : (C,) float32
 *   state      : (3, B, C) float32 = {a, b, p}: numerator N = a*e^p and
 *                denominator D = b*e^p of all tokens seen so far, before the
 *                decay of the next step.  p is a natural-log exponent.  The
 *                empty state is (0, 0, -1e38).  After a call, p follows the
 *                running-max convention p <- max(p - w, k_t).
 *
 * Ownership and execution.  The caller allocates every buffer, in device
 * memory of the current CUDA device.  The library allocates nothing and keeps
 * no state except a per-device SM-count cache and a thread-local message for
 * the last CUDA error.  Every call is asynchronous on `stream` (a cudaStream_t;
 * NULL is the legacy default stream) and returns before the GPU finishes.
 *
 * Errors.  Every entry point returns a wkv_status.  Argument errors are found
 * on the host before anything is launched; nothing is written then.
 * WKV_ERR_CUDA reports a launch failure (wkv_last_cuda_error() has the text).
 * Errors that only the GPU can see (a cross-block wait that ran out of time)
 * are recorded in the workspace and read with wkv_workspace_status().
 */
#ifndef WKV_H_
#define WKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

/* dtype of k, v, r and y.  w, u and the state are always float32. */
typedef enum { WKV_F32 = 0, WKV_BF16 = 1 } wkv_dtype;

typedef enum {
    WKV_OK = 0,
    WKV_ERR_NULLPTR = -1,    /* a required pointer is NULL */
    WKV_ERR_SHAPE = -2,      /* negative size, or B*T*C / L*B*C beyond 2^62 */
    WKV_ERR_DTYPE = -3,      /* dtype is not a wkv_dtype */
    WKV_ERR_ALIGN = -4,      /* pointer not aligned to its element (workspace: 256 B) */
    WKV_ERR_ALIAS = -5,      /* an output overlaps an input or another output */
    WKV_ERR_CUDA = -6,       /* CUDA launch error; see wkv_last_cuda_error() */
    WKV_ERR_TIMEOUT = -7,    /* a cross-block wait on the GPU gave up (from wkv_workspace_status) */
    WKV_ERR_WORKSPACE = -8,  /* wkv_backward: workspace NULL or smaller than wkv_backward_workspace_bytes() */
    WKV_ERR_SCRATCH = -9     /* wkv_forward_noalloc: problem needs more than its built-in scratch */
} wkv_status;

/*
 * wkv_forward -- parallel ("GPT") mode over one chunk of T tokens.
 *
 * For every lane (b, c) it computes y[b,t,c] = sigmoid(r[b,t,c]) * wkv_t (no
 * sigmoid factor when r is NULL) for t = 0..T-1, where the state `state_in`
 * enters the sums as the tokens before the chunk: it contributes
 * e^{-t w} * N_in to the numerator (and D_in to the denominator) of output t.
 * state_out receives the state after token T-1, so feeding it back as the
 * next chunk's state_in reproduces one unchunked pass.
 *
 *   B, T, C      sizes, each >= 0.  B == 0 or C == 0: nothing to do.  T == 0:
 *                y untouched, state_out = state_in (or the empty state).
 *   dtype        wkv_dtype of k, v, r, y.
 *   w, u         (C,) float32 device arrays; w > 0 (not checked on the device).
 *   k, v         (B,T,C) device arrays, required.
 *   r            (B,T,C) device array, or NULL for no gate.
 *   state_in     (3,B,C) float32 device array, or NULL for the empty state.
 *   y            (B,T,C) device array, written.  Must not overlap any input.
 *   state_out    (3,B,C) float32 device array, or NULL.  May be the same
 *                pointer as state_in (in-place update); any other overlap
 *                with an input or with y is WKV_ERR_ALIAS.
 *   workspace    optional device scratch of at least
 *                wkv_forward_workspace_bytes(B,T,C,dtype) bytes, 256-byte
 *                aligned, zeroed once by wkv_workspace_init() before its
 *                first use and reusable by any later call with any shape.
 *                Calls sharing a workspace must be ordered on the GPU (same
 *                stream, or synchronised); they race otherwise.  With it,
 *                CTAs that split one sequence exchange partial states
 *                through it (decoupled look-back, state hand-off), which is
 *                the fastest schedule for most shapes.  An ungated bfloat16
 *                call longer than 2048 tokens with 48 to 147 channel blocks
 *                of 64 (B * ceil(C/64)) runs as a chain of launches of 1024
 *                tokens instead, handing the state from launch to launch
 *                through the workspace (see WKV_FLAG_CHAIN_NEXT below).
 *                NULL (or too small: it is then not touched) is accepted for
 *                every shape; the call then runs a schedule that needs no
 *                scratch: the sequential kernel for T <= 16; the cluster
 *                kernel (thread block clusters of ceil(T/128) CTAs that
 *                combine their parts' summaries in distributed shared
 *                memory) when 17 <= T <= 1024, C is a multiple of 4 (of 8
 *                for bfloat16), k, v, r, w, u, state_in are 16-byte aligned
 *                and y, state_out aligned to two elements; otherwise, for
 *                such TMA-eligible arrays, the lane-resident kernel with
 *                whole sequences' channel blocks per CTA, and for any other
 *                layout the per-lane recurrence.  Those last two give the
 *                same results but can be several times slower when there
 *                are few lanes (one long sequence) or slightly more lane
 *                blocks than the GPU holds at once.
 *   stream       CUDA stream of the launch.
 *
 * The operator's own call is (B, T, C, dtype, w, u, k, v, r, state_in, y,
 * state_out, stream).  The two workspace arguments are an addition to it: the
 * library allocates nothing, so the scratch of the fastest schedules has to
 * come from the caller.  Passing NULL, 0 gives the plain call on every shape.
 */
int wkv_forward(int64_t B, int64_t T, int64_t C, int dtype,
                const float* w, const float* u,
                const void* k, const void* v, const void* r,
                const float* state_in, void* y, float* state_out,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * wkv_forward_ex -- wkv_forward with launch flags.  flags == 0 is exactly
 * wkv_forward.  Any bit other than those below is WKV_ERR_SHAPE.
 *
 *   WKV_FLAG_INPUTS_READY  the caller declares that k, v, r, w and u are not
 *       written by any work still running on `stream` when this call is
 *       enqueued (they were produced earlier and are left alone).  Every
 *       kernel here is launched with programmatic dependent launch, so its
 *       thread blocks can start while the stream's previous kernel drains;
 *       with this flag the stream kernel (the chunk of a carried stream: few
 *       lane blocks, up to 8 parts of 256 bfloat16 / 128 float32 tokens)
 *       loads its inputs and forms every segment summary and prefix before
 *       it waits for that kernel, and only the state fold and the outputs
 *       wait.  state_in (written by the previous chunk), y and state_out are
 *       touched only after the wait, so chaining chunks with the state in
 *       place stays correct.  Without the flag, every kernel waits for the
 *       previous kernel before its first memory access.  Setting it while
 *       an input is still being written gives wrong results.
 */
#define WKV_FLAG_INPUTS_READY 1u
/*
 *   WKV_FLAG_CHAIN_BEGIN, WKV_FLAG_CHAIN_NEXT  (each implies
 *       WKV_FLAG_INPUTS_READY; setting both is WKV_ERR_SHAPE) a chain of
 *       chunk calls on `stream` that carry one state: the first call passes
 *       WKV_FLAG_CHAIN_BEGIN and reads state_in after the previous kernel of
 *       the stream ends, as with WKV_FLAG_INPUTS_READY.  Every later call
 *       passes WKV_FLAG_CHAIN_NEXT, declaring that its state_in is the
 *       state_out of the previous call of the chain, that nothing has
 *       written it since, and that that call was given the same workspace,
 *       B, C and dtype.  When the stream kernel runs and the workspace holds
 *       at least 256 + 16 * B * C bytes (every workspace of
 *       wkv_forward_workspace_bytes() for T > 64 does), each call publishes
 *       the state it leaves in the workspace as soon as that state is formed,
 *       before its outputs (one 16-byte word per channel, tagged with the
 *       call's position in the chain), and a WKV_FLAG_CHAIN_NEXT call waits
 *       for that word instead of for the end of the previous kernel.  Each
 *       call still writes state_out, and its kernel does not finish before
 *       the previous one has.  The first call clears the words (one
 *       cudaMemsetAsync of 16 * B * C bytes before its kernel).
 *       The workspace belongs to the chain until the chain ends: any other
 *       call on it ends the chain, and a WKV_FLAG_CHAIN_NEXT call with no
 *       matching predecessor (other workspace, sizes, or a state_in that is
 *       not the previous state_out) reads state_in as a first call does.
 *       With either flag, y may be written before the previous kernel of the
 *       stream ends: it must not be the previous call's y.  A wait for the
 *       previous word that exceeds the wait limit records WKV_ERR_TIMEOUT in
 *       the workspace (wkv_workspace_status) and makes the state and outputs
 *       NaN.  A false declaration gives wrong results or a timeout, never a
 *       hang.
 */
#define WKV_FLAG_CHAIN_BEGIN 2u
#define WKV_FLAG_CHAIN_NEXT 4u

int wkv_forward_ex(int64_t B, int64_t T, int64_t C, int dtype,
                   const float* w, const float* u,
                   const void* k, const void* v, const void* r,
                   const float* state_in, void* y, float* state_out,
                   void* workspace, size_t workspace_bytes, unsigned flags,
                   cudaStream_t stream);

/* Bytes of workspace wkv_forward needs for these sizes (0: none).  Returns 0
 * for invalid sizes too; wkv_forward then reports the argument error. */
size_t wkv_forward_workspace_bytes(int64_t B, int64_t T, int64_t C, int dtype);

/* Zero `bytes` bytes of a workspace on `stream` (cudaMemsetAsync).  Needed
 * once after allocation, and again after wkv_workspace_status() reported an
 * error. */
int wkv_workspace_init(void* workspace, size_t bytes, cudaStream_t stream);

/* Synchronise `stream`, then read the error word the kernels keep in the
 * workspace: WKV_OK, or WKV_ERR_TIMEOUT if a wait for another block's partial
 * result gave up (those outputs were written as NaN). */
int wkv_workspace_status(const void* workspace, cudaStream_t stream);

/*
 * wkv_state -- the state a chunk leaves behind, without its outputs.
 *
 * state_out = the state after T tokens entered from state_in (NULL: the
 * empty state): exactly wkv_forward's state_out for the same k, v, w and
 * state_in, with no y.  The state does not depend on u or on the gate, so
 * neither is taken.  Entered from the empty state it is the chunk's
 * summary, the element of the scan that "並列学習の定式化" (article
 * "RWKVアーキテクチャ徹底解説") says the parallel mode performs: summaries of
 * consecutive chunks combine associatively (wkv_state_combine).  That is what
 * lets one sequence be split along T across GPUs ("Process million-token
 * sequences" on the skill page "rwkv-architecture" streams a long document
 * through chunks with the state carried): each GPU forms its chunk's summary,
 * the summaries are exchanged and folded into every chunk's entering state,
 * and each GPU then runs wkv_forward on its chunk from that state.
 *
 *   B, T, C      sizes, each >= 0 (B == 0 or C == 0: nothing to do; T == 0:
 *                state_out = state_in).
 *   dtype        wkv_dtype of k and v.
 *   w            (C,) float32.   k, v: (B,T,C) device arrays.
 *   state_in     (3,B,C) float32 or NULL.
 *   state_out    (3,B,C) float32, required; may equal state_in, must not
 *                overlap anything else.
 *   workspace    as for wkv_forward (optional; NULL runs a scratch-free
 *                schedule).
 * Reads k and v once; writes only state_out.  Errors as wkv_forward.
 */
int wkv_state(int64_t B, int64_t T, int64_t C, int dtype, const float* w,
              const void* k, const void* v, const float* state_in, float* state_out,
              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * wkv_state_combine -- fold chunk summaries into a state.
 *
 * state_out = the state after n consecutive chunks of lens[0], ...,
 * lens[n-1] tokens entered from state_in (NULL: the empty state), given each
 * chunk's own summary (wkv_state from the empty state).  With summary
 * (q, A, B) of a chunk of L tokens and a state (p, a, b) before it, the
 * state after it is p' = max(p - L w, q), a' = e^{p - L w - p'} a +
 * e^{q - p'} A, b' likewise: the recurrence of "リカレント定式化" applied to a
 * whole chunk at once.  Folding is associative, so the result equals one
 * wkv_state call over the concatenated chunks (up to rounding).
 *
 *   B, C         sizes (>= 0).
 *   n            number of chunks, 0 <= n <= 64 (0: state_out = state_in).
 *   w            (C,) float32 device array.
 *   lens         HOST array of n token counts (each >= 0), read during the
 *                call.
 *   states       (n,3,B,C) float32 device array of the summaries.
 *   state_in     (3,B,C) float32 device array or NULL.
 *   state_out    (3,B,C) float32 device array; may equal state_in, must not
 *                overlap states or w.
 * WKV_ERR_SHAPE for n outside 0..64 or a negative length.
 */
int wkv_state_combine(int64_t B, int64_t C, int n, const float* w, const int64_t* lens,
                      const float* states, const float* state_in, float* state_out,
                      cudaStream_t stream);

/*
 * wkv_step -- RNN ("decode") mode: one token for L independent layers, each
 * with B sequences, updating the state in place.  Equal to wkv_forward with
 * T = 1 on each layer (the article's dual-mode section and the skill page's
 * "RNN mode (sequential processing, same result)").
 *
 *   L, B, C      sizes, each >= 0 (any 0: nothing to do).
 *   dtype        wkv_dtype of k, v, r, y.
 *   w, u         (L, C) float32 device arrays, one row per layer.
 *   k, v         (L, B, C) device arrays, required.
 *   r            (L, B, C) device array, or NULL for no gate.
 *   state        (L, 3, B, C) float32 device array, read and overwritten.
 *   y            (L, B, C) device array, written.  No overlaps allowed.
 *   stream       CUDA stream of the launch.
 */
int wkv_step(int64_t L, int64_t B, int64_t C, int dtype,
             const float* w, const float* u,
             const void* k, const void* v, const void* r,
             float* state, void* y, cudaStream_t stream);

/*
 * wkv_forward_noalloc -- wkv_forward for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or forbidden (a
 * plug-in inside a host application that owns every allocation, a runtime
 * that hands out only pre-registered buffers, or a pre-recorded launch
 * sequence that must not touch the allocator).  The article has no counterpart
 * to this entry point; it only changes where the scratch memory comes from.
 *
 * Same arguments and results as wkv_forward, without the workspace.  The
 * cross-block scratch the chunked kernel needs comes from a fixed array
 * inside the library (WKV_NOALLOC_SCRATCH_BYTES bytes of device memory that
 * every GPU which loads the library keeps until the process exits), so
 * nothing is allocated.
 *
 *   - It runs the kernels wkv_forward runs with a workspace, with the array
 *     standing in for the workspace.
 *   - Limit: problems whose scratch need (wkv_forward_noalloc_scratch_bytes)
 *     exceeds WKV_NOALLOC_SCRATCH_BYTES are rejected with WKV_ERR_SCRATCH
 *     before anything runs (wkv_forward with a NULL workspace serves them
 *     without scratch, more slowly).  Calls whose wkv_forward needs no
 *     workspace, and TMA-eligible calls of at most 1024 tokens, which run
 *     the cluster kernel (described under wkv_forward's workspace), use no
 *     scratch: those share no array and need no ordering.
 *   - The first call on a device that uses the array looks up its device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before capturing a stream into a graph.  The address is
 *     kept per device ordinal for the process: it serves the device's
 *     primary context (the CUDA runtime's) and is not looked up again after
 *     cudaDeviceReset or for another driver context on the same device.
 *   - Every call on a device shares the one array and clears the part it
 *     uses at the start (a cudaMemsetAsync on `stream`).  Calls that may
 *     overlap on the GPU (different streams without ordering) race on it
 *     and give wrong results; order them.
 *   - A cross-block wait that runs out is recorded in the array's header
 *     (outputs are NaN then); wkv_forward_noalloc_status() reads it.  The
 *     next call that uses the array clears it.
 */
#define WKV_NOALLOC_SCRATCH_BYTES (32u << 20)

int wkv_forward_noalloc(int64_t B, int64_t T, int64_t C, int dtype,
                        const float* w, const float* u,
                        const void* k, const void* v, const void* r,
                        const float* state_in, void* y, float* state_out,
                        cudaStream_t stream);

/* Scratch bytes wkv_forward_noalloc would use for these sizes (0: none); an
 * upper bound: calls that take the cluster kernel (see wkv_forward's
 * workspace) use none and are not subject to WKV_NOALLOC_SCRATCH_BYTES. */
size_t wkv_forward_noalloc_scratch_bytes(int64_t B, int64_t T, int64_t C, int dtype);

/* Synchronise `stream`, then read the error word of the built-in array on
 * the current device: WKV_OK, or WKV_ERR_TIMEOUT if the last
 * wkv_forward_noalloc call that used the array had a wait for another
 * block's partial result give up (its outputs were written as NaN).  WKV_OK
 * when no call on this device has used the array.  Order it after the call
 * it checks and before the next one that uses the array. */
int wkv_forward_noalloc_status(cudaStream_t stream);

/*
 * wkv_backward -- gradients of wkv_forward over one chunk (reverse mode).
 * The pages state that the parallel mode is what trains the model (article
 * section "並列学習の定式化") but print no gradient; this is the chain rule
 * through the recurrence of "リカレント定式化", per lane, with N_t, D_t the
 * state's numerator and denominator before token t, lam = e^{-w},
 * den_t = D_t + e^{u+k_t}, wkv_t = (N_t + e^{u+k_t} v_t) / den_t:
 *
 *   dnum_t = g_t dy_t / den_t,  dden_t = -dnum_t wkv_t   (g_t = sigmoid(r_t), or 1)
 *   gN_t = dnum_t + lam gN_{t+1},  gD_t = dden_t + lam gD_{t+1}     (dL/dN_t, dL/dD_t)
 *   dv_t = dnum_t e^{u+k_t} + gN_{t+1} e^{k_t}
 *   dk_t = (dnum_t v_t + dden_t) e^{u+k_t} + (gN_{t+1} v_t + gD_{t+1}) e^{k_t}
 *   du = sum (dnum_t v_t + dden_t) e^{u+k_t},   dw = -lam sum (gN_{t+1} N_t + gD_{t+1} D_t)
 *   dr_t = dy_t wkv_t g_t (1 - g_t)
 *
 * Same sizes, dtype, layouts and state semantics as wkv_forward.
 *   w, u, k, v, r, state_in   the forward's inputs (r NULL: no gate; state_in
 *                             NULL: the empty state).
 *   dy                        (B,T,C) dL/dy, in `dtype`.
 *   dstate_out                (3,B,C) float32 dL/d(a, b) of the state the
 *                             forward returned, or NULL (zero).  Its p plane
 *                             is not read: every later use of a state depends
 *                             on it only through N = a e^p and D = b e^p, so
 *                             the chain continues through dL/dN = dL/da e^{-p}.
 *   dk, dv                    (B,T,C) outputs in `dtype`.
 *   dr                        (B,T,C) output in `dtype`; NULL exactly when r is.
 *   dw, du                    (C,) float32 outputs: sums over every sequence
 *                             and token of the channel (written, not added to).
 *                             dw is dL/dw; with w = exp(decay) the decay's
 *                             gradient is dw * w.
 *   dstate_in                 (3,B,C) float32 output dL/d(a0, b0, p0), or NULL;
 *                             dL/dp0 = a0 dL/da0 + b0 dL/db0.  Feeding its a, b
 *                             planes as dstate_out of the previous chunk
 *                             chains chunks exactly.
 *   workspace                 at least wkv_backward_workspace_bytes() bytes,
 *                             256-byte aligned, zeroed once by
 *                             wkv_workspace_init() before its first use (a
 *                             wkv_forward workspace of that size serves too).
 * Requirements of this version: every array 16-byte aligned and rows of a
 * multiple of 16 bytes, i.e. C a multiple of 4 for fp32 and of 8 for bf16
 * (WKV_ERR_ALIGN otherwise).  No output may overlap an input or another
 * output (WKV_ERR_ALIAS).  T == 0: dw = du = 0 and dstate_in passes
 * dstate_out through.  Asynchronous on `stream` like every call.
 */
int wkv_backward(int64_t B, int64_t T, int64_t C, int dtype,
                 const float* w, const float* u,
                 const void* k, const void* v, const void* r,
                 const float* state_in, const void* dy, const float* dstate_out,
                 void* dk, void* dv, void* dr, float* dw, float* du, float* dstate_in,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Bytes of workspace wkv_backward needs for these sizes (0 for invalid sizes
 * or no elements). */
size_t wkv_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int dtype);

/* Static English text for a wkv_status value. */
const char* wkv_strerror(int status);

/* Text of the last CUDA error seen by a call on this host thread ("" if none). */
const char* wkv_last_cuda_error(void);

/* ABI version of this header: 1. */
int wkv_abi_version(void);

/*
 * wkv5_forward -- multi-head WKV with matrix-valued states (the v5 "Eagle"
 * and v6 "Finch" generations of the article's "RWKVバージョンの進化 / v4から
 * v7まで": "multi-headed WKV, matrix-valued states" of h * (d/h)^2 numbers
 * per layer, and "data-dependent time decay").  The pages give no formula
 * beyond that line; this library reads it as follows.  Channels form H heads
 * of N = C / H; each head of each sequence keeps an N x N state S (key
 * channel i, value channel j).  Token t reads the state before its own
 * update, as the v4 operator's parallel loop does ("並列学習の定式化"), and
 * then every key row decays by e^{-w_t[i]} and the token's outer product is
 * added:
 *
 *   y[b,t,hN+j] = sum_i r_t[i] ( S[i][j] + u[hN+i] k_t[i] v_t[j] )
 *   S[i][j]    <- e^{-w_t[i]} S[i][j] + k_t[i] v_t[j]
 *
 * (r_t, k_t, v_t, w_t: the head's N channels of token t.)  There is no
 * normalising denominator and no exponential of k: with one channel per
 * head, k = e^{k4}, u = e^{u4} and r = 1 this is the v4 sum's numerator.
 *
 *   B, T, C, H   sizes; C % H == 0 and N = C / H is 32 or 64 (the pages' head
 *                size is 64); B == 0 or C == 0: nothing to do; T == 0:
 *                state_out = state_in (zeros if NULL).
 *   dtype        wkv_dtype of r, k, v, y.
 *   w            decay rates (>= 0), float32: (C,) when w_per_token == 0
 *                (v5), (B,T,C) when w_per_token != 0 (v6).
 *   u            (C,) float32 bonus.
 *   r, k, v      (B,T,C) device arrays in dtype.
 *   state_in     (B,H,N,N) float32 or NULL (zeros); S[b][h][i][j].
 *   y            (B,T,C) output in dtype (computed in float32, rounded once).
 *   state_out    (B,H,N,N) float32 or NULL; may equal state_in, must not
 *                overlap anything else.  Feeding it back as the next call's
 *                state_in chains chunks exactly like one pass.
 * Errors as wkv_forward (WKV_ERR_SHAPE for a head size other than 32 or 64).
 * bfloat16 heads of 64 (with y, r, k, v, w and the states 16-byte aligned)
 * run in blocks of up to 64 tokens on the tensor cores: the same sums
 * regrouped into 64 x 64 products, with tf32 operands for the outputs
 * (errors of order 1e-3 of the output's magnitude, below bf16's own
 * rounding) and float32 accuracy kept for the state.  Every other call runs
 * the recurrence in float32 on the CUDA cores (2 N multiply-adds per
 * element); the environment variable WKV5_KERNEL=recurrent, read once per
 * process, keeps every call on it.  Asynchronous on `stream`; no workspace.
 */
int wkv5_forward(int64_t B, int64_t T, int64_t C, int64_t H, int dtype,
                 const float* w, int w_per_token, const float* u,
                 const void* r, const void* k, const void* v,
                 const float* state_in, void* y, float* state_out,
                 cudaStream_t stream);

/*
 * wkv_token_shift -- the token shift that precedes the R, K, V projections of
 * every sub-layer (the article's section "トークンシフト：秘密の要素"): each
 * token's input mixed with the previous token's,
 *     out[m, b, t, c] = mu[m, c] * x[b, t, c] + (1 - mu[m, c]) * x[b, t-1, c],
 * with one learned weight per channel, for nmix mixes of one input (RWKV-4's
 * time mixing takes three: for K, V and R).  x[b, -1, :] is x_prev[b, :], the
 * input carried from the previous chunk or decode step; a fresh sequence
 * (x_prev NULL) mixes its first token with zeros.  Decode is T = 1.
 *
 *   B, T, C      sizes, each >= 0.  B == 0 or C == 0: nothing to do.
 *                T == 0: out untouched, x_last = x_prev (zeros if NULL).
 *   dtype        wkv_dtype of x, x_prev, out, x_last.
 *   nmix         number of mixes, 1..8.
 *   x            (B,T,C) device array, required.
 *   mu           (nmix, C) float32 device array, required.
 *   x_prev       (B,C) device array, or NULL for zeros.
 *   out          (nmix,B,T,C) device array, written; must not overlap any
 *                other argument.  Computed in float32 as mu*x_t +
 *                (1-mu)*x_{t-1} and rounded once to dtype.
 *   x_last       (B,C) device array or NULL: receives x[:, T-1, :], the
 *                x_prev of the next call.  May be the same pointer as x_prev
 *                (in-place update); other overlaps are WKV_ERR_ALIAS.
 *   stream       CUDA stream of the launch.
 *
 * Returns WKV_OK or an error before launching: WKV_ERR_SHAPE (negative size,
 * nmix outside 1..8, nmix*B*T*C beyond 2^62), WKV_ERR_NULLPTR, WKV_ERR_DTYPE,
 * WKV_ERR_ALIGN (a pointer not aligned to its element type), WKV_ERR_ALIAS,
 * WKV_ERR_CUDA.  16-byte aligned arrays with C a multiple of 4 (float32) or
 * 8 (bfloat16) take 16-byte accesses; any other layout runs element-wise.
 */
int wkv_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int nmix,
                    const void* x, const float* mu, const void* x_prev,
                    void* out, void* x_last, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_H_ */
