"""B200 (sm_100a) RWKV-4 WKV operator: Python binding of libwkv.so.

The binding only marshals arguments: every step of the operator runs in the
CUDA kernels behind the C ABI declared in ``include/wkv.h``.  There is no CPU
fallback; if ``libwkv.so`` is missing the import fails with instructions.

Two layers:

* ``lib()`` returns the ctypes handle; its functions carry the C names
  (``wkv_forward``, ``wkv_step``, ``wkv_forward_workspace_bytes``, ...) and take
  plain integers / pointers.
* ``wkv_forward(...)`` and ``wkv_step(...)`` below take torch CUDA tensors,
  allocate outputs and the workspace with torch when not given, pass
  ``data_ptr()`` values and the current stream, and raise ``WkvError`` on a
  non-zero status.
"""
import ctypes
import functools
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwkv.so")

WKV_F32 = 0
WKV_BF16 = 1
STATUS = {
    0: "WKV_OK", -1: "WKV_ERR_NULLPTR", -2: "WKV_ERR_SHAPE", -3: "WKV_ERR_DTYPE",
    -4: "WKV_ERR_ALIGN", -5: "WKV_ERR_ALIAS", -6: "WKV_ERR_CUDA", -7: "WKV_ERR_TIMEOUT",
    -8: "WKV_ERR_WORKSPACE", -9: "WKV_ERR_SCRATCH",
}
# the functions include/wkv.h declares
EXPORTS = ("wkv_forward", "wkv_forward_ex", "wkv_forward_workspace_bytes", "wkv_workspace_init", "wkv_workspace_status",
           "wkv_step", "wkv_forward_noalloc", "wkv_forward_noalloc_scratch_bytes", "wkv_forward_noalloc_status",
           "wkv_backward", "wkv_state", "wkv_state_combine", "wkv5_forward",
           "wkv_backward_workspace_bytes", "wkv_token_shift", "wkv_strerror", "wkv_last_cuda_error",
           "wkv_abi_version")

_lib = None
_lock = threading.Lock()


class WkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().wkv_strerror(status).decode()
        if status == -6:
            msg += ": " + lib().wkv_last_cuda_error().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def lib():
    """ctypes handle of libwkv.so with argument types set."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run "
                              "`python -c 'import __graft_entry__ as g; g.build()'` from the repository root "
                              "(or rwkv_wkv_recurrence_02_b200/build_ext.py)")
        L = ctypes.CDLL(LIB_PATH)
        i64, vp, i32, sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.wkv_forward.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.wkv_forward.restype = i32
        L.wkv_forward_ex.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, ctypes.c_uint, vp]
        L.wkv_forward_ex.restype = i32
        L.wkv_forward_workspace_bytes.argtypes = [i64, i64, i64, i32]
        L.wkv_forward_workspace_bytes.restype = sz
        L.wkv_workspace_init.argtypes = [vp, sz, vp]
        L.wkv_workspace_init.restype = i32
        L.wkv_workspace_status.argtypes = [vp, vp]
        L.wkv_workspace_status.restype = i32
        L.wkv_step.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.wkv_step.restype = i32
        L.wkv_token_shift.argtypes = [i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
        L.wkv_token_shift.restype = i32
        L.wkv_forward_noalloc.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.wkv_forward_noalloc.restype = i32
        L.wkv_forward_noalloc_scratch_bytes.argtypes = [i64, i64, i64, i32]
        L.wkv_forward_noalloc_scratch_bytes.restype = sz
        L.wkv_state.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.wkv_state.restype = i32
        L.wkv_state_combine.argtypes = [i64, i64, i32, vp, vp, vp, vp, vp, vp]
        L.wkv_state_combine.restype = i32
        L.wkv5_forward.argtypes = [i64, i64, i64, i64, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.wkv5_forward.restype = i32
        L.wkv_forward_noalloc_status.argtypes = [vp]
        L.wkv_forward_noalloc_status.restype = i32
        L.wkv_backward.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   vp, sz, vp]
        L.wkv_backward.restype = i32
        L.wkv_backward_workspace_bytes.argtypes = [i64, i64, i64, i32]
        L.wkv_backward_workspace_bytes.restype = sz
        L.wkv_strerror.argtypes = [i32]
        L.wkv_strerror.restype = ctypes.c_char_p
        L.wkv_last_cuda_error.argtypes = []
        L.wkv_last_cuda_error.restype = ctypes.c_char_p
        L.wkv_abi_version.argtypes = []
        L.wkv_abi_version.restype = i32
        _lib = L
        return L


# ---------------------------------------------------------------------------
# torch front end (plumbing only)
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return WKV_F32
    if t.dtype == torch.bfloat16:
        return WKV_BF16
    raise TypeError(f"k/v/r/y must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_ptr(stream, device=None):
    """cudaStream_t of `stream`, or of the current stream of `device`."""
    torch = _torch()
    if stream is not None:
        return stream.cuda_stream
    idx = device.index if device is not None and device.index is not None else torch.cuda.current_device()
    return torch._C._cuda_getCurrentRawStream(idx)


def _check(status, where):
    if status != 0:
        raise WkvError(status, where)


def _need(t, name, shape, dtype, device):
    if t is None:
        return
    if t.shape == shape and t.dtype == dtype and t.device == device and t.is_contiguous():
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


class Workspace:
    """Device scratch for wkv_forward's cross-block exchange, grown on demand.

    Zeroed once per allocation (wkv_workspace_init); afterwards calls reuse it
    without clearing.  Calls that share one Workspace must be ordered on the
    GPU (the default: the current stream)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int, stream=None):
        torch = _torch()
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            dev = self.device if self.device is not None else torch.device("cuda", torch.cuda.current_device())
            self.buf = torch.empty(int(nbytes) + 256, dtype=torch.uint8, device=dev)
            _check(lib().wkv_workspace_init(self._aligned_ptr(), self.buf.numel() - 256, _stream_ptr(stream, self.buf.device)),
                   "wkv_workspace_init")
        return self._aligned_ptr(), self.buf.numel() - 256

    def _aligned_ptr(self):
        p = self.buf.data_ptr()
        return (p + 255) & ~255

    def status(self, stream=None) -> int:
        if self.buf is None:
            return 0
        return lib().wkv_workspace_status(self._aligned_ptr(), _stream_ptr(stream, self.buf.device))

    def reset(self, stream=None):
        if self.buf is not None:
            _check(lib().wkv_workspace_init(self._aligned_ptr(), self.buf.numel() - 256, _stream_ptr(stream, self.buf.device)),
                   "wkv_workspace_init")


_workspaces = {}


def default_workspace(device) -> Workspace:
    key = (device.type, device.index)
    ws = _workspaces.get(key)
    if ws is None:
        ws = _workspaces[key] = Workspace(device)
    return ws


@functools.lru_cache(maxsize=1024)
def workspace_bytes(B: int, T: int, C: int, dtype_code: int) -> int:
    return int(lib().wkv_forward_workspace_bytes(B, T, C, dtype_code))


WKV_FLAG_INPUTS_READY = 1
WKV_FLAG_CHAIN_BEGIN = 2
WKV_FLAG_CHAIN_NEXT = 4


def wkv_forward(w, u, k, v, r=None, state_in=None, *, y=None, state_out=None, want_state=True,
                workspace: Workspace = None, use_workspace=True, inputs_ready=False, chain=None, stream=None):
    """Parallel mode over one chunk.  k, v, r: (B, T, C) CUDA tensors (float32
    or bfloat16); w, u: (C,) float32; state_in: (3, B, C) float32 or None.
    Returns (y, state_out) (state_out None if want_state is False and none
    was given).  state_out may be state_in for an in-place update.
    use_workspace=False passes no workspace (the scratch-free schedules).
    inputs_ready=True passes WKV_FLAG_INPUTS_READY: k, v, r, w, u are not
    written by work still running on the stream (see include/wkv.h).
    chain="begin" / "next" passes WKV_FLAG_CHAIN_BEGIN / WKV_FLAG_CHAIN_NEXT
    (a chain of chunk calls carrying one state through the workspace; see
    include/wkv.h): the first call of a chain passes "begin", every later
    one "next" with the previous call's state_out as its state_in."""
    torch = _torch()
    if k.dim() != 3:
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("wkv_forward runs on CUDA tensors only")
    code = _dtype_code(k)
    _need(v, "v", (B, T, C), k.dtype, dev)
    _need(r, "r", (B, T, C), k.dtype, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(u, "u", (C,), torch.float32, dev)
    _need(k, "k", (B, T, C), k.dtype, dev)
    _need(state_in, "state_in", (3, B, C), torch.float32, dev)
    if y is None:
        y = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    _need(y, "y", (B, T, C), k.dtype, dev)
    if state_out is None and want_state:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", (3, B, C), torch.float32, dev)
    sp = _stream_ptr(stream, dev)
    if use_workspace:
        ws = workspace if workspace is not None else default_workspace(dev)
        need = workspace_bytes(B, T, C, code)
        if chain is not None:
            need = max(need, 256 + 16 * B * C)   # the chain's words follow the header
        ws_ptr, ws_bytes = ws.get(need, stream)
    else:
        ws_ptr, ws_bytes = None, 0
    flags = WKV_FLAG_INPUTS_READY if inputs_ready else 0
    if chain is not None:
        if chain not in ("begin", "next"):
            raise ValueError("chain must be None, 'begin' or 'next'")
        flags |= WKV_FLAG_CHAIN_BEGIN if chain == "begin" else WKV_FLAG_CHAIN_NEXT
    if flags:
        _check(lib().wkv_forward_ex(B, T, C, code, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                                    _ptr(y), _ptr(state_out), ws_ptr, ws_bytes, flags, sp),
               "wkv_forward_ex")
    else:
        _check(lib().wkv_forward(B, T, C, code, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                                 _ptr(y), _ptr(state_out), ws_ptr, ws_bytes, sp), "wkv_forward")
    return y, state_out


def wkv_forward_noalloc(w, u, k, v, r=None, state_in=None, *, y, state_out=None, stream=None):
    """wkv_forward without a workspace, for callers that cannot allocate device
    memory: the scratch comes from a fixed array inside the library.  The
    caller supplies every output buffer (y, and state_out if wanted); this
    function allocates nothing.  Raises WkvError(WKV_ERR_SCRATCH) for problems
    larger than the built-in scratch.  Calls must be ordered on the GPU."""
    torch = _torch()
    B, T, C = k.shape
    dev = k.device
    code = _dtype_code(k)
    for t, name in ((v, "v"), (r, "r"), (y, "y")):
        _need(t, name, (B, T, C), k.dtype, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(u, "u", (C,), torch.float32, dev)
    _need(state_in, "state_in", (3, B, C), torch.float32, dev)
    _need(state_out, "state_out", (3, B, C), torch.float32, dev)
    _check(lib().wkv_forward_noalloc(B, T, C, code, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                                     _ptr(y), _ptr(state_out), _stream_ptr(stream, dev)), "wkv_forward_noalloc")
    return y, state_out


def wkv_state(w, k, v, state_in=None, *, state_out=None, workspace: Workspace = None, use_workspace=True,
              stream=None):
    """State after the chunk k, v (B, T, C) entered from state_in (None: the
    empty state), without outputs; from the empty state it is the chunk's
    summary.  Returns state_out (3, B, C) float32 (may be state_in)."""
    torch = _torch()
    if k.dim() != 3:
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("wkv_state runs on CUDA tensors only")
    code = _dtype_code(k)
    _need(v, "v", (B, T, C), k.dtype, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(k, "k", (B, T, C), k.dtype, dev)
    _need(state_in, "state_in", (3, B, C), torch.float32, dev)
    if state_out is None:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", (3, B, C), torch.float32, dev)
    sp = _stream_ptr(stream, dev)
    if use_workspace:
        ws = workspace if workspace is not None else default_workspace(dev)
        ws_ptr, ws_bytes = ws.get(workspace_bytes(B, T, C, code), stream)
    else:
        ws_ptr, ws_bytes = None, 0
    _check(lib().wkv_state(B, T, C, code, _ptr(w), _ptr(k), _ptr(v), _ptr(state_in), _ptr(state_out), ws_ptr,
                           ws_bytes, sp), "wkv_state")
    return state_out


def wkv_state_combine(w, lens, states, state_in=None, *, state_out=None, stream=None):
    """Fold the summaries states (n, 3, B, C) of n consecutive chunks of
    lens[j] tokens into the state entering from state_in (None: empty).
    Returns state_out (3, B, C)."""
    torch = _torch()
    n = len(lens)
    if states.dim() != 4 or states.shape[0] < n or states.shape[1] != 3:
        raise ValueError("states must be (n, 3, B, C)")
    _, _, B, C = states.shape
    dev = states.device
    if dev.type != "cuda":
        raise ValueError("wkv_state_combine runs on CUDA tensors only")
    _need(states, "states", tuple(states.shape), torch.float32, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(state_in, "state_in", (3, B, C), torch.float32, dev)
    if state_out is None:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", (3, B, C), torch.float32, dev)
    arr = (ctypes.c_int64 * max(1, n))(*[int(x) for x in lens])
    _check(lib().wkv_state_combine(B, C, n, _ptr(w), arr, _ptr(states), _ptr(state_in), _ptr(state_out),
                                   _stream_ptr(stream, dev)), "wkv_state_combine")
    return state_out


def wkv5_forward(w, u, r, k, v, H, state_in=None, *, y=None, state_out=None, want_state=True, stream=None):
    """Multi-head matrix-state WKV (v5 / v6).  r, k, v: (B, T, C) float32 or
    bfloat16 CUDA tensors, C = H * N with N in {32, 64}; w: (C,) decay rates
    (v5) or (B, T, C) float32 per token (v6); u: (C,) float32; state_in:
    (B, H, N, N) float32 or None (zeros).  Returns (y, state_out)."""
    torch = _torch()
    if k.dim() != 3:
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    if C % H != 0:
        raise ValueError("C must be a multiple of H")
    N = C // H
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("wkv5_forward runs on CUDA tensors only")
    code = _dtype_code(k)
    for t, name in ((r, "r"), (v, "v"), (k, "k")):
        _need(t, name, (B, T, C), k.dtype, dev)
    per_token = w.dim() == 3
    _need(w, "w", (B, T, C) if per_token else (C,), torch.float32, dev)
    _need(u, "u", (C,), torch.float32, dev)
    _need(state_in, "state_in", (B, H, N, N), torch.float32, dev)
    if y is None:
        y = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    _need(y, "y", (B, T, C), k.dtype, dev)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, N, N), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", (B, H, N, N), torch.float32, dev)
    _check(lib().wkv5_forward(B, T, C, H, code, _ptr(w), int(per_token), _ptr(u), _ptr(r), _ptr(k), _ptr(v),
                              _ptr(state_in), _ptr(y), _ptr(state_out), _stream_ptr(stream, dev)), "wkv5_forward")
    return y, state_out


def wkv_forward_noalloc_status(stream=None, device=None) -> int:
    """Synchronise the stream and return the error word of the library's
    built-in scratch array on the current device: 0, or WKV_ERR_TIMEOUT (-7)
    if the last wkv_forward_noalloc call that used it had a cross-block wait
    give up."""
    return int(lib().wkv_forward_noalloc_status(_stream_ptr(stream, device)))


@functools.lru_cache(maxsize=1024)
def backward_workspace_bytes(B: int, T: int, C: int, dtype_code: int) -> int:
    return int(lib().wkv_backward_workspace_bytes(B, T, C, dtype_code))


def wkv_backward(w, u, k, v, r=None, state_in=None, *, dy, dstate_out=None, dk=None, dv=None, dr=None,
                 dw=None, du=None, dstate_in=None, want_dstate_in=True, workspace: Workspace = None, stream=None):
    """Gradients of wkv_forward.  dy: (B, T, C) like k; dstate_out: (3, B, C)
    float32 dL/d(a, b) of the returned state, or None.  Returns (dk, dv, dr,
    dw, du, dstate_in); dr is None without a gate, dw and du are (C,) float32
    sums over sequences and tokens."""
    torch = _torch()
    B, T, C = k.shape
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("wkv_backward runs on CUDA tensors only")
    code = _dtype_code(k)
    for t, name in ((v, "v"), (r, "r"), (dy, "dy")):
        _need(t, name, (B, T, C), k.dtype, dev)
    _need(w, "w", (C,), torch.float32, dev)
    _need(u, "u", (C,), torch.float32, dev)
    _need(k, "k", (B, T, C), k.dtype, dev)
    _need(state_in, "state_in", (3, B, C), torch.float32, dev)
    _need(dstate_out, "dstate_out", (3, B, C), torch.float32, dev)
    if dk is None:
        dk = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    if dv is None:
        dv = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    if dr is None and r is not None:
        dr = torch.empty((B, T, C), dtype=k.dtype, device=dev)
    if dw is None:
        dw = torch.empty((C,), dtype=torch.float32, device=dev)
    if du is None:
        du = torch.empty((C,), dtype=torch.float32, device=dev)
    if dstate_in is None and want_dstate_in:
        dstate_in = torch.empty((3, B, C), dtype=torch.float32, device=dev)
    for t, name in ((dk, "dk"), (dv, "dv"), (dr, "dr")):
        _need(t, name, (B, T, C), k.dtype, dev)
    _need(dw, "dw", (C,), torch.float32, dev)
    _need(du, "du", (C,), torch.float32, dev)
    _need(dstate_in, "dstate_in", (3, B, C), torch.float32, dev)
    ws = workspace if workspace is not None else default_workspace(dev)
    sp = _stream_ptr(stream, dev)
    ws_ptr, ws_bytes = ws.get(backward_workspace_bytes(B, T, C, code), stream)
    _check(lib().wkv_backward(B, T, C, code, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                              _ptr(dy), _ptr(dstate_out), _ptr(dk), _ptr(dv), _ptr(dr), _ptr(dw), _ptr(du),
                              _ptr(dstate_in), ws_ptr, ws_bytes, sp), "wkv_backward")
    return dk, dv, dr, dw, du, dstate_in


def wkv_token_shift(x, mu, x_prev=None, *, out=None, x_last=None, want_last=True, stream=None):
    """Token shift: x (B, T, C) float32 or bfloat16, mu (nmix, C) float32,
    x_prev (B, C) of x's dtype or None (zeros).  Returns (out, x_last) with
    out[m, b, t] = mu[m] * x[b, t] + (1 - mu[m]) * x[b, t - 1] (nmix, B, T, C)
    and x_last = x[:, T - 1] (B, C), the next call's x_prev; x_last may be
    x_prev for an in-place update."""
    torch = _torch()
    if x.dim() != 3 or mu.dim() != 2:
        raise ValueError("x must be (B, T, C) and mu (nmix, C)")
    B, T, C = x.shape
    nmix = mu.shape[0]
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("wkv_token_shift runs on CUDA tensors only")
    code = _dtype_code(x)
    _need(x, "x", (B, T, C), x.dtype, dev)
    _need(mu, "mu", (nmix, C), torch.float32, dev)
    _need(x_prev, "x_prev", (B, C), x.dtype, dev)
    if out is None:
        out = torch.empty((nmix, B, T, C), dtype=x.dtype, device=dev)
    _need(out, "out", (nmix, B, T, C), x.dtype, dev)
    if x_last is None and want_last:
        x_last = torch.empty((B, C), dtype=x.dtype, device=dev)
    _need(x_last, "x_last", (B, C), x.dtype, dev)
    _check(lib().wkv_token_shift(B, T, C, code, nmix, _ptr(x), _ptr(mu), _ptr(x_prev), _ptr(out), _ptr(x_last),
                                 _stream_ptr(stream, dev)), "wkv_token_shift")
    return out, x_last


def wkv_step(w, u, k, v, state, r=None, *, y=None, stream=None):
    """RNN mode: one token for L layers.  w, u: (L, C) float32; k, v, r:
    (L, B, C); state: (L, 3, B, C) float32, updated in place.  Returns y."""
    torch = _torch()
    if k.dim() != 3:
        raise ValueError("k must be (L, B, C)")
    Lr, B, C = k.shape
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("wkv_step runs on CUDA tensors only")
    code = _dtype_code(k)
    _need(v, "v", (Lr, B, C), k.dtype, dev)
    _need(r, "r", (Lr, B, C), k.dtype, dev)
    _need(w, "w", (Lr, C), torch.float32, dev)
    _need(u, "u", (Lr, C), torch.float32, dev)
    _need(state, "state", (Lr, 3, B, C), torch.float32, dev)
    if y is None:
        y = torch.empty((Lr, B, C), dtype=k.dtype, device=dev)
    _need(y, "y", (Lr, B, C), k.dtype, dev)
    _check(lib().wkv_step(Lr, B, C, code, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state), _ptr(y),
                          _stream_ptr(stream, dev)), "wkv_step")
    return y
