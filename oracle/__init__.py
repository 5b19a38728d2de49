"""fp64 CPU oracle for the RWKV-4 WKV operator (ctypes front end of wkv_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never import it; the two share no code.

Every function takes numpy arrays in the layouts of the C ABI:
k, v, r: (B, T, C) float32 (bf16 inputs are widened to float32 by the caller,
which is exact); w, u: (C,) float32; state: (3, B, C) float64 = {a, b, p}.
Results are float64.  See wkv_oracle.c for the passages each function follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

FRESH_P = -1e38

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, p, i32, d = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_wkv_brute.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, p, i32]
        L.oracle_wkv_forward.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, p, p, i32]
        L.oracle_wkv_step.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, i32]
        L.oracle_wkv_summary.argtypes = [d, i64, p, p, p]
        L.oracle_wkv_combine.argtypes = [d, d, d, d, d, d, d, i64, p]
        L.oracle_wkv_backward.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, p, p, p, p, p, p, p, i32]
        L.oracle_token_shift.argtypes = [i64, i64, i64, i64, p, p, p, p, p]
        L.oracle_wkv5_forward.argtypes = [i64, i64, i64, i64, i32, p, p, p, p, p, p, p, p, p]
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _f32(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _check_forward_args(k, w, u, v, r, state_in):
    if k.ndim != 3:
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    if v.shape != k.shape or (r is not None and r.shape != k.shape):
        raise ValueError("k, v, r must share one (B, T, C) shape")
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be (C,)")
    if state_in is not None and state_in.shape != (3, B, C):
        raise ValueError("state must be (3, B, C)")
    return B, T, C


def wkv_brute(w, u, k, v, r=None, state_in=None, want_scale=False, nthreads=0):
    """Explicit-sum definition, O(T^2) per lane.  Returns y (and yscale)."""
    w, u, k, v, r, state_in = _f32(w), _f32(u), _f32(k), _f32(v), _f32(r), _f64(state_in)
    B, T, C = _check_forward_args(k, w, u, v, r, state_in)
    y = np.empty((B, T, C), np.float64)
    ys = np.empty((B, T, C), np.float64) if want_scale else None
    lib().oracle_wkv_brute(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                           _ptr(state_in), _ptr(y), _ptr(ys), int(nthreads))
    return (y, ys) if want_scale else y


def wkv_forward(w, u, k, v, r=None, state_in=None, want_scale=False, nthreads=0):
    """Log-space recurrence over one chunk.  Returns (y, state_out[, yscale])."""
    w, u, k, v, r, state_in = _f32(w), _f32(u), _f32(k), _f32(v), _f32(r), _f64(state_in)
    B, T, C = _check_forward_args(k, w, u, v, r, state_in)
    y = np.empty((B, T, C), np.float64)
    ys = np.empty((B, T, C), np.float64) if want_scale else None
    st = np.empty((3, B, C), np.float64)
    lib().oracle_wkv_forward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                             _ptr(state_in), _ptr(y), _ptr(ys), _ptr(st), int(nthreads))
    return (y, st, ys) if want_scale else (y, st)


def wkv_step(w, u, k, v, state, r=None, nthreads=0):
    """One decode token for L layers.  w, u: (L, C); k, v, r: (L, B, C);
    state: (L, 3, B, C) float64, updated IN PLACE.  Returns y (L, B, C)."""
    w, u, k, v, r = _f32(w), _f32(u), _f32(k), _f32(v), _f32(r)
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64 and state.flags.c_contiguous):
        raise ValueError("state must be a C-contiguous float64 array (updated in place)")
    Lr, B, C = k.shape
    if state.shape != (Lr, 3, B, C) or w.shape != (Lr, C) or u.shape != (Lr, C):
        raise ValueError("shape mismatch")
    y = np.empty((Lr, B, C), np.float64)
    lib().oracle_wkv_step(Lr, B, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                          _ptr(state), _ptr(y), int(nthreads))
    return y


def wkv_backward(w, u, k, v, r=None, state_in=None, dy=None, dstate_out=None, nthreads=0):
    """Gradients of wkv_forward: given dy (B, T, C) and dstate_out (3, B, C)
    (dL/d(a, b) of the returned state; its p plane is not read), returns
    (dk, dv, dr, dw, du, dstate_in) as float64; dr is None without a gate,
    dw and du are (C,) sums over sequences and tokens, dstate_in is
    dL/d(a0, b0, p0) of state_in (zeros for the empty state)."""
    w, u, k, v, r, state_in = _f32(w), _f32(u), _f32(k), _f32(v), _f32(r), _f64(state_in)
    B, T, C = _check_forward_args(k, w, u, v, r, state_in)
    dy, dstate_out = _f64(dy), _f64(dstate_out)
    if dy is None or dy.shape != (B, T, C):
        raise ValueError("dy must be (B, T, C)")
    if dstate_out is not None and dstate_out.shape != (3, B, C):
        raise ValueError("dstate_out must be (3, B, C)")
    dk = np.empty((B, T, C), np.float64)
    dv = np.empty((B, T, C), np.float64)
    dr = np.empty((B, T, C), np.float64) if r is not None else None
    dw = np.empty(C, np.float64)
    du = np.empty(C, np.float64)
    ds = np.empty((3, B, C), np.float64)
    lib().oracle_wkv_backward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                              _ptr(dy), _ptr(dstate_out), _ptr(dk), _ptr(dv), _ptr(dr), _ptr(dw), _ptr(du),
                              _ptr(ds), int(nthreads))
    return dk, dv, dr, dw, du, ds


def token_shift(x, mu, x_prev=None):
    """Token shift: x (B, T, C), mu (nmix, C), x_prev (B, C) or None (zeros).
    Returns (out (nmix, B, T, C), x_last (B, C)) as float64, where
    out[m, b, t] = mu[m] * x[b, t] + (1 - mu[m]) * x[b, t - 1] and x[b, -1] is
    x_prev[b]; x_last is the input the next call mixes its first token with."""
    x, mu, x_prev = _f32(x), _f32(mu), _f32(x_prev)
    if x.ndim != 3 or mu.ndim != 2:
        raise ValueError("x must be (B, T, C) and mu (nmix, C)")
    B, T, C = x.shape
    nmix = mu.shape[0]
    if mu.shape[1] != C or (x_prev is not None and x_prev.shape != (B, C)):
        raise ValueError("shape mismatch")
    out = np.empty((nmix, B, T, C), np.float64)
    last = np.empty((B, C), np.float64)
    lib().oracle_token_shift(B, T, C, nmix, _ptr(x), _ptr(mu), _ptr(x_prev), _ptr(out), _ptr(last))
    return out, last


def wkv5_forward(w, u, k, v, r, H, state_in=None, want_scale=False):
    """Multi-head matrix-state WKV (v5: w of shape (C,); v6: w of shape
    (B, T, C), a decay rate per token).  k, v, r: (B, T, C) with C = H * N;
    u: (C,); state_in: (B, H, N, N) float64 or None (zeros).  Returns
    (y, state_out[, yscale]) in float64; see wkv5_oracle.c."""
    w, u, k, v, r, state_in = _f32(w), _f32(u), _f32(k), _f32(v), _f32(r), _f64(state_in)
    if k.ndim != 3 or v.shape != k.shape or r.shape != k.shape:
        raise ValueError("k, v, r must share one (B, T, C) shape")
    B, T, C = k.shape
    if C % H != 0:
        raise ValueError("C must be a multiple of H")
    N = C // H
    wmode = 0 if w.shape == (C,) else 1
    if wmode == 1 and w.shape != (B, T, C):
        raise ValueError("w must be (C,) or (B, T, C)")
    if u.shape != (C,):
        raise ValueError("u must be (C,)")
    if state_in is not None and state_in.shape != (B, H, N, N):
        raise ValueError("state must be (B, H, N, N)")
    y = np.empty((B, T, C), np.float64)
    ys = np.empty((B, T, C), np.float64) if want_scale else None
    st = np.empty((B, H, N, N), np.float64)
    lib().oracle_wkv5_forward(B, T, H, N, wmode, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(state_in),
                              _ptr(y), _ptr(ys), _ptr(st))
    return (y, st, ys) if want_scale else (y, st)


def fresh_state(B, C):
    """The empty state (0, 0, -1e38) as a (3, B, C) float64 array."""
    s = np.zeros((3, B, C), np.float64)
    s[2] = FRESH_P
    return s


def summary(w, k, v):
    """(q, A, Bd) of one lane's segment started from the empty state."""
    k, v = _f64(k), _f64(v)
    out = np.empty(3, np.float64)
    lib().oracle_wkv_summary(float(w), len(k), _ptr(k), _ptr(v), _ptr(out))
    return out


def combine(w, s, seg, n):
    """State after a segment of length n with summary seg=(q, A, Bd), from s=(p, a, b)."""
    out = np.empty(3, np.float64)
    lib().oracle_wkv_combine(float(w), float(s[0]), float(s[1]), float(s[2]),
                             float(seg[0]), float(seg[1]), float(seg[2]), int(n), _ptr(out))
    return out


def represented(state):
    """(log|N|, sign N, log D) of a (3, ...) state {a, b, p}: the quantities a
    state stands for, independent of how it is scaled."""
    a, b, p = state[0], state[1], state[2]
    with np.errstate(divide="ignore"):
        return np.log(np.abs(a)) + p, np.sign(a), np.log(b) + p
