"""Helpers that compare the CUDA path with the fp64 oracle on identical inputs.

Error metric: for every output, |y_gpu - y_oracle| / s, where s is the
oracle's magnitude scale of that output (sigmoid(r) times the weighted mean of
|v| under the same weights; |y| <= s always).  It is the relative error of a
weighted average measured against the size of what is averaged, so it stays
meaningful where y itself crosses zero.  The tolerances are 2e-5 for float32
inputs and outputs, 1e-2 for bfloat16 inputs and outputs with float32 state
(the bfloat16 output rounding alone is up to 2^-9 of |y|).
"""
import numpy as np
import torch

import oracle

TOL = {torch.float32: 2e-5, torch.bfloat16: 1e-2}


def to_np32(t):
    return None if t is None else t.detach().to("cpu", torch.float32).numpy()


def to_np64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def oracle_forward(w, u, k, v, r=None, s0=None, nthreads=0):
    """Oracle on the exact values the GPU saw (bf16 widened exactly to f32)."""
    return oracle.wkv_forward(to_np32(w), to_np32(u), to_np32(k), to_np32(v), to_np32(r), to_np64(s0),
                              want_scale=True, nthreads=nthreads)


def output_error(y_gpu, y_ref, scale):
    y = to_np64(y_gpu)
    assert y.shape == y_ref.shape
    if y.size == 0:
        return 0.0
    assert np.all(np.isfinite(y)), "non-finite output"
    return float(np.max(np.abs(y - y_ref) / scale))


def plain_relative_error(y_gpu, y_ref, scale, floor=1e-3):
    """The plain relative error |y - y_ref| / |y_ref| over the outputs with
    |y_ref| >= floor * scale (elsewhere y_ref is near a cancellation and the
    plain ratio says nothing), and how many outputs that covers.  It is at
    most the scale-relative error divided by `floor`."""
    y = to_np64(y_gpu)
    keep = np.abs(y_ref) >= floor * scale
    if not np.any(keep):
        return 0.0, 0
    return float(np.max(np.abs(y - y_ref)[keep] / np.abs(y_ref)[keep])), int(keep.sum())


def state_error(s_gpu, s_ref):
    """Errors of the state's represented quantities: ratio N/D (against the
    scale 1 + |N/D|) and log D, and of the running-max exponent p
    (against max(1, |p|))."""
    s = to_np64(s_gpu)
    a, b, p = s[0], s[1], s[2]
    ra, rb, rp = s_ref[0], s_ref[1], s_ref[2]
    assert np.all(np.isfinite(s)), "non-finite state"
    ratio = np.max(np.abs(a / b - ra / rb) / (1.0 + np.abs(ra / rb)))
    logd = np.max(np.abs((np.log(b) + p) - (np.log(rb) + rp)) / np.maximum(1.0, np.abs(np.log(rb) + rp)))
    pe = np.max(np.abs(p - rp) / np.maximum(1.0, np.abs(rp)))
    return float(ratio), float(logd), float(pe)


def sample_channels(C, n=48, seed=0):
    """Channels to check on full-size runs: both ends, around the channel
    block edges of the kernels (multiples of 32 and 64), and random ones."""
    g = np.random.default_rng(seed)
    fixed = [0, 1, 31, 32, 33, 63, 64, 65, 127, 128, C - 2, C - 1]
    rand = g.choice(C, size=max(0, n - len(fixed)), replace=False)
    idx = sorted(set(int(c) for c in fixed + list(rand) if 0 <= c < C))
    return torch.tensor(idx, dtype=torch.long)


def argmax_index(k, w, T, p0=None):
    """Index j of the term that sets the running max after T tokens:
    argmax over j of k_j - (T-1-j) w, with j = -1 standing for the initial
    state (p0 - T w).  Also returns the gap to the runner-up."""
    k64 = k.astype(np.float64)          # (B, T, C)
    w64 = w.astype(np.float64)[None, None, :]
    cand = k64 - (T - 1 - np.arange(T))[None, :, None] * w64
    if p0 is not None:
        init = (p0 - T * w.astype(np.float64)[None, :])[:, None, :]
        cand = np.concatenate([init, cand], axis=1)
        off = 1
    else:
        off = 0
    order = np.sort(cand, axis=1)
    gap = order[:, -1, :] - order[:, -2, :] if cand.shape[1] > 1 else np.full(order[:, -1, :].shape, np.inf)
    return np.argmax(cand, axis=1) - off, gap, cand


def gpu_argmax_index(p_gpu, cand, off):
    """Index of the candidate exponent closest to the GPU's final p."""
    return np.argmin(np.abs(cand - p_gpu[:, None, :]), axis=1) - off
