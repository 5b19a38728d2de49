"""Pins of the oracle's reverse mode (oracle.wkv_backward), each independent of
its code: central finite differences of the explicit-sum definition written
here in numpy (fp64), closed forms, and invariants of the definition.

The loss is L = sum(dy * y) + (ga * N_T + gb * D_T) * e^{-p_T}, with p_T held
at the returned state's value: dstate_out = (ga, gb) is dL/d(a_T, b_T) of the
state the forward returns, a_T = N_T e^{-p_T}, b_T = D_T e^{-p_T}.
"""
import numpy as np
import pytest

import oracle


def definition(w, u, k, v, r, s0):
    """y (B, T, C) and (N_T, D_T) straight from the explicit sum of the article
    "RWKVアーキテクチャ徹底解説" (section "コア計算"), with the carried state as one
    more past term a0 e^{p0 - t w}; fp64 throughout, shifted per output."""
    B, T, C = k.shape
    a0, b0, p0 = (s0[0], s0[1], s0[2]) if s0 is not None else (np.zeros((B, C)), np.zeros((B, C)),
                                                               np.full((B, C), -1e300))
    y = np.empty((B, T, C))
    for t in range(T):
        ex_state = p0 - t * w                                  # (B, C)
        ex_past = k[:, :t] - (t - 1 - np.arange(t))[None, :, None] * w   # (B, t, C)
        ex_cur = u + k[:, t]                                   # (B, C)
        m = np.maximum(ex_state, ex_cur)
        if t:
            m = np.maximum(m, ex_past.max(axis=1))
        es, ep, ec = np.exp(ex_state - m), np.exp(ex_past - m[:, None]), np.exp(ex_cur - m)
        num = a0 * es + (ep * v[:, :t]).sum(axis=1) + ec * v[:, t]
        den = b0 * es + ep.sum(axis=1) + ec
        g = 1.0 / (1.0 + np.exp(-r[:, t])) if r is not None else 1.0
        y[:, t] = g * num / den
    ex = k - (T - 1 - np.arange(T))[None, :, None] * w        # (B, T, C)
    N = a0 * np.exp(p0 - T * w) + (np.exp(ex) * v).sum(axis=1)
    D = b0 * np.exp(p0 - T * w) + np.exp(ex).sum(axis=1)
    return y, N, D


def loss(params, dy, ds, pT):
    y, N, D = definition(*params)
    L = float((dy * y).sum())
    if ds is not None:
        L += float(((ds[0] * N + ds[1] * D) * np.exp(-pT)).sum())
    return L


def make(B, T, C, gate, state, seed, k_std=1.0, decay=(-3.0, 1.0)):
    g = np.random.default_rng(seed)
    f32 = lambda x: np.asarray(x, np.float32)
    w = f32(np.exp(g.uniform(*decay, C)))
    u = f32(g.normal(0, 1, C))
    k = f32(g.normal(0, k_std, (B, T, C)))
    v = f32(g.normal(0, 1, (B, T, C)))
    r = f32(g.normal(0, 1, (B, T, C))) if gate else None
    s0 = None
    if state:
        p = g.uniform(-5, 5, (B, C))
        b = g.uniform(0.5, 1.5, (B, C))
        s0 = np.stack([b * g.normal(0, 1, (B, C)), b, p])
    dy = g.normal(0, 1, (B, T, C))
    return w, u, k, v, r, s0, dy


def finite_difference(params, dy, ds, pT, h=1e-5):
    """Central differences of the loss in every input element, fp64."""
    grads = []
    for i, x in enumerate(params):
        if x is None:
            grads.append(None)
            continue
        x = np.asarray(x, np.float64)
        gx = np.empty_like(x)
        for j in np.ndindex(x.shape):
            step = h * max(1.0, abs(x[j]))
            xp, xm = x.copy(), x.copy()
            xp[j] += step
            xm[j] -= step
            pp = list(params)
            pm = list(params)
            pp[i], pm[i] = xp, xm
            gx[j] = (loss(pp, dy, ds, pT) - loss(pm, dy, ds, pT)) / (2 * step)
        grads.append(gx)
    return grads


@pytest.mark.parametrize("gate,state,with_ds,k_std", [
    (False, False, False, 1.0),
    (True, False, False, 1.0),
    (True, True, False, 1.0),
    (True, True, True, 1.0),
    (False, True, True, 4.0),
    (True, False, True, 8.0),
])
def test_backward_matches_finite_differences(gate, state, with_ds, k_std):
    B, T, C = 2, 7, 3
    w, u, k, v, r, s0, dy = make(B, T, C, gate, state, seed=11 + 3 * gate + 5 * state + 7 * with_ds, k_std=k_std)
    _, s_out = oracle.wkv_forward(w, u, k, v, r, s0)
    g = np.random.default_rng(99)
    ds = np.stack([g.normal(0, 1, (B, C)), g.normal(0, 1, (B, C)), g.normal(0, 1, (B, C))]) if with_ds else None
    dk, dv, dr, dw, du, dsi = oracle.wkv_backward(w, u, k, v, r, s0, dy, ds)
    params = [x.astype(np.float64) if x is not None else None for x in (w, u, k, v, r)] + [s0]
    fw, fu, fk, fv, fr, fs = finite_difference(params, dy, ds, s_out[2])
    scale = max(1.0, np.abs(dk).max(), np.abs(dv).max())
    for name, got, ref in [("dw", dw, fw), ("du", du, fu), ("dk", dk, fk), ("dv", dv, fv)]:
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-7 * scale), (name, np.abs(got - ref).max())
    if gate:
        assert np.allclose(dr, fr, rtol=1e-6, atol=1e-7 * scale), np.abs(dr - fr).max()
    if state:
        assert np.allclose(dsi, fs, rtol=1e-6, atol=1e-7 * scale), np.abs(dsi - fs).max()


def test_first_token_closed_form():
    """T = 1 from the empty state: y = g v, so dv = g dy, dr = dy v g (1 - g)
    and nothing else moves."""
    w, u, k, v, r, _, dy = make(2, 1, 5, True, False, seed=3)
    dk, dv, dr, dw, du, ds = oracle.wkv_backward(w, u, k, v, r, None, dy)
    g = 1.0 / (1.0 + np.exp(-r.astype(np.float64)))
    assert np.allclose(dv, g * dy, rtol=1e-14)
    assert np.allclose(dr, dy * v * g * (1 - g), rtol=1e-14)
    assert np.all(np.abs(dk) < 1e-15) and np.all(np.abs(du) < 1e-15) and np.all(np.abs(dw) < 1e-15)
    assert np.all(ds == 0.0)


def test_second_token_does_not_depend_on_w():
    """T = 2 from the empty state: y_1 = (e^{k0} v0 + e^{u+k1} v1) / (e^{k0} +
    e^{u+k1}) has no w in it, so dw = 0."""
    w, u, k, v, _, _, dy = make(3, 2, 4, False, False, seed=5)
    _, _, _, dw, _, _ = oracle.wkv_backward(w, u, k, v, None, None, dy)
    assert np.all(np.abs(dw) < 1e-14)


def test_zero_upstream_gives_zero():
    w, u, k, v, r, s0, dy = make(2, 9, 3, True, True, seed=7)
    out = oracle.wkv_backward(w, u, k, v, r, s0, np.zeros_like(dy), np.zeros((3, 2, 3)))
    for x in out:
        assert np.all(x == 0.0)


def test_linear_in_upstream():
    w, u, k, v, r, s0, dy = make(2, 9, 3, True, True, seed=8)
    ds = np.random.default_rng(1).normal(0, 1, (3, 2, 3))
    a = oracle.wkv_backward(w, u, k, v, r, s0, dy, ds)
    b = oracle.wkv_backward(w, u, k, v, r, s0, 2.5 * dy, 2.5 * ds)
    for x, y in zip(a, b):
        assert np.allclose(2.5 * x, y, rtol=1e-12, atol=1e-300)


def test_values_sum_rule():
    """From the empty state without a gate every output is a convex
    combination of the values, so the dv of a lane sum to its dy."""
    w, u, k, v, _, _, dy = make(3, 40, 5, False, False, seed=9, k_std=3.0)
    _, dv, _, _, _, _ = oracle.wkv_backward(w, u, k, v, None, None, dy)
    assert np.allclose(dv.sum(axis=1), dy.sum(axis=1), rtol=1e-10, atol=1e-10)


def test_key_shift_invariance():
    """Shifting every key and the state's p by the same c leaves y unchanged,
    so the key gradients of a lane and its dp0 sum to zero."""
    w, u, k, v, r, s0, dy = make(2, 30, 4, True, True, seed=12, k_std=2.0)
    dk, _, _, _, _, ds = oracle.wkv_backward(w, u, k, v, r, s0, dy)
    total = dk.sum(axis=1) + ds[2]
    assert np.allclose(total, 0.0, atol=1e-9 * max(1.0, np.abs(dk).max()))


def test_chunked_backward_equals_one_pass():
    """Backward over [T1, T) hands dL/d(state at T1) to the backward over
    [0, T1); summed dw, du and the pieces equal one pass over [0, T)."""
    B, T, C, T1 = 2, 50, 3, 23
    w, u, k, v, r, s0, dy = make(B, T, C, True, True, seed=13)
    ds = np.random.default_rng(2).normal(0, 1, (3, B, C))
    full = oracle.wkv_backward(w, u, k, v, r, s0, dy, ds)
    _, s_mid = oracle.wkv_forward(w, u, k[:, :T1], v[:, :T1], r[:, :T1], s0)
    late = oracle.wkv_backward(w, u, k[:, T1:], v[:, T1:], r[:, T1:], s_mid, dy[:, T1:], ds)
    early = oracle.wkv_backward(w, u, k[:, :T1], v[:, :T1], r[:, :T1], s0, dy[:, :T1], late[5])
    for i in range(3):
        assert np.allclose(np.concatenate([early[i], late[i]], axis=1), full[i], rtol=1e-9, atol=1e-12)
    for i in (3, 4):
        assert np.allclose(early[i] + late[i], full[i], rtol=1e-9, atol=1e-12)
    assert np.allclose(early[5], full[5], rtol=1e-9, atol=1e-12)


def test_instant_decay_keeps_two_tokens():
    """w huge (decay +20): only the previous token survives, so dk of token
    t-2 and earlier gets nothing from output t; checked through dv: with
    dy only on the last output, dv vanishes except on the last two tokens."""
    B, T, C = 1, 8, 3
    w, u, k, v, _, _, _ = make(B, T, C, False, False, seed=14, decay=(20.0, 20.0))
    dy = np.zeros((B, T, C))
    dy[:, -1] = 1.0
    _, dv, _, _, _, _ = oracle.wkv_backward(w, u, k, v, None, None, dy)
    assert np.all(np.abs(dv[:, :-2]) == 0.0)
    assert np.all(np.abs(dv[:, -2:]) > 0.0)
