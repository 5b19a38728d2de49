"""Pins of the multi-head matrix-state WKV oracle (v5 / v6), each something
other than the oracle itself:

- hand-worked exact values (tests/golden/wkv5_hand_worked.json, derivations
  in the file);
- reduction to the v4 operator: one channel per head, keys e^k, bonus e^u and
  r = 1 give the v4 sum's numerator, and with v = 1 its denominator; their
  ratio must equal the v4 oracle (itself pinned by its own hand-worked
  values), which fixes the decay exponent of each past token, the position
  of the bonus and the output-before-update order;
- brute force: the explicit sum over past tokens with the products of decay
  factors, written out here in numpy, on tiny random inputs (v5 and v6);
- closed forms: instant decay keeps only the previous token;
- invariants: chunked = one pass (bit-exact), v6 with a decay constant in time
  = v5, heads independent, linear in v and in r, |y| <= yscale;
- negative control: the order "decay, then output" fails the pins above.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "wkv5_hand_worked.json")


def rand_case(B, T, H, N, v6=False, seed=0, state=True):
    g = np.random.default_rng(seed)
    C = H * N
    w = (g.uniform(0.0, 2.0, (B, T, C)) if v6 else g.uniform(0.0, 2.0, C)).astype(np.float32)
    u = g.normal(0, 1, C).astype(np.float32)
    k, v, r = (g.normal(0, 1, (B, T, C)).astype(np.float32) for _ in range(3))
    s0 = g.normal(0, 1, (B, H, N, N)) if state else None
    return w, u, k, v, r, s0


def brute(w, u, k, v, r, H, s0=None):
    """y_t[j] = sum_i r_t[i] ( P(0,t)[i] S0[i][j] + sum_{s<t} P(s+1,t)[i] k_s[i] v_s[j]
    + u[i] k_t[i] v_t[j] ), P(a,t)[i] = prod_{m=a}^{t-1} e^{-w_m[i]}."""
    B, T, C = k.shape
    N = C // H
    k, v, r, u = (x.astype(np.float64) for x in (k, v, r, u))
    wt = np.broadcast_to(w.astype(np.float64), (B, T, C))
    y = np.zeros((B, T, C))
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            for t in range(T):
                acc = np.zeros(N)
                for i in range(N):
                    ci = h * N + i
                    tot = np.zeros(N)
                    if s0 is not None:
                        tot += np.exp(-wt[b, :t, ci].sum()) * s0[b, h, i]
                    for s in range(t):
                        tot += np.exp(-wt[b, s + 1:t, ci].sum()) * k[b, s, ci] * v[b, s, sl]
                    tot += u[ci] * k[b, t, ci] * v[b, t, sl]
                    acc += r[b, t, ci] * tot
                y[b, t, sl] = acc
    return y


def test_hand_worked_values():
    d = json.load(open(GOLDEN))
    assert len(d["cases"]) == 3
    for c in d["cases"]:
        f = lambda x: np.array(x, np.float32)[None]
        w = np.array(c["w"], np.float32)
        w = w if w.ndim == 1 else w[None]
        s0 = None if c["state_in"] is None else np.array(c["state_in"], np.float64)[None, None]
        y, s = oracle.wkv5_forward(w, np.array(c["u"], np.float32), f(c["k"]), f(c["v"]), f(c["r"]), c["H"], s0)
        np.testing.assert_allclose(y[0], np.array(c["y"]), rtol=1e-6, atol=1e-6, err_msg=c["name"])
        np.testing.assert_allclose(s[0, 0], np.array(c["state_out"]), rtol=1e-6, atol=1e-6, err_msg=c["name"])


@pytest.mark.parametrize("with_state", [False, True])
def test_reduces_to_v4_with_one_channel_per_head(with_state):
    g = np.random.default_rng(11)
    B, T, C = 2, 40, 5
    w = np.exp(g.uniform(-3, 1, C)).astype(np.float32)
    u4 = g.normal(0, 1, C).astype(np.float32)
    k4 = g.normal(0, 1, (B, T, C)).astype(np.float32)
    v = g.normal(0, 1, (B, T, C)).astype(np.float32)
    s4 = None
    s_num = s_den = None
    if with_state:
        p0 = g.uniform(-2, 2, (B, C))
        b0 = g.uniform(0.5, 1.5, (B, C))
        a0 = b0 * g.normal(0, 1, (B, C))
        s4 = np.stack([a0, b0, p0])
        s_num = (a0 * np.exp(p0)).reshape(B, C, 1, 1)
        s_den = (b0 * np.exp(p0)).reshape(B, C, 1, 1)
    ek, eu = np.exp(k4.astype(np.float64)).astype(np.float32), np.exp(u4.astype(np.float64)).astype(np.float32)
    one = np.ones((B, T, C), np.float32)
    num, _ = oracle.wkv5_forward(w, eu, ek, v, one, C, s_num)
    den, _ = oracle.wkv5_forward(w, eu, ek, one, one, C, s_den)
    y4, _ = oracle.wkv_forward(w, u4, k4, v, None, s4)
    # float32 rounding of e^k and e^u: ~1e-7 relative
    np.testing.assert_allclose(num / den, y4, rtol=2e-6, atol=2e-6)


@pytest.mark.parametrize("v6", [False, True])
def test_brute_force(v6):
    w, u, k, v, r, s0 = rand_case(2, 9, 2, 3, v6=v6, seed=3 + v6)
    y, _ = oracle.wkv5_forward(w, u, k, v, r, 2, s0)
    np.testing.assert_allclose(y, brute(w, u, k, v, r, 2, s0), rtol=1e-11, atol=1e-11)
    y0, _ = oracle.wkv5_forward(w, u, k, v, r, 2, None)
    np.testing.assert_allclose(y0, brute(w, u, k, v, r, 2, None), rtol=1e-11, atol=1e-11)


def test_instant_decay_keeps_the_previous_token():
    w, u, k, v, r, _ = rand_case(1, 6, 1, 4, seed=5, state=False)
    w = np.full_like(w, 1000.0)       # e^{-1000} = 0 in fp64
    y, _ = oracle.wkv5_forward(w, u, k, v, r, 1)
    k64, v64, r64 = (x[0].astype(np.float64) for x in (k, v, r))
    for t in range(6):
        prev = np.outer(k64[t - 1], v64[t - 1]) if t > 0 else 0.0
        expect = r64[t] @ (prev + np.outer(u.astype(np.float64) * k64[t], v64[t]))
        np.testing.assert_allclose(y[0, t], expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("v6", [False, True])
def test_chunked_equals_one_pass(v6):
    w, u, k, v, r, s0 = rand_case(2, 50, 3, 4, v6=v6, seed=7)
    y, s = oracle.wkv5_forward(w, u, k, v, r, 3, s0)
    st, ys = s0, []
    for a, b in [(0, 1), (1, 17), (17, 17), (17, 50)]:
        c = lambda x: np.ascontiguousarray(x[:, a:b])
        yy, st = oracle.wkv5_forward(c(w) if v6 else w, u, c(k), c(v), c(r), 3, st)
        ys.append(yy)
    assert np.array_equal(np.concatenate(ys, axis=1), y)
    assert np.array_equal(st, s)


def test_v6_with_constant_decay_is_v5():
    w, u, k, v, r, s0 = rand_case(2, 20, 2, 4, seed=9)
    y5, s5 = oracle.wkv5_forward(w, u, k, v, r, 2, s0)
    y6, s6 = oracle.wkv5_forward(np.ascontiguousarray(np.broadcast_to(w, k.shape)), u, k, v, r, 2, s0)
    assert np.array_equal(y5, y6) and np.array_equal(s5, s6)


def test_heads_are_independent():
    w, u, k, v, r, s0 = rand_case(1, 12, 3, 4, seed=13)
    y, s = oracle.wkv5_forward(w, u, k, v, r, 3, s0)
    k2 = k.copy()
    k2[..., 4:8] = 7.0                 # head 1 only
    y2, s2 = oracle.wkv5_forward(w, u, k2, v, r, 3, s0)
    assert np.array_equal(y[..., :4], y2[..., :4]) and np.array_equal(y[..., 8:], y2[..., 8:])
    assert np.array_equal(s[:, 0], s2[:, 0]) and np.array_equal(s[:, 2], s2[:, 2])
    assert not np.allclose(y[..., 4:8], y2[..., 4:8])


def test_linear_in_v_and_r():
    w, u, k, v, r, _ = rand_case(1, 15, 2, 3, seed=17, state=False)
    g = np.random.default_rng(1)
    v2, r2 = g.normal(0, 1, v.shape).astype(np.float32), g.normal(0, 1, r.shape).astype(np.float32)
    y = lambda vv, rr: oracle.wkv5_forward(w, u, k, vv, rr, 2)[0]
    np.testing.assert_allclose(y(v + v2, r), y(v, r) + y(v2, r), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(y(v, r + r2), y(v, r) + y(v, r2), rtol=1e-6, atol=1e-9)


def test_scale_bounds_the_output():
    w, u, k, v, r, s0 = rand_case(2, 30, 2, 4, v6=True, seed=19)
    y, _, ys = oracle.wkv5_forward(w, u, k, v, r, 2, s0, want_scale=True)
    assert np.all(np.abs(y) <= ys * (1 + 1e-12))
    pos = lambda x: np.abs(x).astype(np.float32)
    yp, _, ysp = oracle.wkv5_forward(w, np.abs(u), pos(k), pos(v), pos(r), 2, np.abs(s0), want_scale=True)
    np.testing.assert_allclose(yp, ysp, rtol=1e-12)


def decay_first(w, u, k, v, r, H, s0=None):
    """A plausible mistake planted in a copy of the recurrence: the state is
    decayed and the token added before the output is read."""
    B, T, C = k.shape
    N = C // H
    wt = np.broadcast_to(w.astype(np.float64), (B, T, C))
    y = np.zeros((B, T, C))
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            S = np.zeros((N, N)) if s0 is None else s0[b, h].copy()
            for t in range(T):
                S = np.exp(-wt[b, t, sl])[:, None] * S + np.outer(k[b, t, sl], v[b, t, sl])
                y[b, t, sl] = r[b, t, sl] @ (S + np.outer(u[sl] * k[b, t, sl], v[b, t, sl]))
    return y


def test_planted_order_mistake_is_caught():
    d = json.load(open(GOLDEN))
    c = d["cases"][0]
    f = lambda x: np.array(x, np.float32)[None]
    y_bad = decay_first(np.array(c["w"], np.float32), np.array(c["u"], np.float32), f(c["k"]), f(c["v"]),
                        f(c["r"]), 1)
    assert not np.allclose(y_bad[0], np.array(c["y"]), atol=1e-3)
    w, u, k, v, r, _ = rand_case(1, 8, 2, 3, seed=23, state=False)
    assert not np.allclose(decay_first(w, u, k, v, r, 2), brute(w, u, k, v, r, 2), atol=1e-3)
