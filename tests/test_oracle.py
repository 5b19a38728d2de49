"""Pins for the fp64 CPU oracle, independent of the oracle's own formulas.

Each test fixes the oracle to something other than itself: hand-derived exact
values of the explicit-sum definition (tests/golden), closed forms, limits that
reduce the operator to a textbook quantity, invariances of the definition, and
the brute-force O(T^2) sum on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
rng = np.random.default_rng(12345)


def lane_arrays(case):
    k = np.array(case["k"], np.float32).reshape(1, -1, 1)
    v = np.array(case["v"], np.float32).reshape(1, -1, 1)
    r = None if case["r"] is None else np.array(case["r"], np.float32).reshape(1, -1, 1)
    w = np.array([case["w"]], np.float32)
    u = np.array([case["u"]], np.float32)
    s0 = None
    if case["state_in"] is not None:
        s0 = np.array(case["state_in"], np.float64).astype(np.float32).astype(np.float64).reshape(3, 1, 1)
    return w, u, k, v, r, s0


def rand_case(B, T, C, gate, random_state, k_std=1.0, decay=(-3.0, 1.0), u_std=1.0):
    w = np.exp(rng.uniform(*decay, size=C)).astype(np.float32)
    u = (rng.standard_normal(C) * u_std).astype(np.float32)
    k = (rng.standard_normal((B, T, C)) * k_std).astype(np.float32)
    v = rng.standard_normal((B, T, C)).astype(np.float32)
    r = rng.standard_normal((B, T, C)).astype(np.float32) if gate else None
    s0 = None
    if random_state:
        b = rng.uniform(0.5, 1.5, size=(B, C))
        s0 = np.stack([b * rng.standard_normal((B, C)), b, rng.uniform(-5, 5, size=(B, C))])
        s0 = s0.astype(np.float32).astype(np.float64)
    return w, u, k, v, r, s0


def rel_err(y, ref, scale):
    return float(np.max(np.abs(y - ref) / scale)) if y.size else 0.0


# --------------------------------------------------------------------------
# hand-derived exact values
# --------------------------------------------------------------------------
@pytest.mark.parametrize("idx", range(3))
def test_golden_hand_worked(idx):
    case = json.load(open(GOLDEN))["cases"][idx]
    w, u, k, v, r, s0 = lane_arrays(case)
    exp_y = np.array(case["y"])
    yb = oracle.wkv_brute(w, u, k, v, r, s0)[0, :, 0]
    yf, st = oracle.wkv_forward(w, u, k, v, r, s0)
    np.testing.assert_allclose(yb, exp_y, rtol=2e-6, atol=0)
    np.testing.assert_allclose(yf[0, :, 0], exp_y, rtol=2e-6, atol=0)
    a, b, p = st[:, 0, 0]
    np.testing.assert_allclose(a * math.exp(p), case["N_out"], rtol=2e-6)
    np.testing.assert_allclose(b * math.exp(p), case["D_out"], rtol=2e-6)


# --------------------------------------------------------------------------
# brute force vs recurrence
# --------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,C,gate,rs", [(1, 64, 32, False, False), (2, 37, 5, True, True),
                                           (3, 1, 4, True, True), (1, 200, 3, True, False),
                                           (2, 2, 7, False, True)])
def test_brute_matches_recurrence(B, T, C, gate, rs):
    w, u, k, v, r, s0 = rand_case(B, T, C, gate, rs)
    yb, sb = oracle.wkv_brute(w, u, k, v, r, s0, want_scale=True)
    yf, _, sf = oracle.wkv_forward(w, u, k, v, r, s0, want_scale=True)
    assert rel_err(yf, yb, sb) < 1e-12
    np.testing.assert_allclose(sf, sb, rtol=1e-12)


def test_brute_matches_recurrence_large_keys():
    """Keys up to +-60 and an initial state at p=+-50: nothing overflows."""
    w, u, k, v, r, s0 = rand_case(2, 48, 6, True, True, k_std=25.0)
    k = np.clip(k, -60, 60).astype(np.float32)
    s0[2] = np.where(rng.random(s0[2].shape) < 0.5, 50.0, -50.0)
    yb, sb = oracle.wkv_brute(w, u, k, v, r, s0, want_scale=True)
    yf, st = oracle.wkv_forward(w, u, k, v, r, s0)
    assert np.all(np.isfinite(yb)) and np.all(np.isfinite(yf)) and np.all(np.isfinite(st))
    assert rel_err(yf, yb, sb) < 1e-12


# --------------------------------------------------------------------------
# closed forms and limits
# --------------------------------------------------------------------------
def test_first_token_is_value():
    w, u, k, v, r, _ = rand_case(3, 1, 9, True, False)
    y, _ = oracle.wkv_forward(w, u, k, v, r)
    sig = 1.0 / (1.0 + np.exp(-r.astype(np.float64)))
    np.testing.assert_allclose(y, sig * v, rtol=1e-15)


def test_second_token_ignores_decay():
    w, u, k, v, _, _ = rand_case(2, 2, 6, False, False)
    y1 = oracle.wkv_forward(w, u, k, v)[0]
    y2 = oracle.wkv_forward(w * 7.0, u, k, v)[0]
    np.testing.assert_array_equal(y1[:, 1], y2[:, 1])
    k64, v64, u64 = k.astype(np.float64), v.astype(np.float64), u.astype(np.float64)
    e0, e1 = np.exp(k64[:, 0]), np.exp(u64 + k64[:, 1])
    np.testing.assert_allclose(y1[:, 1], (e0 * v64[:, 0] + e1 * v64[:, 1]) / (e0 + e1), rtol=1e-14)


def test_instant_decay_keeps_two_tokens():
    w, u, k, v, _, _ = rand_case(1, 20, 5, False, False)
    w = np.full_like(w, np.exp(20.0))
    y = oracle.wkv_forward(w, u, k, v)[0][0]
    k64, v64, u64 = k[0].astype(np.float64), v[0].astype(np.float64), u.astype(np.float64)
    ep, ec = np.exp(k64[:-1]), np.exp(u64 + k64[1:])
    np.testing.assert_allclose(y[1:], (ep * v64[:-1] + ec * v64[1:]) / (ep + ec), rtol=1e-13)


def test_huge_bonus_returns_current_value():
    w, u, k, v, _, s0 = rand_case(2, 30, 4, False, True)
    y = oracle.wkv_forward(w, np.full_like(u, 200.0), k, v, None, s0)[0]
    np.testing.assert_allclose(y, v, rtol=1e-12)


def test_negative_bonus_gives_past_mean():
    """With u = -200 the current token drops out and y_t is N/D of the state
    after the first t tokens, which the oracle also returns as a state."""
    w, u, k, v, _, s0 = rand_case(2, 25, 3, False, True)
    um = np.full_like(u, -200.0)
    y = oracle.wkv_forward(w, um, k, v, None, s0)[0]
    for t in (1, 7, 24):
        _, st = oracle.wkv_forward(w, u, k[:, :t], v[:, :t], None, s0)
        np.testing.assert_allclose(y[:, t], st[0] / st[1], rtol=1e-12)


def test_zero_receptance_halves():
    w, u, k, v, _, s0 = rand_case(2, 17, 5, False, True)
    y0 = oracle.wkv_forward(w, u, k, v, None, s0)[0]
    yg = oracle.wkv_forward(w, u, k, v, np.zeros_like(k), s0)[0]
    np.testing.assert_array_equal(yg, 0.5 * y0)


def test_max_convention_closed_form():
    """p after T tokens = max(p0 - T*w, max_i k_i - (T-1-i)*w)."""
    w, u, k, v, _, s0 = rand_case(3, 40, 6, False, True, k_std=3.0)
    _, st = oracle.wkv_forward(w, u, k, v, None, s0)
    T = k.shape[1]
    w64 = w.astype(np.float64)
    cand = k.astype(np.float64) - (T - 1 - np.arange(T))[None, :, None] * w64[None, None, :]
    expect = np.maximum(s0[2] - T * w64[None, :], cand.max(axis=1))
    np.testing.assert_allclose(st[2], expect, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# invariants of the definition
# --------------------------------------------------------------------------
def test_constant_value_is_fixed_point():
    w, u, k, _, _, _ = rand_case(2, 100, 8, False, False, k_std=5.0)
    v = np.full(k.shape, 0.37, np.float32)
    y = oracle.wkv_forward(w, u, k, v)[0]
    np.testing.assert_allclose(y, np.float64(np.float32(0.37)), rtol=4 * 2.0 ** -52 * 8)


def test_affine_in_value():
    w, u, k, v, _, _ = rand_case(2, 60, 5, False, False)
    y = oracle.wkv_forward(w, u, k, v)[0]
    alpha, beta = np.float32(-2.5), np.float32(0.75)
    v2 = (alpha * v + beta).astype(np.float32)
    y2 = oracle.wkv_forward(w, u, k, v2)[0]
    # the map is exact in the inputs actually passed (v2 is float32-rounded)
    yb = oracle.wkv_brute(w, u, k, v2)
    np.testing.assert_allclose(y2, yb, rtol=1e-12)
    np.testing.assert_allclose(y2, alpha * y + beta, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("shift", [50.0, -50.0, 7.0])
def test_key_shift_invariance(shift):
    w, u, k, v, r, s0 = rand_case(2, 50, 6, True, True)
    y = oracle.wkv_forward(w, u, k, v, r, s0)[0]
    k2 = (k.astype(np.float64) + shift).astype(np.float32)
    s2 = s0.copy()
    s2[2] += shift
    y2 = oracle.wkv_forward(w, u, k2, v, r, s2)[0]
    # float32 rounding of k+shift perturbs exponents by <= ulp(60) ~ 4e-6
    np.testing.assert_allclose(y2, y, rtol=5e-5, atol=5e-5)


@pytest.mark.parametrize("kval", [60.0, -60.0])
def test_extreme_constant_keys_stay_finite(kval):
    w, u, _, v, r, _ = rand_case(1, 300, 4, True, False)
    k = np.full(v.shape, kval, np.float32)
    y, st = oracle.wkv_forward(w, u, k, v, r)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(st))
    yb = oracle.wkv_brute(w, u, k, v, r)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-300)


def test_alternating_extreme_keys():
    w, u, _, v, r, _ = rand_case(1, 64, 4, True, False)
    k = np.where(np.arange(64)[None, :, None] % 2 == 0, 60.0, -60.0) * np.ones(v.shape)
    k = k.astype(np.float32)
    yb, sb = oracle.wkv_brute(w, u, k, v, r, want_scale=True)
    yf = oracle.wkv_forward(w, u, k, v, r)[0]
    assert np.all(np.isfinite(yf))
    assert rel_err(yf, yb, sb) < 1e-12


def test_chunked_equals_single_pass_bit_exact():
    """Streaming with a carried state is the same computation as one pass."""
    w, u, k, v, r, s0 = rand_case(2, 97, 5, True, True)
    y, st = oracle.wkv_forward(w, u, k, v, r, s0)
    s = s0
    parts = []
    for a, b in [(0, 10), (10, 11), (11, 64), (64, 97)]:
        yc, s = oracle.wkv_forward(w, u, k[:, a:b], v[:, a:b], r[:, a:b], s)
        parts.append(yc)
    np.testing.assert_array_equal(np.concatenate(parts, axis=1), y)
    np.testing.assert_array_equal(s, st)


def test_rnn_mode_equals_parallel_mode_bit_exact():
    """Step-by-step decode reproduces the parallel pass (the dual modes)."""
    w, u, k, v, r, s0 = rand_case(3, 21, 4, True, True)
    y, st = oracle.wkv_forward(w, u, k, v, r, s0)
    state = s0[None].copy()
    for t in range(k.shape[1]):
        yt = oracle.wkv_step(w[None], u[None], k[None, :, t], v[None, :, t], state, r[None, :, t])
        np.testing.assert_array_equal(yt[0], y[:, t])
    np.testing.assert_array_equal(state[0], st)


def test_step_layers_are_independent():
    Lr, B, C = 3, 2, 5
    w = np.exp(rng.uniform(-3, 1, size=(Lr, C))).astype(np.float32)
    u = rng.standard_normal((Lr, C)).astype(np.float32)
    k, v, r = (rng.standard_normal((Lr, B, C)).astype(np.float32) for _ in range(3))
    state = np.stack([oracle.fresh_state(B, C) for _ in range(Lr)])
    state[:, 0] = rng.standard_normal((Lr, B, C))
    state[:, 1] = 1.0
    state[:, 2] = rng.uniform(-2, 2, size=(Lr, B, C))
    init = state.copy()
    y = oracle.wkv_step(w, u, k, v, state, r)
    for l in range(Lr):
        yl, sl = oracle.wkv_forward(w[l], u[l], k[l][:, None], v[l][:, None], r[l][:, None], init[l])
        np.testing.assert_array_equal(y[l], yl[:, 0])
        np.testing.assert_array_equal(state[l], sl)


def test_forgetting_state_changes_output():
    w, u, k, v, _, s0 = rand_case(1, 30, 4, False, True)
    s0[2] = 3.0
    y1 = oracle.wkv_forward(w, u, k, v, None, s0)[0]
    y2 = oracle.wkv_forward(w, u, k, v, None, None)[0]
    assert np.max(np.abs(y1 - y2)) > 1e-3


def test_scale_bounds_output():
    w, u, k, v, r, s0 = rand_case(2, 40, 6, True, True)
    y, _, s = oracle.wkv_forward(w, u, k, v, r, s0, want_scale=True)
    assert np.all(np.abs(y) <= s * (1 + 1e-12))
    vp = np.abs(v)
    s0p = s0.copy()
    s0p[0] = np.abs(s0p[0])
    yp, _, sp = oracle.wkv_forward(w, u, k, vp, None, s0p, want_scale=True)
    np.testing.assert_allclose(yp, sp, rtol=1e-13)


# --------------------------------------------------------------------------
# scan algebra (segment summaries)
# --------------------------------------------------------------------------
def test_summary_is_recurrence_state():
    w = 0.3
    kk, vv = rng.standard_normal(17) * 2, rng.standard_normal(17)
    s = oracle.summary(w, kk, vv)
    _, st = oracle.wkv_forward(np.float32([w]), np.float32([0.0]), kk.astype(np.float32).reshape(1, -1, 1),
                               vv.astype(np.float32).reshape(1, -1, 1))
    # summary takes float64 keys; compare on represented quantities
    np.testing.assert_allclose(s[1] * np.exp(s[0]), st[0, 0, 0] * np.exp(st[2, 0, 0]), rtol=1e-6)


def test_combine_matches_sequential_and_is_associative():
    w = 0.41
    n1, n2, n3 = 9, 4, 13
    kk = rng.standard_normal(n1 + n2 + n3) * 3
    vv = rng.standard_normal(n1 + n2 + n3)
    start = np.array([1.5, -0.7, 2.0])      # (p, a, b)
    x = oracle.summary(w, kk[:n1], vv[:n1])
    y = oracle.summary(w, kk[n1:n1 + n2], vv[n1:n1 + n2])
    z = oracle.summary(w, kk[n1 + n2:], vv[n1 + n2:])
    xy = oracle.summary(w, kk[:n1 + n2], vv[:n1 + n2])
    # sequential reference: run the recurrence on the whole thing from start
    seq = np.array([start[1], start[2], start[0]])
    for i in range(n1 + n2 + n3):
        _, st = oracle.wkv_forward(np.float32([w]), np.float32([0.0]),
                                   np.float32([[[kk[i]]]]), np.float32([[[vv[i]]]]), None,
                                   np.array(seq).reshape(3, 1, 1))
        seq = st[:, 0, 0]
    left = oracle.combine(w, oracle.combine(w, oracle.combine(w, start, x, n1), y, n2), z, n3)
    x_yz = oracle.combine(w, start, oracle.combine(w, x, oracle.combine(w, y, z, n3), n2 + n3), n1 + n2 + n3)
    xy_z = oracle.combine(w, oracle.combine(w, start, xy, n1 + n2), z, n3)
    for res in (left, x_yz, xy_z):
        # k in float32 for the sequential path differs by rounding only
        np.testing.assert_allclose(res[1] * np.exp(res[0] - seq[2]), seq[0], rtol=1e-5)
        np.testing.assert_allclose(res[2] * np.exp(res[0] - seq[2]), seq[1], rtol=1e-5)
    np.testing.assert_allclose(left, x_yz, rtol=1e-12)
    np.testing.assert_allclose(left, xy_z, rtol=1e-12)


# --------------------------------------------------------------------------
# reading of the recurrent form printed with an extra decay on the output
# --------------------------------------------------------------------------
def extra_decay_form(w, u, k, v):
    """The output form printed under 'リカレント定式化': the previous state is
    decayed once more before the output.  Pure-Python loops, one lane."""
    a = b = 0.0
    p = -1e38
    out = []
    for kt, vt in zip(k, v):
        lp = p - w
        o = max(lp, u + kt)
        e1, e2 = math.exp(lp - o), math.exp(u + kt - o)
        out.append((e1 * a + e2 * vt) / (e1 * b + e2))
        q = max(lp, kt)
        a = math.exp(lp - q) * a + math.exp(kt - q) * vt
        b = math.exp(lp - q) * b + math.exp(kt - q)
        p = q
    return np.array(out)


def test_extra_decay_form_is_not_the_definition():
    """The definition fixes the printed output form with the extra e^-w as a
    misprint: it disagrees with the explicit sum as soon as the past matters,
    and agrees with it exactly when the bonus is shifted by w."""
    w, u, k, v, _, _ = rand_case(1, 24, 1, False, False)
    wc, uc = float(w[0]), float(u[0])
    kk, vv = k[0, :, 0].astype(np.float64), v[0, :, 0].astype(np.float64)
    brute = oracle.wkv_brute(w, u, k, v)[0, :, 0]
    alt = extra_decay_form(wc, uc, kk, vv)
    assert np.max(np.abs(alt[1:] - brute[1:])) > 1e-3
    shifted = oracle.wkv_brute(w, np.float32([uc + wc]), k, v)[0, :, 0]
    np.testing.assert_allclose(alt, shifted, rtol=1e-6)
