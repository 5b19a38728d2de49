"""Randomised properties of the oracle (hypothesis), on top of the fixed pins:
the facts every correct implementation of the definition satisfies, drawn
over shapes, split points and parameter ranges the fixed cases do not reach.

- Chunking: a carried state reproduces one pass at any split (the carried
  state of "Process million-token sequences").
- Brute force: the explicit sum ("コア計算") equals the recurrence.
- Scan algebra: the summary of a concatenation is the combination of the
  summaries ("並列学習の定式化": the parallel mode is a scan).
- Token shift: any split with the carried token reproduces one pass.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])


def draw_case(seed, B, T, C, gate, state, k_std):
    g = np.random.default_rng(seed)
    w = np.exp(g.uniform(-3, 1, C)).astype(np.float32)
    u = g.normal(0, 1, C).astype(np.float32)
    k = (g.normal(0, 1, (B, T, C)) * k_std).astype(np.float32)
    v = g.normal(0, 1, (B, T, C)).astype(np.float32)
    r = g.normal(0, 1, (B, T, C)).astype(np.float32) if gate else None
    s0 = None
    if state:
        b = g.uniform(0.5, 1.5, (B, C))
        s0 = np.stack([b * g.normal(0, 1, (B, C)), b, g.uniform(-5, 5, (B, C))]).astype(np.float32).astype(np.float64)
    return w, u, k, v, r, s0


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), B=st.integers(1, 3), T=st.integers(2, 80), C=st.integers(1, 5),
       gate=st.booleans(), state=st.booleans(), k_std=st.sampled_from([1.0, 3.0, 20.0]), data=st.data())
def test_chunked_equals_one_pass_at_any_split(seed, B, T, C, gate, state, k_std, data):
    w, u, k, v, r, s0 = draw_case(seed, B, T, C, gate, state, k_std)
    split = data.draw(st.integers(1, T - 1))
    y, s = oracle.wkv_forward(w, u, k, v, r, s0)
    sl = lambda x, a, b: None if x is None else x[:, a:b]
    y1, s1 = oracle.wkv_forward(w, u, sl(k, 0, split), sl(v, 0, split), sl(r, 0, split), s0)
    y2, s2 = oracle.wkv_forward(w, u, sl(k, split, T), sl(v, split, T), sl(r, split, T), s1)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(s2, s)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), T=st.integers(1, 40), C=st.integers(1, 4), gate=st.booleans(),
       state=st.booleans(), k_std=st.sampled_from([1.0, 5.0, 30.0]))
def test_explicit_sum_equals_recurrence(seed, T, C, gate, state, k_std):
    w, u, k, v, r, s0 = draw_case(seed, 2, T, C, gate, state, k_std)
    yb, scale = oracle.wkv_brute(w, u, k, v, r, s0, want_scale=True)
    yf = oracle.wkv_forward(w, u, k, v, r, s0)[0]
    assert np.max(np.abs(yb - yf) / scale) <= 1e-12


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), n1=st.integers(1, 30), n2=st.integers(1, 30),
       k_std=st.sampled_from([1.0, 10.0]), w_log=st.floats(-4.0, 2.0))
def test_summary_of_concatenation_is_the_combination(seed, n1, n2, k_std, w_log):
    g = np.random.default_rng(seed)
    w = float(np.exp(w_log))
    k = g.normal(0, k_std, n1 + n2)
    v = g.normal(0, 1, n1 + n2)
    whole = oracle.summary(w, k, v)
    first, second = oracle.summary(w, k[:n1], v[:n1]), oracle.summary(w, k[n1:], v[n1:])
    both = oracle.combine(w, first, second, n2)
    # compare the represented N = a e^p and D = b e^p, relative to D
    N = lambda s: s[1] * np.exp(s[0] - whole[0])
    D = lambda s: s[2] * np.exp(s[0] - whole[0])
    assert abs(D(both) - D(whole)) <= 1e-12 * D(whole)
    assert abs(N(both) - N(whole)) <= 1e-12 * D(whole) * max(1.0, float(np.max(np.abs(v))))


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), B=st.integers(1, 3), T=st.integers(2, 50), C=st.integers(1, 6),
       nmix=st.integers(1, 8), prev=st.booleans(), data=st.data())
def test_token_shift_any_split_with_carried_token(seed, B, T, C, nmix, prev, data):
    g = np.random.default_rng(seed)
    x = g.normal(0, 1, (B, T, C)).astype(np.float32)
    mu = g.uniform(0, 1, (nmix, C)).astype(np.float32)
    xp = g.normal(0, 1, (B, C)).astype(np.float32) if prev else None
    split = data.draw(st.integers(1, T - 1))
    whole, last = oracle.token_shift(x, mu, xp)
    a, la = oracle.token_shift(x[:, :split], mu, xp)
    b, lb = oracle.token_shift(x[:, split:], mu, la.astype(np.float32))
    assert np.array_equal(np.concatenate([a, b], axis=2), whole)
    assert np.array_equal(lb, last)
