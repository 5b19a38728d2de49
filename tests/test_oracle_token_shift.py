"""Pins for the oracle's token shift (x'_t = mu x_t + (1 - mu) x_{t-1}, one
learned mu per channel, from the token-shift section of the RWKV article),
independent of the oracle's own code: hand-derived exact values
(tests/golden), the two limits mu = 1 and mu = 0 that reduce it to the input
and to the input delayed by one token, chunking, affinity, and a planted
swap of mu and 1 - mu that the pins must catch."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_shift_hand_worked.json")
rng = np.random.default_rng(2024)


def golden_cases():
    return json.load(open(GOLDEN))["cases"]


def arrays(case):
    x = np.array(case["x"], np.float32)
    mu = np.array(case["mu"], np.float32)
    xp = None if case["x_prev"] is None else np.array(case["x_prev"], np.float32)
    return x, mu, xp


@pytest.mark.parametrize("idx", range(2))
def test_golden_hand_worked(idx):
    case = golden_cases()[idx]
    x, mu, xp = arrays(case)
    out, last = oracle.token_shift(x, mu, xp)
    assert np.array_equal(out, np.array(case["out"]))          # exact binary fractions
    assert np.array_equal(last, np.array(case["x_last"]))


def test_planted_swap_of_mu_fails_the_golden():
    """A plausible mistake, mu and 1 - mu exchanged, computed by handing the
    oracle 1 - mu: it must disagree with the hand-worked values."""
    case = golden_cases()[0]
    x, mu, xp = arrays(case)
    out, _ = oracle.token_shift(x, (1.0 - mu).astype(np.float32), xp)
    assert not np.array_equal(out, np.array(case["out"]))


def test_limits_identity_and_delay():
    B, T, C = 3, 17, 5
    x = rng.standard_normal((B, T, C)).astype(np.float32)
    xp = rng.standard_normal((B, C)).astype(np.float32)
    mu = np.stack([np.ones(C), np.zeros(C)]).astype(np.float32)
    out, last = oracle.token_shift(x, mu, xp)
    assert np.array_equal(out[0], x.astype(np.float64))                    # mu = 1: the token itself
    delayed = np.concatenate([xp[:, None, :], x[:, :-1, :]], axis=1)
    assert np.array_equal(out[1], delayed.astype(np.float64))              # mu = 0: the previous token
    assert np.array_equal(last, x[:, -1, :].astype(np.float64))


def test_fresh_sequence_mixes_with_zeros():
    x = rng.standard_normal((2, 4, 3)).astype(np.float32)
    mu = rng.uniform(0, 1, (1, 3)).astype(np.float32)
    out, _ = oracle.token_shift(x, mu, None)
    out0, _ = oracle.token_shift(x, mu, np.zeros((2, 3), np.float32))
    assert np.array_equal(out, out0)
    assert np.allclose(out[0, :, 0, :], mu[0].astype(np.float64) * x[:, 0, :], rtol=0, atol=0)


@pytest.mark.parametrize("split", [1, 7, 16])
def test_chunked_equals_single_pass(split):
    """x_last of one call, fed as the next call's x_prev, reproduces one pass."""
    B, T, C = 2, 17, 4
    x = rng.standard_normal((B, T, C)).astype(np.float32)
    xp = rng.standard_normal((B, C)).astype(np.float32)
    mu = rng.uniform(0, 1, (3, C)).astype(np.float32)
    whole, last = oracle.token_shift(x, mu, xp)
    a, la = oracle.token_shift(x[:, :split], mu, xp)
    b, lb = oracle.token_shift(x[:, split:], mu, la.astype(np.float32))
    assert np.array_equal(np.concatenate([a, b], axis=2), whole)
    assert np.array_equal(lb, last)


def test_affine_in_the_input_and_between_neighbours():
    B, T, C = 2, 9, 6
    # multiples of 1/256 in [-4, 4]: alpha x + beta below is exact in float32
    x = rng.integers(-1024, 1025, (B, T, C)) / 256.0
    xp = rng.integers(-1024, 1025, (B, C)) / 256.0
    mu = rng.uniform(0, 1, (2, C)).astype(np.float32)
    out, _ = oracle.token_shift(x.astype(np.float32), mu, xp.astype(np.float32))
    alpha, beta = 0.5, 3.0
    x2 = (alpha * x.astype(np.float32) + beta).astype(np.float32)
    xp2 = (alpha * xp.astype(np.float32) + beta).astype(np.float32)
    out2, _ = oracle.token_shift(x2, mu, xp2)
    assert np.allclose(out2, alpha * out + beta, rtol=1e-12, atol=1e-12)
    # a convex mix lies between the two tokens it mixes
    prev = np.concatenate([xp[:, None, :], x[:, :-1, :]], axis=1).astype(np.float32)
    lo = np.minimum(x.astype(np.float32), prev) - 1e-12
    hi = np.maximum(x.astype(np.float32), prev) + 1e-12
    assert np.all((out >= lo) & (out <= hi))


def test_empty_sequence_passes_the_state_through():
    xp = rng.standard_normal((2, 3)).astype(np.float32)
    out, last = oracle.token_shift(np.zeros((2, 0, 3), np.float32), np.ones((1, 3), np.float32), xp)
    assert out.shape == (1, 2, 0, 3)
    assert np.array_equal(last, xp.astype(np.float64))
