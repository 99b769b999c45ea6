"""Pins for the CPU oracle of the Gated DeltaNet recurrence (no GPU).

The pages state the mechanism (each write overwrites the state along the
current key direction; injected noise plateaus; an impulse is forgotten
within hundreds of steps: bayesiansapien wiki, "The four-part mechanism
study", part 3).  These tests check the oracle against properties that
follow from that mechanism and from the mathematics, not against a retyped
formula: exact overwrite along k, decay-only action orthogonal to k, the
delta rule as a gradient step on the key-value regression loss (finite
differences), the chunked form against the token-by-token form, and the
closed-form contraction and plateau against simulation.
"""
import numpy as np
import pytest

from oracle.gdn import (gdn_error_contraction, gdn_error_trace, gdn_noise_plateau,
                        gdn_recurrence_chunked, gdn_recurrence_seq)


def unit_rows(rng, T, d):
    k = rng.standard_normal((T, d))
    return k / np.linalg.norm(k, axis=1, keepdims=True)


def test_full_write_overwrites_along_the_key():
    """beta = 1, no decay: after each write the state maps k_t exactly to v_t."""
    rng = np.random.default_rng(0)
    T, dk, dv = 40, 16, 12
    k, v, q = unit_rows(rng, T, dk), rng.standard_normal((T, dv)), rng.standard_normal((T, dk))
    S0 = rng.standard_normal((dv, dk))
    for t in range(1, T + 1):
        _, S = gdn_recurrence_seq(q[:t], k[:t], v[:t], np.zeros(t), np.ones(t), S0=S0)
        np.testing.assert_allclose(S @ k[t - 1], v[t - 1], rtol=0, atol=1e-12)


def test_directions_orthogonal_to_the_key_only_decay():
    rng = np.random.default_rng(1)
    dk, dv = 24, 8
    S0 = rng.standard_normal((dv, dk))
    k = unit_rows(rng, 1, dk)
    v, q = rng.standard_normal((1, dv)), rng.standard_normal((1, dk))
    g, beta = np.array([-0.3]), np.array([0.7])
    _, S1 = gdn_recurrence_seq(q, k, v, g, beta, S0=S0)
    u = rng.standard_normal(dk)
    u -= (u @ k[0]) * k[0]                                  # u orthogonal to k
    np.testing.assert_allclose(S1 @ u, np.exp(-0.3) * (S0 @ u), rtol=1e-12, atol=1e-12)


def test_no_write_no_decay_keeps_the_state():
    rng = np.random.default_rng(2)
    T, dk, dv = 30, 8, 8
    S0 = rng.standard_normal((dv, dk))
    q = rng.standard_normal((T, dk))
    O, S = gdn_recurrence_seq(q, unit_rows(rng, T, dk), rng.standard_normal((T, dv)),
                              np.zeros(T), np.zeros(T), S0=S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(O, q @ S0.T, rtol=1e-12, atol=1e-12)


def test_write_is_a_gradient_step_on_the_regression_loss():
    """S_t = X - beta grad L(X) with X = alpha S_{t-1}, L(X) = |X k - v|^2 / 2;
    the gradient is taken by central finite differences."""
    rng = np.random.default_rng(3)
    dk, dv = 6, 5
    S0 = rng.standard_normal((dv, dk))
    k, v, q = unit_rows(rng, 1, dk), rng.standard_normal((1, dv)), rng.standard_normal((1, dk))
    g, beta = -0.2, 0.45
    X = np.exp(g) * S0

    def loss(Y):
        r = Y @ k[0] - v[0]
        return 0.5 * r @ r

    grad = np.zeros_like(X)
    h = 1e-6
    for i in range(dv):
        for j in range(dk):
            E = np.zeros_like(X)
            E[i, j] = h
            grad[i, j] = (loss(X + E) - loss(X - E)) / (2 * h)
    _, S1 = gdn_recurrence_seq(q, k, v, np.array([g]), np.array([beta]), S0=S0)
    np.testing.assert_allclose(S1, X - beta * grad, rtol=0, atol=1e-8)


@pytest.mark.parametrize("T,chunk", [(1, 64), (63, 64), (64, 64), (300, 64), (257, 32), (100, 7)])
def test_chunked_form_equals_the_token_by_token_form(T, chunk):
    rng = np.random.default_rng(T * 7 + chunk)
    dk, dv = 32, 48
    q = rng.standard_normal((T, dk))
    k = unit_rows(rng, T, dk)
    v = rng.standard_normal((T, dv))
    g = -np.exp(rng.uniform(-1, 1.5, T)) * np.log1p(np.exp(rng.normal(0, 1, T)))   # decay-gate range
    beta = 1.0 / (1.0 + np.exp(-rng.normal(0, 1.5, T)))
    S0 = rng.standard_normal((dv, dk))
    O1, S1 = gdn_recurrence_seq(q, k, v, g, beta, S0=S0)
    O2, S2 = gdn_recurrence_chunked(q, k, v, g, beta, chunk=chunk, S0=S0)
    scale = max(1.0, np.abs(O1).max())
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-10 * scale)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-10 * max(1.0, np.abs(S1).max()))


def test_impulse_decays_at_the_closed_form_rate():
    """Mean over keys of |Delta_t|^2 / |Delta_0|^2 against rho^t (no noise)."""
    rng = np.random.default_rng(4)
    dk, dv, T, trials, beta, alpha = 32, 16, 120, 200, 0.6, 1.0
    rho = gdn_error_contraction(alpha, beta, dk)
    acc = np.zeros(T)
    for _ in range(trials):
        e0 = rng.standard_normal((dv, dk))
        acc += gdn_error_trace(unit_rows(rng, T, dk), beta, alpha, None, e0=e0) / np.sum(e0 * e0)
    mean = acc / trials
    expect = rho ** np.arange(1, T + 1)
    np.testing.assert_allclose(mean, expect, rtol=0.05)


def test_noise_plateaus_where_an_accumulator_grows():
    """With noise every step the delta-rule error settles at sigma^2 / (1 - rho);
    a purely additive state's error grows as t sigma^2."""
    rng = np.random.default_rng(5)
    dk, dv, T, beta, alpha = 32, 16, 3000, 0.5, 1.0
    sigma = 0.01
    noise = rng.standard_normal((T, dv, dk)) * sigma
    sigma2 = sigma ** 2 * dv * dk
    trace = gdn_error_trace(unit_rows(rng, T, dk), beta, alpha, noise)
    plateau = gdn_noise_plateau(sigma2, alpha, beta, dk)
    tail = trace[T // 2:]
    assert abs(tail.mean() / plateau - 1.0) < 0.1
    # flat: the last quarter's mean matches the third quarter's
    assert abs(trace[3 * T // 4:].mean() / trace[T // 2: 3 * T // 4].mean() - 1.0) < 0.1
    additive = np.cumsum(noise, axis=0)
    acc = np.sum(additive * additive, axis=(1, 2))
    t = np.arange(1, T + 1)
    assert abs(acc[-1] / (t[-1] * sigma2) - 1.0) < 0.1
    assert acc[-1] > 10 * tail.mean()


def test_forgetting_time_is_hundreds_of_steps_at_model_width():
    """At a GDN head width of 128 and beta = 1/2 the e-folding time of an
    impulse is d_k / (2 beta - beta^2) ~ 170 steps: "hundreds of steps"."""
    tau = -1.0 / np.log(gdn_error_contraction(1.0, 0.5, 128))
    assert 100 <= tau <= 1000
    assert abs(tau - 128 / 0.75) / tau < 0.01
