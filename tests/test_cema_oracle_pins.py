"""Pins of the CEMA oracle against things other than itself: a direct
double-sum closed form, scipy's IIR filter with complex coefficients, the
real EMA special case (pandas), impulse and constant-input closed forms, and
structural properties (linearity, resets, carried state)."""
import numpy as np
import pandas as pd
import pytest
import scipy.signal

from oracle import cema_oracle as C

RNG = np.random.default_rng(7)


def _params(D, h, rng=RNG, long_memory=False):
    ad = rng.uniform(1e-3, 0.05, (D, h)) if long_memory else rng.uniform(0.05, 0.9, (D, h))
    alpha = rng.uniform(0.2, 1.0, (D, h))
    delta = np.minimum(ad / alpha, 1.0)
    theta = rng.uniform(0, np.pi, (D, h))
    beta = rng.normal(size=(D, h))
    eta = rng.normal(size=(D, h)) + 1j * rng.normal(size=(D, h))
    return alpha, delta, theta, beta, eta


def _direct(x, alpha, delta, theta, beta, eta, reset=None, state=None):
    """h_t = sum_{s = start(t)}^{t} q^{t-s} alpha beta x_s (+ q^{t+1} h_{-1}
    when no reset <= t), with start(t) the last reset <= t: the recurrence
    unrolled, evaluated as an explicit double sum."""
    B, L, D = x.shape
    q = (1 - alpha * delta) * np.exp(1j * theta)
    y = np.zeros((B, L, D))
    for b in range(B):
        for t in range(L):
            r = [s for s in range(t + 1) if reset is not None and reset[b, s]]
            start = r[-1] if r else 0
            hcur = np.zeros_like(q)
            for s in range(start, t + 1):
                hcur = hcur + q ** (t - s) * alpha * beta * x[b, s][:, None]
            if not r and state is not None:
                hcur = hcur + q ** (t + 1) * state[b]
            y[b, t] = np.real(np.sum(eta * hcur, axis=1))
    return y


def test_matches_direct_double_sum_with_resets_and_state():
    B, L, D, h = 2, 37, 3, 4
    p = _params(D, h)
    x = RNG.normal(size=(B, L, D))
    reset = np.zeros((B, L), bool)
    reset[0, 11] = reset[0, 30] = reset[1, 5] = True
    state = RNG.normal(size=(B, D, h)) + 1j * RNG.normal(size=(B, D, h))
    y, _ = C.cema_forward(x, *p, reset=reset, state=state)
    np.testing.assert_allclose(y, _direct(x, *p, reset=reset, state=state), rtol=1e-11, atol=1e-11)


def test_matches_scipy_lfilter_complex():
    """Per (d, j), h is the output of the first-order IIR filter with
    numerator [alpha beta] and denominator [1, -q] (zero initial state)."""
    B, L, D, h = 1, 500, 5, 16
    p = _params(D, h, long_memory=True)
    alpha, delta, theta, beta, eta = p
    x = RNG.normal(size=(B, L, D))
    y, hL = C.cema_forward(x, *p)
    q = (1 - alpha * delta) * np.exp(1j * theta)
    ref = np.zeros((L, D))
    for d in range(D):
        for j in range(h):
            hs = scipy.signal.lfilter([alpha[d, j] * beta[d, j]], [1.0, -q[d, j]], x[0, :, d].astype(np.complex128))
            ref[:, d] += np.real(eta[d, j] * hs)
            assert abs(hs[-1] - hL[0, d, j]) < 1e-10
    np.testing.assert_allclose(y[0], ref, rtol=1e-10, atol=1e-10)


def test_real_case_is_the_textbook_ema():
    """h = 1, theta = 0, delta = 1, beta = eta = 1: y_t = alpha x_t + (1 - alpha) y_{t-1}."""
    L, a = 200, 0.13
    x = RNG.normal(size=L)
    x[0] = 0.0   # pandas starts from y_0 = x_0; the oracle from h_{-1} = 0
    y, _ = C.cema_forward(x[None, :, None], np.full((1, 1), a), np.ones((1, 1)), np.zeros((1, 1)),
                          np.ones((1, 1)), np.ones((1, 1)))
    ref = pd.Series(x).ewm(alpha=a, adjust=False).mean().to_numpy()
    np.testing.assert_allclose(y[0, :, 0], ref, rtol=1e-12, atol=1e-14)


def test_impulse_response_is_geometric():
    D, h, L, t0 = 2, 8, 60, 9
    alpha, delta, theta, beta, eta = _params(D, h)
    x = np.zeros((1, L, D))
    x[0, t0, 1] = 1.0
    y, _ = C.cema_forward(x, alpha, delta, theta, beta, eta)
    q = (1 - alpha[1] * delta[1]) * np.exp(1j * theta[1])
    for t in range(L):
        want = 0.0 if t < t0 else np.real(np.sum(eta[1] * alpha[1] * beta[1] * q ** (t - t0)))
        assert abs(y[0, t, 1] - want) < 1e-12
        assert y[0, t, 0] == 0.0


def test_constant_input_closed_form():
    D, h, L = 3, 16, 80
    alpha, delta, theta, beta, eta = _params(D, h)
    x = np.full((1, L, D), 0.7)
    y, _ = C.cema_forward(x, alpha, delta, theta, beta, eta)
    q = (1 - alpha * delta) * np.exp(1j * theta)
    for t in (0, 1, 17, L - 1):
        hs = 0.7 * alpha * beta * (1 - q ** (t + 1)) / (1 - q)
        np.testing.assert_allclose(y[0, t], np.real(np.sum(eta * hs, axis=1)), rtol=1e-12, atol=1e-12)


def test_linearity():
    B, L, D, h = 2, 50, 4, 16
    p = _params(D, h)
    x1, x2 = RNG.normal(size=(2, B, L, D))
    y1, _ = C.cema_forward(x1, *p)
    y2, _ = C.cema_forward(x2, *p)
    y12, _ = C.cema_forward(2.5 * x1 - 0.5 * x2, *p)
    np.testing.assert_allclose(y12, 2.5 * y1 - 0.5 * y2, rtol=1e-11, atol=1e-11)


def test_reset_cuts_the_history_and_splits_the_sequence():
    B, L, D, h, tr = 1, 90, 3, 16, 41
    p = _params(D, h, long_memory=True)
    x = RNG.normal(size=(B, L, D))
    reset = np.zeros((B, L), bool)
    reset[0, tr] = True
    y, _ = C.cema_forward(x, *p, reset=reset)
    x2 = x.copy()
    x2[0, :tr] = RNG.normal(size=(tr, D))
    y2, _ = C.cema_forward(x2, *p, reset=reset)
    np.testing.assert_array_equal(y[0, tr:], y2[0, tr:])
    assert np.abs(y[0, :tr] - y2[0, :tr]).max() > 1e-3
    ya, _ = C.cema_forward(x[:, :tr], *p)
    yb, _ = C.cema_forward(x[:, tr:], *p)
    np.testing.assert_allclose(y, np.concatenate([ya, yb], axis=1), rtol=1e-12, atol=1e-12)


def test_carried_state_continues_the_sequence():
    B, L, D, h, L1 = 2, 70, 3, 16, 29
    p = _params(D, h, long_memory=True)
    x = RNG.normal(size=(B, L, D))
    y, hL = C.cema_forward(x, *p)
    ya, ha = C.cema_forward(x[:, :L1], *p)
    yb, hb = C.cema_forward(x[:, L1:], *p, state=ha)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hb, hL, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mistake", ["no_rotation", "no_damping_delta", "reset_ignored"])
def test_pins_catch_planted_mistakes(mistake, monkeypatch):
    """A plausible slip in the oracle fails the direct closed form."""
    B, L, D, h = 1, 30, 2, 4
    p = _params(D, h)
    x = RNG.normal(size=(B, L, D))
    reset = np.zeros((B, L), bool)
    reset[0, 13] = True
    good = _direct(x, *p, reset=reset)
    if mistake == "no_rotation":
        monkeypatch.setattr(C, "decay", lambda a, d, th: (1 - np.asarray(a) * np.asarray(d)) + 0j)
        y, _ = C.cema_forward(x, *p, reset=reset)
    elif mistake == "no_damping_delta":
        monkeypatch.setattr(C, "decay", lambda a, d, th: (1 - np.asarray(a)) * np.exp(1j * np.asarray(th)))
        y, _ = C.cema_forward(x, *p, reset=reset)
    else:
        y, _ = C.cema_forward(x, *p, reset=None)
    assert np.abs(y - good).max() > 1e-6
