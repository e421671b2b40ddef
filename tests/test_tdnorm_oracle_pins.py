"""Pins of the timestep-decay-normalisation oracle against things other than
itself: torch's group_norm (beta = 0), pandas' bias-adjusted EWM (the decayed,
bias-corrected statistics), exactness of the bias correction on constant
statistics, equivariance and causality; planted mistakes fail a pin."""
import numpy as np
import pandas as pd
import pytest
import torch

from oracle import tdnorm_oracle as N

RNG = np.random.default_rng(11)


def _affine(D):
    return RNG.normal(1.0, 0.2, D), RNG.normal(0.0, 0.2, D)


def test_zero_decay_is_group_norm_per_timestep():
    B, L, D, G = 2, 9, 24, 4
    x = RNG.normal(size=(B, L, D)) * 3 + 1
    g, b = _affine(D)
    y = N.tdnorm_forward(x, G, 0.0, 0.0, 1e-5, g, b)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x.reshape(B * L, D, 1)), G,
                                         torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    np.testing.assert_allclose(y, ref.numpy().reshape(B, L, D), rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("beta", [0.9, 0.99, 0.5])
def test_decayed_statistics_are_bias_adjusted_ewm(beta):
    B, L, G = 1, 300, 3
    mu = RNG.normal(size=(B, L, G))
    s2 = RNG.uniform(0.5, 2.0, size=(B, L, G))
    mh, vh = N.decayed_stats(mu, s2, beta, beta ** 0.5)
    for g in range(G):
        np.testing.assert_allclose(mh[0, :, g], pd.Series(mu[0, :, g]).ewm(alpha=1 - beta, adjust=True).mean(),
                                   rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(vh[0, :, g],
                                   pd.Series(s2[0, :, g]).ewm(alpha=1 - beta ** 0.5, adjust=True).mean(),
                                   rtol=1e-10, atol=1e-12)


def test_bias_correction_is_exact_for_constant_statistics():
    B, L, D, G = 1, 50, 16, 2
    row = RNG.normal(size=D)
    x = np.broadcast_to(row, (B, L, D)).copy()
    g, b = _affine(D)
    y = N.tdnorm_forward(x, G, 0.9, 0.999, 1e-6, g, b)
    y0 = N.tdnorm_forward(x[:, :1], G, 0.0, 0.0, 1e-6, g, b)
    np.testing.assert_allclose(y, np.broadcast_to(y0, y.shape), rtol=1e-9, atol=1e-9)


def test_shift_and_scale_equivariance_without_eps():
    B, L, D, G = 1, 40, 12, 3
    x = RNG.normal(size=(B, L, D))
    one, zero = np.ones(D), np.zeros(D)
    y = N.tdnorm_forward(x, G, 0.8, 0.95, 0.0, one, zero)
    y2 = N.tdnorm_forward(3.5 * x - 2.0, G, 0.8, 0.95, 0.0, one, zero)
    np.testing.assert_allclose(y2, y, rtol=1e-9, atol=1e-9)


def test_causal():
    B, L, D, G, t = 1, 60, 8, 2, 33
    x = RNG.normal(size=(B, L, D))
    g, b = _affine(D)
    y = N.tdnorm_forward(x, G, 0.9, 0.99, 1e-5, g, b)
    x2 = x.copy()
    x2[:, t + 1:] = RNG.normal(size=(B, L - t - 1, D)) * 10
    y2 = N.tdnorm_forward(x2, G, 0.9, 0.99, 1e-5, g, b)
    np.testing.assert_array_equal(y[:, :t + 1], y2[:, :t + 1])


@pytest.mark.parametrize("mistake", ["no_bias_correction", "beta1_for_variance", "unbiased_variance"])
def test_pins_catch_planted_mistakes(mistake, monkeypatch):
    """Each plausible slip makes one of the independent pins above fail."""
    orig_ds, orig_gs = N.decayed_stats, N.group_stats
    if mistake == "no_bias_correction":
        def broken(mu, s2, b1, b2):
            mh, vh = orig_ds(mu, s2, b1, b2)
            t = np.arange(1, mu.shape[1] + 1)[None, :, None]
            return mh * (1 - b1 ** t), vh * (1 - b2 ** t)
        monkeypatch.setattr(N, "decayed_stats", broken)
    elif mistake == "beta1_for_variance":
        monkeypatch.setattr(N, "decayed_stats", lambda mu, s2, b1, b2: orig_ds(mu, s2, b1, b1))
    else:
        def broken_stats(xx, GG):
            mu, s2 = orig_gs(xx, GG)
            n = np.asarray(xx).shape[2] // GG
            return mu, s2 * n / (n - 1)
        monkeypatch.setattr(N, "group_stats", broken_stats)
    pins = (test_zero_decay_is_group_norm_per_timestep, lambda: test_decayed_statistics_are_bias_adjusted_ewm(0.9))
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0
