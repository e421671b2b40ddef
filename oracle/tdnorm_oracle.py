"""Plain fp64 CPU oracle for timestep decay normalisation, the normalisation
Gecko applies before its projections.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module.  The product path never
calls it and shares no code with it.

Sources (web pages on "Gecko: An Efficient Neural Architecture Inherently
Processing Sequences with Arbitrary Lengths", arXiv 2601.06463):
  [digest]  paper.rainbus.top Chinese digest, section on technical novelty:
            the cumulative mean m_t = beta1 m_{t-1} + (1 - beta1) mu_t with
            Adam-style bias correction, replacing Megalodon's cumulative
            statistics whose current contribution shrinks as t grows.
  [summary] paperlayer.ai summary, section 2.2 (Megalodon's timestep
            normalisation: cumulative means and variances of groups of the
            input across previous timesteps) and section 3.1 (decay
            hyperparameters beta1, beta2 fix the share of the current mean
            and variance; initialisation bias correction of both).

Readings taken where the pages are silent (listed in the design notes):
  T1  mu_t and sigma2_t of group g are the mean and the (biased) variance of
      x_t over the features of that group (D / G contiguous features).
  T2  the variance statistic follows the printed mean update with beta2:
      v_t = beta2 v_{t-1} + (1 - beta2) sigma2_t, m_0 = v_0 = 0.
  T3  bias correction as in Adam: m^_t = m_t / (1 - beta1^t),
      v^_t = v_t / (1 - beta2^t), t counted from 1.
  T4  output y_t = (x_t - m^_t) / sqrt(v^_t + eps) * gamma + bias, with a
      per-feature affine (gamma, bias) as in group normalisation.
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np

__all__ = ["group_stats", "decayed_stats", "tdnorm_forward"]


def group_stats(x, G: int):
    """mu, sigma2 [B, L, G]: mean and biased variance of each feature group (T1)."""
    x = np.asarray(x, dtype=np.float64)
    B, L, D = x.shape
    xg = x.reshape(B, L, G, D // G)
    mu = xg.mean(axis=3)
    return mu, ((xg - mu[..., None]) ** 2).mean(axis=3)


def decayed_stats(mu, s2, beta1: float, beta2: float):
    """Bias-corrected decayed statistics m^_t, v^_t [B, L, G] ([digest], T2, T3)."""
    B, L, G = mu.shape
    m = np.zeros((B, G))
    v = np.zeros((B, G))
    mh = np.empty_like(mu)
    vh = np.empty_like(s2)
    for t in range(L):
        m = beta1 * m + (1.0 - beta1) * mu[:, t]
        v = beta2 * v + (1.0 - beta2) * s2[:, t]
        mh[:, t] = m / (1.0 - beta1 ** (t + 1))
        vh[:, t] = v / (1.0 - beta2 ** (t + 1))
    return mh, vh


def tdnorm_forward(x, G: int, beta1: float, beta2: float, eps: float, gamma, bias):
    """y [B, L, D] float64 for x [B, L, D]; gamma, bias [D] (T4)."""
    x = np.asarray(x, dtype=np.float64)
    B, L, D = x.shape
    mu, s2 = group_stats(x, G)
    mh, vh = decayed_stats(mu, s2, beta1, beta2)
    mh_f = np.repeat(mh, D // G, axis=2)
    vh_f = np.repeat(vh, D // G, axis=2)
    return (x - mh_f) / np.sqrt(vh_f + eps) * np.asarray(gamma, np.float64) + np.asarray(bias, np.float64)
