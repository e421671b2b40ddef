"""Plain fp64 CPU oracle for CEMA, the complex multi-dimensional damped
exponential moving average that produces the layer input X' = CEMA(X).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module.  The product path (the CUDA
library and its Python binding) never calls it, and it shares no code with
that path.

Sources (web pages on "Gecko: An Efficient Neural Architecture Inherently
Processing Sequences with Arbitrary Lengths", arXiv 2601.06463):
  [digest]  paper.rainbus.top Chinese digest, background section on the
            exponential moving average (the CEMA recurrence with damping
            factors alpha, delta and the rotation cos(theta) + i sin(theta)).
  [summary] paperlayer.ai summary, section 2.1 (each input dimension is
            expanded into h hidden dimensions, the damped EMA runs in a
            complex hidden space, and the hidden state is projected back to
            one output per input dimension) and Appendix B.1 (the recurrence
            as an affine map h_t = q_t h_{t-1} + p_t; a document reset is a
            zero multiplicative term, so the state restarts at h_t = p_t).

Readings taken where the pages are silent (listed in the design notes):
  C1  expansion: u_t[d, j] = beta[d, j] * x_t[d] (a real weight per hidden
      dimension; the pages name the expansion but print no formula).
  C2  projection: y_t[d] = Re(sum_j eta[d, j] * h_t[d, j]) with complex eta
      (the pages: "projected back to a one-dimensional output").
  C3  alpha, delta in (0, 1] and theta are given per (d, j) as they enter the
      recurrence (a layer would produce alpha, delta by a sigmoid).
  C4  h_{-1} = 0 unless a carried state is given; a reset at t (document
      start) sets the multiplicative term to zero: h_t = alpha u_t.
  C5  no skip or residual term (none is printed).
All arithmetic is complex128 / float64.
"""
from __future__ import annotations

import numpy as np

__all__ = ["decay", "cema_forward"]


def decay(alpha, delta, theta):
    """q[d, j] = (1 - alpha delta) (cos theta + i sin theta): [digest] EMA
    background, the factor that multiplies h_{t-1}."""
    alpha, delta, theta = (np.asarray(a, dtype=np.float64) for a in (alpha, delta, theta))
    return (1.0 - alpha * delta) * (np.cos(theta) + 1j * np.sin(theta))


def cema_forward(x, alpha, delta, theta, beta, eta, reset=None, state=None):
    """CEMA over x [B, L, D] (any float dtype, computed in fp64).

    alpha, delta, theta, beta: [D, h] real; eta: [D, h] complex; reset:
    [B, L] bool or None (True = the state restarts at that token); state:
    [B, D, h] complex h_{-1} or None (zeros).
    Returns (y [B, L, D] float64, final state h_{L-1} [B, D, h] complex128).

    Steps, in the pages' order: u_t = beta x_t (C1), h_t = alpha u_t +
    q h_{t-1} with q = decay(...) and q -> 0 on a reset (C4), y_t =
    Re(sum_j eta h_t) (C2).
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, D = x.shape
    beta = np.asarray(beta, dtype=np.float64)
    alpha = np.asarray(alpha, dtype=np.float64)
    eta = np.asarray(eta, dtype=np.complex128)
    q = decay(alpha, delta, theta)
    h = np.zeros((B, D, beta.shape[1]), dtype=np.complex128) if state is None else np.array(state, dtype=np.complex128)
    rs = np.zeros((B, L), dtype=bool) if reset is None else np.asarray(reset, dtype=bool)
    y = np.empty((B, L, D))
    for t in range(L):
        u = beta[None] * x[:, t, :, None]                      # [B, D, h]
        keep = (~rs[:, t]).astype(np.float64)[:, None, None]   # 0 on a reset
        h = alpha[None] * u + keep * q[None] * h
        y[:, t] = np.real(np.sum(eta[None] * h, axis=2))
    return y, h
