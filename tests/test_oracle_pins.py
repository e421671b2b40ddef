"""Pins for the fp64 oracle, independent of the oracle itself.

Each test checks the oracle against something the pages or the mathematics
fix: a brute-force restatement in loops, a library routine that the method
reduces to in a special case, an invariant the pages state, an exact closed
form, or a hand-derived golden fixture.  The mutation tests at the end plant
plausible mistakes in the oracle and check that a pin catches each one.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import gecko_oracle as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _as_lists(a):
    return [list(map(float, r)) for r in a]


# ----------------------------------------------------------------- SCA ----

def _sca_brute_err(T=24, d=3, seeds=(0, 1), cs=(1, 2, 3, 4, 6, 8, 12)):
    worst = 0.0
    for seed in seeds:
        r = _rng(seed)
        q, k, v = (r.standard_normal((T, d)) for _ in range(3))
        for c in cs:
            got = G.sca_head(q, k, v, c)
            ref = np.array(brute.sca_banded(_as_lists(q), _as_lists(k), _as_lists(v), c))
            worst = max(worst, float(np.abs(got - ref).max()))
    return worst


def test_sca_matches_banded_mask_brute_force():
    assert _sca_brute_err() < 1e-12


@pytest.mark.parametrize("c", [4, 16, 64])
def test_sca_one_or_two_chunks_is_causal_attention(c):
    # With S <= 2 every query sees exactly its causal prefix, so SCA reduces to
    # ordinary causal softmax attention with scale 1 (a library routine).
    r = _rng(c)
    d = 8
    for T in (c, 2 * c):
        q, k, v = (r.standard_normal((T, d)) for _ in range(3))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
            torch.from_numpy(v)[None, None], is_causal=True, scale=1.0)[0, 0].numpy()
        assert np.abs(G.sca_head(q, k, v, c) - ref).max() < 1e-12


def test_sca_three_chunks_is_not_full_causal_attention():
    # Beyond two chunks the window must drop chunk s-2: compare against causal
    # attention and require a difference exactly in chunk 3.
    r = _rng(5)
    c, d = 4, 4
    q, k, v = (r.standard_normal((3 * c, d)) for _ in range(3))
    full = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], is_causal=True, scale=1.0)[0, 0].numpy()
    got = G.sca_head(q, k, v, c)
    assert np.abs(got[:2 * c] - full[:2 * c]).max() < 1e-12
    assert np.abs(got[2 * c:] - full[2 * c:]).min() > 0.0


def test_sca_constant_values_pass_through():
    r = _rng(3)
    T, d, c = 48, 5, 8
    q, k = r.standard_normal((T, d)) * 3, r.standard_normal((T, d)) * 3
    v = np.tile(r.standard_normal((1, d)), (T, 1))
    assert np.abs(G.sca_head(q, k, v, c) - v).max() < 1e-13


def _probe_window_lo(T, c):
    # Q = K = 0 makes every visible key equally weighted; V[:,0] = t and
    # V[:,1] = 1 make out[t,0] the mean visible position (lo + t) / 2.
    q = np.zeros((T, 2))
    k = np.zeros((T, 2))
    v = np.stack([np.arange(T, dtype=np.float64), np.ones(T)], axis=1)
    out = G.sca_head(q, k, v, c)
    assert np.abs(out[:, 1] - 1.0).max() < 1e-12
    return [int(round(2 * out[t, 0] - t)) for t in range(T)]


def test_sca_mask_probe_matches_golden_windows():
    path = os.path.join(GOLDEN, "sca_window_lo_c4_T16.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    want = {int(t): int(lo) for t, lo in rows}
    got = _probe_window_lo(16, 4)
    assert got == [want[t] for t in range(16)]


@pytest.mark.parametrize("c", [1, 3, 8])
def test_sca_mask_probe_matches_window_rule(c):
    T = 6 * c
    got = _probe_window_lo(T, c)
    assert got == [max(0, (t // c - 1) * c) for t in range(T)]


def test_sca_outputs_lie_in_value_hull():
    r = _rng(9)
    T, d, c = 64, 4, 8
    q, k, v = (r.standard_normal((T, d)) * 2 for _ in range(3))
    out = G.sca_head(q, k, v, c)
    for t in range(T):
        lo = max(0, (t // c - 1) * c)
        w = v[lo:t + 1]
        assert np.all(out[t] <= w.max(axis=0) + 1e-12)
        assert np.all(out[t] >= w.min(axis=0) - 1e-12)


def test_sca_rows_agrees_with_chunked():
    r = _rng(11)
    T, d, c = 64, 6, 16
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    rows = [0, 5, 15, 16, 31, 32, 47, 63]
    assert np.abs(G.sca_rows(q, k, v, c, rows) - G.sca_head(q, k, v, c)[rows]).max() < 1e-12


# ------------------------------------------------------------ z, phi, psi --

def test_psi_rows_sum_to_one_and_are_positive():
    x = _rng(1).standard_normal((50, 16)) * 20
    p = G.psi(x)
    assert np.all(p > 0)
    assert np.abs(p.sum(axis=1) - 1).max() < 1e-12


def test_normaliser_tau_is_one():
    # tau^s[f] = sum over every token of chunks 1..s of phi^s(k)[f] = 1, and
    # hence psi(q) tau = 1 for every query (paperlayer.ai summary, 3.3).
    r = _rng(2)
    c, S, d = 5, 6, 7
    km = r.standard_normal((c * S, d)) * 3
    lz = G.log_z(km, c)
    qm = r.standard_normal((4, d))
    for s in range(1, S + 1):
        tau = G.phi(km[: s * c], lz[s - 1]).sum(axis=0)
        assert np.abs(tau - 1).max() < 1e-12
        assert np.abs(G.psi(qm) @ tau - 1).max() < 1e-12


def test_log_z_is_monotone_and_matches_direct_sum():
    r = _rng(4)
    c, S, d = 4, 9, 3
    km = r.standard_normal((c * S, d))
    lz = G.log_z(km, c)
    assert np.all(np.diff(lz, axis=0) > 0)
    for s in range(1, S + 1):
        direct = np.array([math.log(sum(math.exp(km[t, f]) for t in range(s * c))) for f in range(d)])
        assert np.abs(lz[s - 1] - direct).max() < 1e-12


def test_shift_invariance_survives_large_offsets():
    # phi is invariant to a per-feature constant added to K_m, psi to a per-row
    # constant; exp(1000) overflows fp64, so this pins the log-space path.
    r = _rng(6)
    c, S, d = 4, 5, 3
    km = r.standard_normal((c * S, d))
    qm = r.standard_normal((c * S, d))
    v = r.standard_normal((c * S, d))
    o1, s1, _ = G.awm_head(qm, km, v, c)
    o2, s2, _ = G.awm_head(qm + 700.0, km + 1000.0, v, c)
    assert np.all(np.isfinite(o2))
    assert np.abs(o1 - o2).max() < 1e-9
    assert np.abs(s1[-1] - s2[-1]).max() < 1e-9


# -------------------------------------------------------------- AWM carry --

def test_awm_matches_tokenwise_unnormalised_form():
    r = _rng(7)
    c, S, d, dv = 3, 5, 4, 3
    T = c * S
    km = r.standard_normal((T, d)) * 1.5
    qm = r.standard_normal((T, d))
    v = r.standard_normal((T, dv))
    out, states, lz = G.awm_head(qm, km, v, c)
    b_out, b_states, b_z = brute.awm_tokenwise(_as_lists(qm), _as_lists(km), _as_lists(v), c)
    assert np.abs(out - np.array(b_out)).max() < 1e-12
    for s in range(1, S + 2):
        assert np.abs(states[s] - np.array(b_states[s - 1])).max() < 1e-12
    assert np.abs(lz[-1] - np.log(np.array(b_z))).max() < 1e-12


def test_awm_without_delta_term_is_normalised_linear_attention():
    # Dropping psi(K)M' leaves M'_s = sum_{tokens of chunks < s} exp(k)^T v / z^{s-1}.
    r = _rng(8)
    c, S, d, dv = 4, 6, 3, 2
    T = c * S
    km, qm = r.standard_normal((T, d)), r.standard_normal((T, d))
    v = r.standard_normal((T, dv))
    out, states, _ = G.awm_head(qm, km, v, c, delta=False)
    for s in range(2, S + 2):
        n = (s - 1) * c
        e = np.exp(km[:n])
        closed = (e.T @ v[:n]) / e.sum(axis=0)[:, None]
        assert np.abs(states[s] - closed).max() < 1e-12


def _km_zero_case(S, c, d):
    T = S * c
    v = np.zeros((T, d))
    for t in range(T):
        v[t, t // c] = 1.0          # V[t] = e_{chunk(t)} (0-based basis index)
    km = np.zeros((T, d))
    qm = _rng(12).standard_normal((T, d))  # readout is independent of Q_m here
    return qm, km, v


def test_awm_zero_keys_exact_rationals():
    # K_m = 0 gives phi = 1/(s c), psi = 1/d, and all rows of M'_s equal m_s with
    # m_{s+1} = ((s-2)/s) m_s + mean(V over chunk s)/s, m_1 = 0 (hand derivation
    # from the update with the delta term).  Compare against exact fractions.
    S, c, d = 7, 3, 8
    qm, km, v = _km_zero_case(S, c, d)
    out, states, _ = G.awm_head(qm, km, v, c)
    m = {1: [Fraction(0)] * d}
    for s in range(1, S + 1):
        vbar = [Fraction(1) if j == s - 1 else Fraction(0) for j in range(d)]
        m[s + 1] = [Fraction(s - 2, s) * m[s][j] + vbar[j] / s for j in range(d)]
    for s in range(1, S + 2):
        want = np.array([float(x) for x in m[s]])
        assert np.abs(states[s] - want[None, :]).max() < 1e-14
    for s in range(1, S + 1):
        prev = np.zeros(d) if s == 1 else np.array([float(x) for x in m[s - 1]])
        assert np.abs(out[(s - 1) * c: s * c] - prev[None, :]).max() < 1e-14


def test_awm_zero_keys_matches_golden_fixture():
    path = os.path.join(GOLDEN, "awm_zero_keys_readout.txt")
    want = {}
    for ln in open(path):
        if not ln.strip() or ln.startswith("#"):
            continue
        s, vec = ln.split(":")
        want[int(s)] = [Fraction(x) for x in vec.split()]
    S, c, d = 6, 2, 6
    qm, km, v = _km_zero_case(S, c, d)
    out, _, _ = G.awm_head(qm, km, v, c)
    for s, vec in want.items():
        row = out[(s - 1) * c]
        assert np.abs(row - np.array([float(x) for x in vec])).max() < 1e-14, s


def test_row_weights_sum_to_one_and_carry_is_non_expansive():
    # r_f + sum_i phi_{i,f} = 1, so A_s = diag(r) - Phi^T Psi has inf-norm <= 1.
    r = _rng(13)
    c, S, d = 6, 5, 5
    km = r.standard_normal((c * S, d)) * 2
    lz = G.log_z(km, c)
    for s in range(1, S + 1):
        k_s = km[(s - 1) * c: s * c]
        Phi = G.phi(k_s, lz[s - 1])
        rr = G.z_ratio(lz, s)
        assert np.abs(rr + Phi.sum(axis=0) - 1).max() < 1e-12
        A = np.diag(rr) - Phi.T @ G.psi(k_s)
        assert np.abs(A).sum(axis=1).max() <= 1 + 1e-12


def test_edge_chunks():
    r = _rng(14)
    c, S, d = 4, 4, 3
    T = c * S
    qm, km, v = (r.standard_normal((T, d)) for _ in range(3))
    out, states, lz = G.awm_head(qm, km, v, c)
    assert np.all(out[: 2 * c] == 0.0)             # chunks 1 and 2 read zero
    assert np.all(states[1] == 0.0)                 # M'_1 = 0
    Phi1 = np.exp(km[:c]) / np.exp(km[:c]).sum(axis=0)
    assert np.abs(states[2] - Phi1.T @ v[:c]).max() < 1e-13
    o1, s1, _ = G.awm_head(qm[:c], km[:c], v[:c], c)  # T = c
    assert np.all(o1 == 0.0)
    assert np.abs(s1[-1] - Phi1.T @ v[:c]).max() < 1e-13


def test_literal_printed_form_is_not_the_reading_when_c_equals_d():
    # With c = d the printed "- psi(K) M'" (a c x d matrix) can be added to the
    # d x d state; the oracle must still use the delta-rule reading.
    r = _rng(15)
    c = d = 4
    S = 4
    T = c * S
    qm, km, v = (r.standard_normal((T, d)) for _ in range(3))
    _, states, lz = G.awm_head(qm, km, v, c)
    M = np.zeros((d, d))
    for s in range(1, S + 1):
        k_s, v_s = km[(s - 1) * c: s * c], v[(s - 1) * c: s * c]
        M = G.z_ratio(lz, s)[:, None] * M + G.phi(k_s, lz[s - 1]).T @ v_s - G.psi(k_s) @ M
    assert np.abs(M - states[-1]).max() > 1e-3


def test_streaming_propagation_matches_whole_head():
    r = _rng(16)
    c, S, d = 4, 7, 3
    T = c * S
    qm, km, v = (r.standard_normal((T, d)) for _ in range(3))
    out, states, lz = G.awm_head(qm, km, v, c)
    ch = lambda a: (a[i * c:(i + 1) * c] for i in range(S))
    got, M, l = G.awm_propagate(ch(km), ch(v), ch(qm), c, want_chunks=[1, 3, 7])
    for s, o in got.items():
        assert np.abs(o - out[(s - 1) * c: s * c]).max() < 1e-12
    assert np.abs(M - states[-1]).max() < 1e-12
    assert np.abs(l - lz[-1]).max() < 1e-12


def test_forward_on_small_workload():
    from long_context_sequence_sca_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["fp32_small"]
    x = make_inputs(w)
    o_sca, o_mem, M, lz = G.forward(*(x[n].numpy() for n in ("q", "k", "v", "qm", "km")), w.c)
    assert o_sca.shape == (1, 1, 512, 64) and M.shape == (1, 1, 64, 64) and lz.shape == (1, 1, 64)
    assert np.all(np.isfinite(o_sca)) and np.all(np.isfinite(o_mem))
    assert np.all(o_mem[:, :, : 2 * w.c] == 0)


# ------------------------------------------------------- planted mistakes --

def _awm_tokenwise_err():
    r = _rng(7)
    c, S, d, dv = 3, 5, 4, 3
    T = c * S
    km = r.standard_normal((T, d)) * 1.5
    qm = r.standard_normal((T, d))
    v = r.standard_normal((T, dv))
    out, states, _ = G.awm_head(qm, km, v, c)
    b_out, b_states, _ = brute.awm_tokenwise(_as_lists(qm), _as_lists(km), _as_lists(v), c)
    e = np.abs(out - np.array(b_out)).max()
    for s in range(1, S + 2):
        e = max(e, np.abs(states[s] - np.array(b_states[s - 1])).max())
    return float(e)


MUTANTS = {
    "window includes chunk s-2": ("window_lo", lambda t, c: max(0, (t // c - 2) * c)),
    "window drops previous chunk": ("window_lo", lambda t, c: (t // c) * c),
    "softmax scale 1/sqrt(d)": ("SCA_SCALE", 0.5),
    "ratio index shifted": ("z_ratio", lambda lz, s: np.zeros(lz.shape[1]) if s <= 2 else np.exp(lz[s - 3] - lz[s - 2])),
    "ratio inverted": ("z_ratio", lambda lz, s: np.zeros(lz.shape[1]) if s == 1 else np.exp(lz[s - 1] - lz[s - 2])),
    "psi over time instead of features": ("psi", lambda x: np.exp(x - x.max(0)) / np.exp(x - x.max(0)).sum(0)),
    "phi uses previous z": ("phi", lambda k, l: np.exp(k - l[None, :] + 0.1)),
    "delta sign flipped": ("carry_step", lambda M, k, v, lz, s, delta=True:
                           G.z_ratio(lz, s)[:, None] * M + G.phi(k, lz[s - 1]).T @ (v + G.psi(k) @ M)),
    "delta operand transposed": ("carry_step", lambda M, k, v, lz, s, delta=True:
                                 G.z_ratio(lz, s)[:, None] * M + G.phi(k, lz[s - 1]).T @ (v - G.psi(k) @ M.T)),
    "readout off by a factor": ("readout", lambda qm, M: G.psi(qm) @ M * 1.01),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, repl = MUTANTS[name]
    monkeypatch.setattr(G, attr, repl)
    caught = False
    try:
        caught |= _sca_brute_err(T=12, cs=(2, 3, 4)) > 1e-9
        caught |= _awm_tokenwise_err() > 1e-9
        x = _rng(1).standard_normal((6, 5))
        caught |= np.abs(G.psi(x).sum(axis=1) - 1).max() > 1e-9
    except Exception:
        caught = True
    assert caught, name
