"""Pins of the gradient oracle against things other than itself: central
finite differences of the (independently pinned) forward oracle, element by
element on tiny inputs; torch's scaled-dot-product-attention backward where
SCA reduces to causal attention (one or two chunks); invariants that follow
from the forward's symmetries; and planted mistakes that must fail a pin."""
import numpy as np
import pytest
import torch

from oracle import gecko_backward_oracle as GB
from oracle import gecko_oracle as F

RNG = np.random.default_rng(5)


def _inputs(T, d, scale=0.7):
    q, k, qm, km = (RNG.normal(size=(T, d)) * scale for _ in range(4))
    v = RNG.normal(size=(T, d))
    return q, k, v, qm, km


def _loss(q, k, v, qm, km, c, W):
    """Scalar test loss: weighted sums of both outputs and of the exported state."""
    o_sca = F.sca_head(q, k, v, c)
    o_mem, st, lz = F.awm_head(qm, km, v, c, keep_states=False)
    return ((W["sca"] * o_sca).sum() + (W["mem"] * o_mem).sum()
            + (W["M"] * st[-1]).sum() + (W["lz"] * lz[-1]).sum())


def _grads(q, k, v, qm, km, c, W):
    dq, dk, dv1 = GB.sca_head_backward(q, k, v, c, W["sca"])
    dqm, dkm, dv2 = GB.awm_head_backward(qm, km, v, c, W["mem"], W["M"], W["lz"])
    return dict(q=dq, k=dk, v=dv1 + dv2, qm=dqm, km=dkm)


def _finite_differences(x, c, W, h=1e-5):
    """Central differences of the loss for every element of every input."""
    out = {}
    for name in x:
        g = np.zeros_like(x[name])
        for idx in np.ndindex(*x[name].shape):
            for sgn in (1, -1):
                y = {n: a.copy() for n, a in x.items()}
                y[name][idx] += sgn * h
                g[idx] += sgn * _loss(y["q"], y["k"], y["v"], y["qm"], y["km"], c, W)
            g[idx] /= 2 * h
        out[name] = g
    return out


def _case(T, c, d, state_grads=True):
    x = dict(zip(("q", "k", "v", "qm", "km"), _inputs(T, d)))
    W = dict(sca=RNG.normal(size=(T, d)), mem=RNG.normal(size=(T, d)),
             M=RNG.normal(size=(d, d)) if state_grads else np.zeros((d, d)),
             lz=RNG.normal(size=d) if state_grads else np.zeros(d))
    return x, W


@pytest.mark.parametrize("T,c,d", [(16, 4, 3), (15, 3, 2), (8, 8, 3), (12, 2, 2)])
def test_gradients_match_finite_differences(T, c, d):
    x, W = _case(T, c, d)
    got = _grads(x["q"], x["k"], x["v"], x["qm"], x["km"], c, W)
    want = _finite_differences(x, c, W)
    for name in x:
        np.testing.assert_allclose(got[name], want[name], rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("nchunks", [1, 2])
def test_sca_gradients_equal_causal_attention_backward(nchunks):
    """With at most two chunks every query sees all earlier keys, so SCA is
    causal softmax attention (scale 1): torch's SDPA backward in fp64."""
    c, d = 16, 8
    T = nchunks * c
    q, k, v, _, _ = _inputs(T, d)
    do = RNG.normal(size=(T, d))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None], is_causal=True, scale=1.0)
    o.backward(torch.tensor(do)[None])
    dq, dk, dv = GB.sca_head_backward(q, k, v, c, do)
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-10, atol=1e-12)


def test_sca_lse_matches_torch_logsumexp_on_causal_case():
    c, d = 8, 4
    q, k, _, _, _ = _inputs(2 * c, d)
    sc = torch.tensor(q @ k.T)
    sc = sc.masked_fill(torch.ones_like(sc, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(GB.sca_lse(q, k, c), torch.logsumexp(sc, dim=1).numpy(), rtol=1e-12)


def test_gradient_invariants():
    """Adding one vector to every key shifts each score row by a constant, so
    the key gradients of SCA sum to zero; the AWM outputs do not change when a
    scalar is added to all of K_m, and psi is a row softmax, so the K_m
    gradients sum to zero and each Q_m gradient row sums to zero."""
    T, c, d = 48, 8, 5
    q, k, v, qm, km = _inputs(T, d, scale=1.5)
    do_s, do_m = RNG.normal(size=(T, d)), RNG.normal(size=(T, d))
    _, dk, _ = GB.sca_head_backward(q, k, v, c, do_s)
    np.testing.assert_allclose(dk.sum(axis=0), 0, atol=1e-11)
    dqm, dkm, _ = GB.awm_head_backward(qm, km, v, c, do_m)
    np.testing.assert_allclose(dqm.sum(axis=1), 0, atol=1e-11)
    assert abs(dkm.sum()) < 1e-10 * np.abs(dkm).sum()


def test_first_two_chunks_give_no_query_gradient_to_memory():
    """Chunks 1 and 2 read M'_0 = M'_1 = 0, so their Q_m get no gradient."""
    T, c, d = 24, 4, 3
    q, k, v, qm, km = _inputs(T, d)
    dqm, _, _ = GB.awm_head_backward(qm, km, v, c, RNG.normal(size=(T, d)))
    assert np.all(dqm[:2 * c] == 0) and np.abs(dqm[2 * c:]).max() > 0


def test_batched_backward_matches_per_head():
    B, H, T, c, d = 2, 2, 16, 4, 3
    x = [RNG.normal(size=(B, H, T, d)) for _ in range(7)]
    dq, dk, dv, dqm, dkm = GB.backward(*x[:5], c, x[5], x[6])
    h = (1, 0)
    a = GB.sca_head_backward(x[0][h], x[1][h], x[2][h], c, x[5][h])
    m = GB.awm_head_backward(x[3][h], x[4][h], x[2][h], c, x[6][h])
    np.testing.assert_array_equal(dq[h], a[0])
    np.testing.assert_array_equal(dkm[h], m[1])
    np.testing.assert_array_equal(dv[h], a[2] + m[2])


@pytest.mark.parametrize("mistake", ["no_ratio_term", "log_z_held_constant", "softmax_without_centering"])
def test_planted_mistakes_fail_finite_differences(mistake, monkeypatch):
    """Each plausible slip in the reverse pass breaks the finite-difference pin:
    dropping the z-ratio carry of G, treating log z as a constant, or a
    softmax backward without its row-sum term."""
    T, c, d = 12, 3, 2
    x, W = _case(T, c, d)
    want = _finite_differences(x, c, W)      # forward untouched
    if mistake == "no_ratio_term":
        monkeypatch.setattr(F, "z_ratio", lambda logz, s: np.zeros(logz.shape[1]))
    elif mistake == "log_z_held_constant":
        monkeypatch.setattr(GB, "_log_z_backward", lambda km, c, l, L, dL: np.zeros_like(km))
    else:
        monkeypatch.setattr(GB, "_softmax_backward", lambda y, dy: y * dy)
    got = _grads(x["q"], x["k"], x["v"], x["qm"], x["km"], c, W)
    assert any(not np.allclose(got[n], want[n], rtol=1e-6, atol=1e-8) for n in x)


def test_row_by_row_sca_gradients_agree_with_whole_head():
    T, c, d = 40, 8, 4
    q, k, v, _, _ = _inputs(T, d)
    do = RNG.normal(size=(T, d))
    dq, dk, dv = GB.sca_head_backward(q, k, v, c, do)
    rows = [0, 7, 8, 15, 16, 23, 39]
    np.testing.assert_allclose(GB.sca_query_rows_backward(q, k, v, do, c, rows), dq[rows], rtol=1e-10, atol=1e-12)
    kr, vr = GB.sca_key_rows_backward(q, k, v, do, c, rows)
    np.testing.assert_allclose(kr, dk[rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(vr, dv[rows], rtol=1e-10, atol=1e-12)
