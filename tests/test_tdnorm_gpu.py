"""GPU parity of timestep decay normalisation (gecko_tdnorm_forward) against
the fp64 oracle on the same seeded inputs: fp32 max-abs <= 1e-4; bf16
max-abs <= 2e-2 and rel-L2 <= 5e-3 (outputs are O(1) after normalisation)."""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import NORM_WORKLOADS, NormWorkload, make_norm_inputs
from oracle import tdnorm_oracle as N

pytestmark = pytest.mark.gpu

TOL = {"f32": dict(max_abs=1e-4), "bf16": dict(max_abs=2e-2, rel_l2=5e-3)}


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib
    build.build()
    lib.load()
    return lib


def _close(got, want, tol, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want).max()
    assert err <= tol["max_abs"], f"{what}: max-abs {err:.3e}"
    if "rel_l2" in tol:
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e}"


def _run(L, w, inp, **kw):
    return L.tdnorm_forward(inp["x"], inp["gamma"], inp["bias"], w.G, w.beta1, w.beta2, w.eps, **kw)


def _oracle(w, inp, groups=None):
    x, g, b = inp["x"], inp["gamma"], inp["bias"]
    G = w.G
    if groups is not None:
        gs = w.D // w.G
        idx = torch.cat([torch.arange(q * gs, (q + 1) * gs) for q in groups]).to(x.device)
        x, g, b = x[:, :, idx], g[idx], b[idx]
        G = len(groups)
    return N.tdnorm_forward(x.double().cpu().numpy(), G, w.beta1, w.beta2, w.eps, g.double().cpu().numpy(),
                            b.double().cpu().numpy())


@pytest.mark.parametrize("name", ["tdnorm_f32_small", "tdnorm_bf16_small"])
def test_small_workloads_match_oracle(L, name):
    w = NORM_WORKLOADS[name]
    inp = make_norm_inputs(w, device="cuda")
    y = _run(L, w, inp)
    torch.cuda.synchronize()
    _close(y.double().cpu().numpy(), _oracle(w, inp), TOL[w.dtype], "y")


@pytest.mark.parametrize("w", [
    NormWorkload("tdn_one_token", 61, "f32", 3, 1, 64, 4),
    NormWorkload("tdn_one_group", 62, "f32", 1, 300, 40, 1),
    NormWorkload("tdn_groups_of_8", 63, "bf16", 2, 500, 96, 12),
    NormWorkload("tdn_no_decay", 64, "f32", 1, 200, 32, 2, beta1=0.0, beta2=0.0),
    NormWorkload("tdn_long_scan", 65, "f32", 1, 5000, 16, 2, beta1=0.999, beta2=0.9999),
], ids=lambda w: w.name)
def test_edge_cases(L, w):
    inp = make_norm_inputs(w, device="cuda")
    y = _run(L, w, inp)
    torch.cuda.synchronize()
    _close(y.double().cpu().numpy(), _oracle(w, inp), TOL[w.dtype], "y")


def test_in_place(L):
    w = NORM_WORKLOADS["tdnorm_bf16_small"]
    inp = make_norm_inputs(w, device="cuda")
    want = _run(L, w, inp).clone()
    x = inp["x"].clone()
    got = _run(L, w, dict(inp, x=x), y=x)
    torch.cuda.synchronize()
    assert got.data_ptr() == x.data_ptr() and torch.equal(got, want)


def test_seven_b_width_sampled_groups(L):
    """D = 4096, 32 groups, 32K tokens: groups are independent, so the oracle
    runs on four of them over the whole sequence."""
    w = NORM_WORKLOADS["tdnorm_bf16_7b_32k"]
    inp = make_norm_inputs(w, device="cuda")
    y = _run(L, w, inp)
    torch.cuda.synchronize()
    groups = [0, 7, 19, 31]
    gs = w.D // w.G
    idx = torch.cat([torch.arange(q * gs, (q + 1) * gs) for q in groups]).to(y.device)
    _close(y[:, :, idx].double().cpu().numpy(), _oracle(w, inp, groups), TOL["bf16"], "y (sampled groups)")
