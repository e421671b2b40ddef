"""GPU parity of the CEMA kernels (gecko_cema_forward) against the fp64 CEMA
oracle on the same seeded inputs.  Tolerances as for the attention path:
fp32 max-abs <= 1e-4; bf16 output max-abs <= 2e-2 and rel-L2 <= 5e-3; the
final state (fp32 on both paths) max-abs <= 1e-4."""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import CEMA_WORKLOADS, CemaWorkload, make_cema_inputs
from oracle import cema_oracle as C

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
    cplx = np.iscomplexobj(got) or np.iscomplexobj(want)
    got = np.asarray(got, dtype=np.complex128 if cplx else np.float64)
    want = np.asarray(want, dtype=np.complex128 if cplx else np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want).max()
    assert err <= tol["max_abs"], f"{what}: max-abs {err:.3e}"
    if "rel_l2" in tol:
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e}"


def _oracle(inp, feats=None, state=None):
    sel = slice(None) if feats is None else feats
    p = {k: inp[k].double().cpu().numpy()[sel] for k in ("alpha", "delta", "theta", "beta")}
    e = inp["eta"].double().cpu().numpy()[sel]
    xs = inp["x"] if feats is None else inp["x"][:, :, torch.as_tensor(feats, device=inp["x"].device)]
    x = xs.double().cpu().numpy()
    reset = None if inp["reset"] is None else inp["reset"].cpu().numpy().astype(bool)
    return C.cema_forward(x, p["alpha"], p["delta"], p["theta"], p["beta"], e[..., 0] + 1j * e[..., 1], reset=reset,
                          state=state)


def _run(L, inp, **kw):
    return L.cema_forward(inp["x"], inp["alpha"], inp["delta"], inp["theta"], inp["beta"], inp["eta"],
                          reset=inp["reset"], **kw)


@pytest.mark.parametrize("name", ["cema_f32_small", "cema_bf16_small"])
def test_small_workloads_match_oracle(L, name):
    w = CEMA_WORKLOADS[name]
    inp = make_cema_inputs(w, device="cuda")
    assert int(inp["reset"].sum()) > 0
    y, st = _run(L, inp, return_state=True)
    torch.cuda.synchronize()
    ry, rst = _oracle(inp)
    _close(y.double().cpu().numpy(), ry, TOL[w.dtype], "y")
    got_st = st.double().cpu().numpy()
    _close(got_st[..., 0] + 1j * got_st[..., 1], rst, TOL["f32"], "final state")


@pytest.mark.parametrize("w", [
    CemaWorkload("cema_one_token", 31, "f32", 3, 1, 40),
    CemaWorkload("cema_all_resets", 32, "f32", 1, 300, 130, mean_doc=1),
    CemaWorkload("cema_chunk_edge", 33, "f32", 1, 513, 128, mean_doc=200),
], ids=lambda w: w.name)
def test_edge_cases(L, w):
    inp = make_cema_inputs(w, device="cuda")
    if inp["reset"] is not None:
        inp["reset"][:, 0] = 1
    y = _run(L, inp)
    torch.cuda.synchronize()
    ry, _ = _oracle(inp)
    _close(y.double().cpu().numpy(), ry, TOL["f32"], "y")


def test_segments_chain_through_the_state(L):
    w = CEMA_WORKLOADS["cema_f32_small"]
    inp = make_cema_inputs(w, device="cuda")
    y_all = _run(L, inp)
    cut = 389
    first = {k: v for k, v in inp.items()}
    first["x"] = inp["x"][:, :cut].contiguous()
    first["reset"] = inp["reset"][:, :cut].contiguous()
    second = dict(inp)
    second["x"] = inp["x"][:, cut:].contiguous()
    second["reset"] = inp["reset"][:, cut:].contiguous()
    ya, sa = _run(L, first, return_state=True)
    yb, sb = _run(L, second, state_in=sa, return_state=True)
    torch.cuda.synchronize()
    _close(torch.cat([ya, yb], dim=1).double().cpu().numpy(), y_all.double().cpu().numpy(), TOL["f32"], "y")
    _, rst = _oracle(inp)
    got = sb.double().cpu().numpy()
    _close(got[..., 0] + 1j * got[..., 1], rst, TOL["f32"], "final state")


def test_in_place(L):
    w = CEMA_WORKLOADS["cema_bf16_small"]
    inp = make_cema_inputs(w, device="cuda")
    want = _run(L, inp).clone()
    x = inp["x"].clone()
    inp2 = dict(inp, x=x)
    got = _run(L, inp2, y=x)
    torch.cuda.synchronize()
    assert got.data_ptr() == x.data_ptr()
    assert torch.equal(got, want)


def test_seven_b_width_sampled_features(L):
    """D = 4096, h = 16, 32K tokens: features are independent, so the oracle
    runs on eight sampled features over the whole sequence."""
    w = CEMA_WORKLOADS["cema_bf16_7b_32k"]
    inp = make_cema_inputs(w, device="cuda")
    y, st = _run(L, inp, return_state=True)
    torch.cuda.synchronize()
    feats = np.array([0, 1, 127, 128, 2047, 3001, 4094, 4095])
    ry, rst = _oracle(inp, feats)
    _close(y[:, :, feats].double().cpu().numpy(), ry, TOL["bf16"], "y (sampled features)")
    got = st[:, feats].double().cpu().numpy()
    _close(got[..., 0] + 1j * got[..., 1], rst, TOL["f32"], "final state (sampled features)")


@pytest.mark.parametrize("w,plain", [
    (CemaWorkload("cema_bf16_d100", 34, "bf16", 2, 700, 100, mean_doc=250), False),   # D % 8 != 0: plain loads
    (CemaWorkload("cema_bf16_plain", 35, "bf16", 1, 900, 136, mean_doc=300), True),   # plain path forced
    (CemaWorkload("cema_bf16_tma", 36, "bf16", 3, 777, 264, mean_doc=300), False),    # TMA path, ragged L and D
], ids=lambda v: getattr(v, "name", str(v)))
def test_bf16_paths(L, w, plain, monkeypatch):
    if plain:
        monkeypatch.setenv("GECKO_CEMA_PLAIN", "1")
    inp = make_cema_inputs(w, device="cuda")
    y, st = _run(L, inp, return_state=True)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    ry, rst = _oracle(inp)
    _close(y.double().cpu().numpy(), ry, TOL["bf16"], "y")
    got = st.double().cpu().numpy()
    _close(got[..., 0] + 1j * got[..., 1], rst, TOL["f32"], "final state")
