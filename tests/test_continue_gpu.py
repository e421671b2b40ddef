"""Streaming continuation: a sequence processed in segments through
gecko_sca_awm_forward_continue must give the outputs of the whole sequence.

Each segment passes the previous segment's last chunk of K and V as c
leading rows and the carried state (M'_S, M'_{S+1}, log z^S).  Every
segment's out_sca and out_mem, and the final state, are compared with the
fp64 oracle run over the whole sequence at once.  Tolerances as elsewhere.
"""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import Workload, make_inputs
from oracle import gecko_oracle as G

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


def _close(got, want, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want).max()
    assert err <= TOL[dtype]["max_abs"], f"{what}: max-abs {err:.3e}"
    if "rel_l2" in TOL[dtype]:
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= TOL[dtype]["rel_l2"], f"{what}: rel-L2 {rel:.3e}"


def _np(x):
    return x.detach().double().cpu().numpy()


def _oracle_whole(x, c):
    """Whole-sequence oracle: out_sca, out_mem and, per (b, h), the list of
    states M'_1 .. M'_{S+1} and log z^1 .. log z^S."""
    q, k, v, qm, km = (_np(x[n]) for n in ("q", "k", "v", "qm", "km"))
    B, H = q.shape[:2]
    o_sca = np.empty_like(q)
    o_mem = np.empty_like(q)
    states, logz = {}, {}
    for b in range(B):
        for h in range(H):
            o_sca[b, h] = G.sca_head(q[b, h], k[b, h], v[b, h], c)
            om, st, lz = G.awm_head(qm[b, h], km[b, h], v[b, h], c)
            o_mem[b, h] = om
            states[b, h], logz[b, h] = st, lz
    return o_sca, o_mem, states, logz


CASES = [
    # (workload, segment lengths in chunks, kernels)
    (Workload("cont_bf16_d128", 51, "bf16", 1, 2, 2048, 128, 256), [3, 1, 4], None),
    (Workload("cont_bf16_d64", 52, "bf16", 2, 1, 1536, 64, 128), [2, 5, 5], None),
    (Workload("cont_bf16_simt", 53, "bf16", 1, 2, 1024, 128, 128), [1, 3, 4], "simt"),
    (Workload("cont_fp32", 54, "f32", 1, 2, 768, 64, 64, shared_z=True), [5, 2, 1, 4], None),
]


@pytest.mark.parametrize("w,segs,kernels", CASES, ids=[c[0].name for c in CASES])
def test_segments_match_whole_sequence(L, w, segs, kernels, monkeypatch):
    if kernels:
        monkeypatch.setenv("GECKO_KERNELS", kernels)
    assert sum(segs) * w.c == w.T
    x = make_inputs(w, device="cuda")
    r_sca, r_mem, r_states, r_logz = _oracle_whole(x, w.c)
    state = None
    a = 0
    for n in segs:
        b = a + n * w.c
        lo = a - w.c if state is not None else a
        seg = {name: x[name][:, :, a:b].contiguous() for name in ("q", "qm", "km")}
        kk = x["k"][:, :, lo:b].contiguous()
        vv = x["v"][:, :, lo:b].contiguous()
        o_sca, o_mem, state = L.sca_awm_forward_segment(seg["q"], kk, vv, seg["qm"], seg["km"], w.c,
                                                        state_in=state)
        torch.cuda.synchronize()
        assert L.device_status() == 0
        _close(_np(o_sca), r_sca[:, :, a:b], w.dtype, f"out_sca rows {a}:{b}")
        _close(_np(o_mem), r_mem[:, :, a:b], w.dtype, f"out_mem rows {a}:{b}")
        s_end = b // w.c  # chunks processed so far (1-based index of the last chunk)
        d = w.d
        st = _np(state)
        for bb in range(w.B):
            for hh in range(w.H):
                _close(st[bb, hh, :d * d].reshape(d, d), r_states[bb, hh][s_end], w.dtype, "M'_S")
                _close(st[bb, hh, d * d:2 * d * d].reshape(d, d), r_states[bb, hh][s_end + 1], w.dtype, "M'_{S+1}")
                _close(st[bb, hh, 2 * d * d:], r_logz[bb, hh][s_end - 1], w.dtype, "log z^S")
        a = b


def test_state_may_be_updated_in_place(L):
    w = Workload("cont_inplace", 55, "bf16", 1, 2, 1024, 128, 256)
    x = make_inputs(w, device="cuda")
    r_sca, r_mem, _, _ = _oracle_whole(x, w.c)
    d, c = w.d, w.c
    state = torch.empty(w.B, w.H, 2 * d * d + d, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for a, b in ((0, 2 * c), (2 * c, 4 * c)):
        lo = a - c if a > 0 else a
        q, qm, km = (x[n][:, :, a:b].contiguous() for n in ("q", "qm", "km"))
        kk, vv = (x[n][:, :, lo:b].contiguous() for n in ("k", "v"))
        o_sca, o_mem = torch.empty_like(q), torch.empty_like(q)
        rc = L.gecko_sca_awm_forward_continue(q.data_ptr(), kk.data_ptr(), vv.data_ptr(), qm.data_ptr(),
                                              km.data_ptr(), o_sca.data_ptr(), o_mem.data_ptr(),
                                              state.data_ptr() if a > 0 else 0, state.data_ptr(),
                                              w.B, w.H, b - a, c, d, L.GECKO_BF16, stream)
        assert rc == 0, L.gecko_last_error()
        torch.cuda.synchronize()
        _close(_np(o_sca), r_sca[:, :, a:b], "bf16", "out_sca")
        _close(_np(o_mem), r_mem[:, :, a:b], "bf16", "out_mem")
