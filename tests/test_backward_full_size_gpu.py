"""The backward at the 7B-layer-shaped bench configuration (B=1, H=32,
T=32768, d=128, c=4096, bf16), in the launch configuration bench.py times,
checked on samples the oracle can compute one by one: dq of query rows at
chunk starts, ends and tile edges; dk and dv of key rows whose queries the
oracle can enumerate in seconds; and the complete AWM gradients (dqm, dkm)
of two heads.  Bars as in test_backward_gpu.py."""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import WORKLOADS, make_inputs
from oracle import gecko_backward_oracle as GB

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "qm", "km")


def _close(got, want, what):
    got = np.asarray(got, np.float64)
    scale = max(1.0, float(np.abs(want).max()))
    err = float(np.abs(got - want).max())
    assert err <= 2e-2 * scale, f"{what}: max-abs {err:.3e}"
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert rel <= 1e-2, f"{what}: rel-L2 {rel:.3e}"


@pytest.fixture(scope="module")
def run():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib as L
    build.build()
    L.load()
    w = WORKLOADS["bf16_h32_c4096"]
    x = make_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(77)
    dos = torch.randn(x["q"].shape, generator=g, device="cuda").to(x["q"].dtype)
    dom = torch.randn(x["q"].shape, generator=g, device="cuda").to(x["q"].dtype)
    out_sca, _, lse, lo = L.sca_awm_forward_train(*(x[n] for n in NAMES), w.c)
    grads = L.sca_awm_backward(*(x[n] for n in NAMES), out_sca, lse, dos, dom, w.c, out_sca_lo=lo)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return w, x, dos, dom, grads


def _head(t, h):
    return t[0, h].double().cpu().numpy()


@pytest.mark.parametrize("h", [0, 31])
def test_sampled_query_rows_dq(run, h):
    w, x, dos, dom, grads = run
    c, T = w.c, w.T
    rows = [0, 127, 128, 4095, 4096, 4100, 8191, 8192 + 255, 20000, T - 129, T - 128, T - 1]
    q, k, v, do = _head(x["q"], h), _head(x["k"], h), _head(x["v"], h), _head(dos, h)
    want = GB.sca_query_rows_backward(q, k, v, do, c, rows)
    _close(_head(grads[0], h)[rows], want, f"dq head {h}")


def test_sampled_key_rows_dk_dv(run):
    """Keys of chunk s receive gradient only from queries of chunks s and
    s + 1, whose windows lie in chunks s - 1 .. s + 1: the oracle's whole-head
    backward on that three-chunk slice is exact for the middle chunk's keys
    (and on the last two chunks for the last chunk's keys)."""
    w, x, dos, dom, grads = run
    h, c, S = 5, w.c, w.S
    heads = {n: _head(x[n], h) for n in NAMES}
    do = _head(dos, h)
    _, _, dv_awm = GB.awm_head_backward(heads["qm"], heads["km"], heads["v"], c, _head(dom, h))
    for mid, lo_ch, hi_ch in ((2, 1, 4), (S - 1, S - 2, S)):
        sl = slice(lo_ch * c, hi_ch * c)
        _, dk, dv = GB.sca_head_backward(heads["q"][sl], heads["k"][sl], heads["v"][sl], c, do[sl])
        offs = np.array([0, 1, 127, 128, 2049, c - 129, c - 1])
        keys = mid * c + offs
        local = keys - lo_ch * c
        _close(_head(grads[1], h)[keys], dk[local], f"dk (keys of chunk {mid + 1})")
        _close(_head(grads[2], h)[keys], dv[local] + dv_awm[keys], f"dv (keys of chunk {mid + 1})")


@pytest.mark.parametrize("h", [3, 30])
def test_awm_gradients_of_whole_heads(run, h):
    w, x, dos, dom, grads = run
    dqm, dkm, _ = GB.awm_head_backward(_head(x["qm"], h), _head(x["km"], h), _head(x["v"], h), w.c, _head(dom, h))
    _close(_head(grads[3], h), dqm, f"dqm head {h}")
    _close(_head(grads[4], h), dkm, f"dkm head {h}")
