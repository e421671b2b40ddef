"""SCA with widely spread scores: the softmax's running reference must move
inside a row (O and l rescaled), and the result must still match the fp64
oracle.

The tensor-core SCA kernel exponentiates each 128-key tile against a
reference: the row max of the row's first tile, replaced by a later tile's
row max only when that exceeds it by more than 8 binary orders, at which
point the O accumulator and the running sum are rescaled.  The generator's
ordinary inputs (|q.k| of order 1) rarely move it.  Here q and k are scaled
(x12) so that scores spread over ~200 natural-log units; a CPU model of that
policy, run on the same inputs, confirms that rescales happen.
"""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import Workload, make_inputs
from oracle import gecko_oracle as G

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib
    build.build()
    lib.load()
    return lib


def _rescales(q, k, c):
    """Number of (row, key tile) where the kernel's reference moves up."""
    T = q.shape[0]
    s = (q @ k.T) * LOG2E
    n = 0
    for t in range(T):
        lo = G.window_lo(t, c)
        m_ref = None
        for j in range(lo // 128, t // 128 + 1):
            m = s[t, j * 128:min(j * 128 + 128, t + 1)].max()
            if m_ref is None:
                m_ref = m
            elif m > m_ref + 8.0:
                m_ref = m
                n += 1
    return n


@pytest.mark.parametrize("scale", [12.0])
def test_moving_reference_matches_oracle(L, scale):
    w = Workload("sca_spread", 61, "bf16", 1, 2, 1024, 128, 256)
    x = make_inputs(w, device="cuda")
    q = (x["q"].float() * scale).to(torch.bfloat16).contiguous()
    k = (x["k"].float() * scale).to(torch.bfloat16).contiguous()
    o_sca, _ = L.sca_awm_forward(q, k, x["v"], x["qm"], x["km"], w.c)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    qd, kd, vd = (t.double().cpu().numpy() for t in (q, k, x["v"]))
    got = o_sca.double().cpu().numpy()
    moved = 0
    for h in range(w.H):
        moved += _rescales(qd[0, h], kd[0, h], w.c)
        ref = G.sca_head(qd[0, h], kd[0, h], vd[0, h], w.c)
        err = np.abs(got[0, h] - ref).max()
        rel = np.linalg.norm(got[0, h] - ref) / np.linalg.norm(ref)
        assert np.all(np.isfinite(got[0, h]))
        assert err <= 2e-2 and rel <= 5e-3, (h, err, rel)
    assert moved > 0
