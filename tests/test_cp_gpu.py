"""Context parallelism with the library's kernels on one GPU: the sequence is
split into P segments and cp.cp_forward_emulated runs every rank's phases
(segment log-sums, cp log z, segment maps, composed states, continued
forwards) in one process.  The concatenated outputs must match the oracle's
forward over the whole sequence within the forward's bars (fp32 max-abs
<= 1e-4; bf16 max-abs <= 2e-2 and rel-L2 <= 5e-3)."""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import gecko_oracle as F

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "qm", "km")


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib
    build.build()
    lib.load()
    return lib


def _close(got, want, dtype, what):
    got = got.double().cpu().numpy()
    err = float(np.abs(got - want).max())
    assert err <= (1e-4 if dtype == "f32" else 2e-2), f"{what}: max-abs {err:.3e}"
    if dtype == "bf16":
        rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
        assert rel <= 5e-3, f"{what}: rel-L2 {rel:.3e}"


@pytest.mark.parametrize("w,P", [
    (WORKLOADS["fp32_small"], 2),
    (WORKLOADS["fp32_small"], 4),
    (WORKLOADS["bf16_many_chunks"], 4),
    (Workload("cp_bf16_d128_c128", 81, "bf16", 1, 2, 1024, 128, 128), 2),
    (Workload("cp_bf16_one_chunk_segments", 82, "bf16", 1, 2, 512, 128, 128), 4),
], ids=lambda v: getattr(v, "name", str(v)))
def test_emulated_ranks_match_whole_sequence(L, w, P):
    from long_context_sequence_sca_b200 import cp
    x = make_inputs(w, device="cuda")
    Tr = w.T // P
    segs = [{n: x[n][:, :, r * Tr:(r + 1) * Tr].contiguous() for n in NAMES} for r in range(P)]
    outs = cp.cp_forward_emulated(segs, w.c)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    o_sca = torch.cat([o[0] for o in outs], dim=2)
    o_mem = torch.cat([o[1] for o in outs], dim=2)
    want = F.forward(*(x[n].double().cpu().numpy() for n in NAMES), w.c)
    _close(o_sca, want[0], w.dtype, "out_sca")
    _close(o_mem, want[1], w.dtype, "out_mem")


def test_segment_maps_reproduce_the_continued_state(L):
    """The map (A, b) of a segment, applied to the state entering it, gives
    the state the continued forward ends with."""
    w = Workload("cp_maps", 83, "f32", 1, 2, 512, 64, 64)
    x = make_inputs(w, device="cuda")
    half = w.T // 2
    s0 = {n: x[n][:, :, :half].contiguous() for n in NAMES}
    s1 = {n: x[n][:, :, half:].contiguous() for n in NAMES}
    _, _, st0 = L.sca_awm_forward_segment(s0["q"], s0["k"], s0["v"], s0["qm"], s0["km"], w.c)
    k1 = torch.cat([s0["k"][:, :, -w.c:], s1["k"]], dim=2).contiguous()
    v1 = torch.cat([s0["v"][:, :, -w.c:], s1["v"]], dim=2).contiguous()
    _, _, st1 = L.sca_awm_forward_segment(s1["q"], k1, v1, s1["qm"], s1["km"], w.c, state_in=st0)
    d = w.d
    logz_in = st0[..., 2 * d * d:].contiguous()
    maps = L.awm_segment_maps(s1["km"], s1["v"], logz_in, w.c)
    M_in = st0[..., d * d:2 * d * d].reshape(1, 2, d, d)
    torch.cuda.synchronize()
    want_out = st1[..., d * d:2 * d * d].reshape(1, 2, d, d)
    want_prev = st1[..., :d * d].reshape(1, 2, d, d)
    got_out = maps[:, :, 0] @ M_in + maps[:, :, 1]
    got_prev = maps[:, :, 2] @ M_in + maps[:, :, 3]
    assert torch.allclose(got_out, want_out, atol=1e-5, rtol=1e-4)
    assert torch.allclose(got_prev, want_prev, atol=1e-5, rtol=1e-4)


def test_segment_calls_invalidate_the_reported_state(L):
    """The segment calls work in the forward's workspace, so afterwards
    gecko_awm_state reports no state until the next forward."""
    w = Workload("cp_state_invalidated", 84, "f32", 1, 2, 256, 64, 64)
    x = make_inputs(w, device="cuda")
    L.sca_awm_forward(*(x[n] for n in NAMES), w.c)
    L.awm_state(w.B, w.H, w.d)
    L.awm_segment_logsum(x["km"], w.c)
    with pytest.raises(L.GeckoError) as e:
        L.awm_state(w.B, w.H, w.d)
    assert e.value.code == 6
    L.sca_awm_forward(*(x[n] for n in NAMES), w.c)
    M, _ = L.awm_state(w.B, w.H, w.d)
    torch.cuda.synchronize()
    want = F.forward(*(x[n].double().cpu().numpy() for n in NAMES), w.c)
    assert float(np.abs(M.double().cpu().numpy() - want[2]).max()) <= 1e-4
