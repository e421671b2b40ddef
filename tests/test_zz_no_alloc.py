"""The no-allocation entry point against the allocating one and the oracle.

gecko_sca_awm_forward_noalloc serves callers that must not allocate device
memory (for example a plugin whose host application's memory pool owns all
of the GPU's memory, or a latency-critical loop that cannot pay for
cudaMalloc's device-wide synchronisation).  It runs the same kernels on a
fixed scratch array inside the library, so on consecutive calls that reuse
the scratch its outputs must match the allocating entry point's and the fp64
oracle's within the parity tolerances used elsewhere.  It must also leave
the library's growable workspace and the exported state alone: it creates
no state for gecko_awm_state, does not change the state of an earlier
allocating forward, and takes no device memory.  This file is collected
last.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import Workload, make_inputs
from oracle import gecko_oracle as G

pytestmark = pytest.mark.gpu

TOL = {"f32": dict(max_abs=1e-4), "bf16": dict(max_abs=2e-2, rel_l2=5e-3)}
NAMES = ("q", "k", "v", "qm", "km")


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib
    build.build()
    lib.load()
    return lib


def _close(a, b, dtype, what=""):
    a = a.double().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a, np.float64)
    b = b.double().cpu().numpy() if isinstance(b, torch.Tensor) else np.asarray(b, np.float64)
    assert np.all(np.isfinite(a)), what
    err = np.abs(a - b).max()
    assert err <= TOL[dtype]["max_abs"], f"{what}: max-abs {err:.3e}"
    if "rel_l2" in TOL[dtype]:
        rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
        assert rel <= TOL[dtype]["rel_l2"], f"{what}: rel-L2 {rel:.3e}"


def _noalloc(L, x, w):
    o_sca = torch.full_like(x["q"], float("nan"))
    o_mem = torch.full_like(x["q"], float("nan"))
    dt = L.GECKO_F32 if w.dtype == "f32" else L.GECKO_BF16
    rc = L.gecko_sca_awm_forward_noalloc(*(x[n].data_ptr() for n in NAMES), o_sca.data_ptr(), o_mem.data_ptr(),
                                         w.B, w.H, w.T, w.c, w.d, dt, torch.cuda.current_stream().cuda_stream)
    assert rc == 0, L.gecko_last_error()
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return o_sca, o_mem


def _state_rc(L, w):
    M = torch.empty(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    lz = torch.empty(w.B, w.H, w.d, dtype=torch.float32, device="cuda")
    rc = L.gecko_awm_state(M.data_ptr(), lz.data_ptr(), w.B, w.H, w.d, torch.cuda.current_stream().cuda_stream)
    return rc, M, lz


WORKLOADS = [
    Workload("noalloc_bf16", 31, "bf16", 1, 4, 4096, 128, 512),
    Workload("noalloc_f32", 32, "f32", 1, 2, 512, 64, 64),
]


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_noalloc_matches_allocating_entry_and_oracle_on_two_calls(L, w):
    x = make_inputs(w, device="cuda")
    ref_sca, ref_mem = L.sca_awm_forward(*(x[n] for n in NAMES), w.c)
    torch.cuda.synchronize()
    rc, M0, lz0 = _state_rc(L, w)
    assert rc == 0
    o_sca_o, o_mem_o, _, _ = G.forward(*(x[n].double().cpu().numpy() for n in NAMES), w.c)
    for _ in range(2):
        o_sca, o_mem = _noalloc(L, x, w)
        _close(o_sca, ref_sca, w.dtype, "out_sca vs allocating entry")
        _close(o_mem, ref_mem, w.dtype, "out_mem vs allocating entry")
        _close(o_sca, o_sca_o, w.dtype, "out_sca vs oracle")
        _close(o_mem, o_mem_o, w.dtype, "out_mem vs oracle")
    # the allocating forward's exported state is untouched
    rc, M1, lz1 = _state_rc(L, w)
    assert rc == 0
    assert torch.equal(M0, M1) and torch.equal(lz0, lz1)


def test_noalloc_creates_no_state_and_takes_no_device_memory(L):
    w = WORKLOADS[0]
    x = make_inputs(w, device="cuda")
    _noalloc(L, x, w)            # the scratch address is resolved on a first call
    L.gecko_release()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    o_sca, o_mem = _noalloc(L, x, w)
    free1, _ = torch.cuda.mem_get_info()
    # the allocating forward would need this much working memory
    BH, S, d = w.B * w.H, w.T // w.c, w.d
    ws = 4 * (3 * S + 1) * BH * d * d + 2 * (2 * S + 1) * BH * d * d
    assert free0 - free1 < ws, (free0, free1, ws)
    rc, _, _ = _state_rc(L, w)
    assert rc == 6, "gecko_awm_state must report GECKO_ERR_NO_STATE after a release"
    ref_sca, ref_mem, _, _ = G.forward(*(x[n].double().cpu().numpy() for n in NAMES), w.c)
    _close(o_sca, ref_sca, w.dtype, "out_sca vs oracle")
    _close(o_mem, ref_mem, w.dtype, "out_mem vs oracle")


def test_noalloc_headline_shape_fits_and_equals_the_allocating_entry(L):
    """B=1, H=32, T=32768, c=4096, d=128 (about 79 MB of working memory) fits
    the scratch; the same kernels give the allocating forward's outputs bit
    for bit."""
    w = Workload("noalloc_headline", 34, "bf16", 1, 32, 32768, 128, 4096)
    x = make_inputs(w, device="cuda")
    ref_sca, ref_mem = L.sca_awm_forward(*(x[n] for n in NAMES), w.c)
    o_sca, o_mem = _noalloc(L, x, w)
    assert torch.equal(o_sca, ref_sca) and torch.equal(o_mem, ref_mem)


def test_noalloc_rejects_problems_above_its_scratch(L):
    # 400 chunks of 128 tokens at d = 128 need about 106 MB of working memory
    w = Workload("noalloc_big", 33, "bf16", 1, 1, 128 * 400, 128, 128)
    x = {n: torch.zeros(w.B, w.H, w.T, w.d, dtype=torch.bfloat16, device="cuda")
         for n in ("q", "k", "v", "qm", "km", "o1", "o2")}
    rc = L.gecko_sca_awm_forward_noalloc(*(x[n].data_ptr() for n in ("q", "k", "v", "qm", "km", "o1", "o2")),
                                         w.B, w.H, w.T, w.c, w.d, L.GECKO_BF16,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 8
    assert "no-allocation" in L.gecko_last_error()
