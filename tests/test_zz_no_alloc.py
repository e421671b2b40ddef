"""The no-allocation entry point against the allocating one.

gecko_sca_awm_forward_noalloc serves callers that must not allocate device
memory (for example a plugin whose host application's memory pool owns all
of the GPU's memory, or a latency-critical loop that cannot pay for
cudaMalloc's device-wide synchronisation).  It runs the same kernels on a
fixed scratch array inside the library, so its outputs must match the
allocating entry point's within the parity tolerances used elsewhere, on
consecutive calls that reuse the scratch.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import Workload, make_inputs

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


def _close(a, b, dtype):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.all(np.isfinite(a))
    assert np.abs(a - b).max() <= TOL[dtype]["max_abs"]
    if "rel_l2" in TOL[dtype]:
        assert np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30) <= TOL[dtype]["rel_l2"]


@pytest.mark.parametrize("w", [
    Workload("noalloc_bf16", 31, "bf16", 1, 4, 4096, 128, 512),
    Workload("noalloc_f32", 32, "f32", 1, 2, 512, 64, 64),
], ids=lambda w: w.name)
def test_noalloc_matches_allocating_entry_on_two_calls(L, w):
    x = make_inputs(w, device="cuda")
    ref_sca, ref_mem = L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    dt = L.GECKO_F32 if w.dtype == "f32" else L.GECKO_BF16
    for _ in range(2):
        o_sca = torch.full_like(x["q"], float("nan"))
        o_mem = torch.full_like(x["q"], float("nan"))
        rc = L.gecko_sca_awm_forward_noalloc(
            *(x[n].data_ptr() for n in ("q", "k", "v", "qm", "km")), o_sca.data_ptr(), o_mem.data_ptr(),
            w.B, w.H, w.T, w.c, w.d, dt, stream)
        assert rc == 0, L.gecko_last_error()
        torch.cuda.synchronize()
        assert L.device_status() == 0
        _close(o_sca, ref_sca, w.dtype)
        _close(o_mem, ref_mem, w.dtype)


def test_noalloc_rejects_problems_above_its_scratch(L):
    # 400 chunks of 128 tokens at d = 128 need about 77 MB of working memory
    w = Workload("noalloc_big", 33, "bf16", 1, 1, 128 * 400, 128, 128)
    x = {n: torch.zeros(w.B, w.H, w.T, w.d, dtype=torch.bfloat16, device="cuda")
         for n in ("q", "k", "v", "qm", "km", "o1", "o2")}
    rc = L.gecko_sca_awm_forward_noalloc(*(x[n].data_ptr() for n in ("q", "k", "v", "qm", "km", "o1", "o2")),
                                         w.B, w.H, w.T, w.c, w.d, L.GECKO_BF16,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 8
    assert "no-allocation" in L.gecko_last_error()
