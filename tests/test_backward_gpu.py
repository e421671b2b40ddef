"""GPU parity of the backward (gecko_sca_awm_forward_train +
gecko_sca_awm_backward) against the fp64 gradient oracle on the same seeded
inputs and output gradients.

Tolerances: the gradients are sums of many terms of either sign, so the
absolute bars of the forward are scaled by the size of the reference
gradient: fp32 max-abs <= 1e-4 * max(1, max|ref|); bf16 max-abs <=
2e-2 * max(1, max|ref|) and rel-L2 <= 1e-2.  The bf16 rel-L2 bar is twice
the forward's: P and dS enter the MMAs as bf16, and the dq of a row is a
strongly cancelling sum (its dS terms sum to zero).  The backward takes the
forward's output together with its rounding residual; with the bf16 output
alone, the row term delta = rowsum(dO * O) would carry O's rounding, which
by itself moves the oracle's own dq by several 1e-3 (pinned on the CPU in
test_backward_tolerance_cpu.py) and by several 1e-2 at 8K-key windows;
test_backward_without_residual keeps that path covered.  The SCA row log-sum-exp is compared
against the oracle's as a forward quantity (fp32 1e-4, bf16 2e-2)."""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import gecko_backward_oracle as GB

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
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), what
    scale = max(1.0, float(np.abs(want).max()))
    err = float(np.abs(got - want).max())
    bar = (1e-4 if dtype == "f32" else 2e-2) * scale
    assert err <= bar, f"{what}: max-abs {err:.3e} > {bar:.3e}"
    if dtype == "bf16":
        rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
        assert rel <= 1e-2, f"{what}: rel-L2 {rel:.3e}"


def _douts(x, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(x.shape, generator=g).to(x.dtype).to(x.device) for _ in range(2)]


def _check_backward(L, w: Workload, seed=1234, env=None, monkeypatch=None):
    if env and monkeypatch:
        for k, v in env.items():
            monkeypatch.setenv(k, v)
    x = make_inputs(w, device="cuda")
    dos, dom = _douts(x["q"], seed)
    out_sca, out_mem, lse, lo = L.sca_awm_forward_train(*(x[n] for n in NAMES), w.c)
    grads = L.sca_awm_backward(*(x[n] for n in NAMES), out_sca, lse, dos, dom, w.c, out_sca_lo=lo)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    xs = [x[n].double().cpu().numpy() for n in NAMES]
    ref = GB.backward(*xs, w.c, dos.double().cpu().numpy(), dom.double().cpu().numpy())
    for n, g, r in zip(NAMES, grads, ref):
        _close(g, r, w.dtype, "d" + n)
    ref_lse = np.stack([[GB.sca_lse(xs[0][b, h], xs[1][b, h], w.c) for h in range(w.H)] for b in range(w.B)])
    _close(lse, ref_lse, w.dtype, "lse")
    return out_sca, out_mem


@pytest.mark.parametrize("name", ["fp32_small", "bf16_many_chunks"])
def test_backward_matches_oracle(L, name):
    _check_backward(L, WORKLOADS[name])


@pytest.mark.parametrize("w", [
    Workload("bwd_bf16_d128_c128", 61, "bf16", 1, 2, 1024, 128, 128),
    Workload("bwd_f32_d128_c64", 62, "f32", 1, 1, 384, 128, 64),
    Workload("bwd_bf16_one_chunk", 63, "bf16", 2, 1, 256, 64, 256),
    Workload("bwd_bf16_two_chunks", 64, "bf16", 1, 2, 512, 128, 256),
    # c an odd multiple of 128: chunk boundaries fall between 128-row tiles
    # that are not aligned to 256 rows
    Workload("bwd_bf16_c384", 66, "bf16", 1, 2, 1152, 128, 384),
    Workload("bwd_bf16_c384_d64", 67, "bf16", 2, 1, 1536, 64, 384),
], ids=lambda w: w.name)
def test_backward_shapes(L, w):
    _check_backward(L, w)


def test_backward_simt_kernels_for_bf16(L, monkeypatch):
    """The CUDA-core kernels on a bf16 workload the tensor-core path also
    takes (a second implementation of the same gradients)."""
    _check_backward(L, Workload("bwd_bf16_simt", 65, "bf16", 1, 2, 1024, 128, 128),
                    env={"GECKO_KERNELS": "simt"}, monkeypatch=monkeypatch)


def test_train_forward_outputs_equal_plain_forward(L):
    w = WORKLOADS["bf16_many_chunks"]
    x = make_inputs(w, device="cuda")
    a = L.sca_awm_forward(*(x[n] for n in NAMES), w.c)
    b = L.sca_awm_forward_train(*(x[n] for n in NAMES), w.c)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    # the residual is what the rounding to bf16 dropped: |lo| <= half an ulp of out
    lo, hi = b[3].float(), b[0].float()
    assert torch.all(lo.abs() <= hi.abs() * 2.0 ** -8 + 1e-30)
    assert lo.abs().max() > 0


def test_autograd_function_uses_the_same_kernels(L):
    w = WORKLOADS["fp32_small"]
    x = make_inputs(w, device="cuda")
    ins = [x[n].clone().requires_grad_(True) for n in NAMES]
    o_sca, o_mem = L.ScaAwmFunction.apply(*ins, w.c)
    dos, dom = _douts(x["q"], 7)
    torch.autograd.backward((o_sca, o_mem), (dos, dom))
    out_sca, _, lse, lo = L.sca_awm_forward_train(*(x[n] for n in NAMES), w.c)
    want = L.sca_awm_backward(*(x[n] for n in NAMES), out_sca, lse, dos, dom, w.c, out_sca_lo=lo)
    torch.cuda.synchronize()
    for t, g in zip(ins, want):
        assert torch.equal(t.grad, g)


def test_backward_without_residual(L):
    """out_sca_lo = NULL: delta from the bf16 output alone (still within the
    bar at this window size, see the note at the top)."""
    w = WORKLOADS["bf16_many_chunks"]
    x = make_inputs(w, device="cuda")
    dos, dom = _douts(x["q"], 99)
    out_sca, _, lse, _ = L.sca_awm_forward_train(*(x[n] for n in NAMES), w.c, keep_residual=False)
    grads = L.sca_awm_backward(*(x[n] for n in NAMES), out_sca, lse, dos, dom, w.c)
    torch.cuda.synchronize()
    xs = [x[n].double().cpu().numpy() for n in NAMES]
    ref = GB.backward(*xs, w.c, dos.double().cpu().numpy(), dom.double().cpu().numpy())
    for n, g, r in zip(NAMES, grads, ref):
        _close(g, r, w.dtype, "d" + n)
