"""Parity at full workload sizes, in the launch configuration bench.py times.

The CUDA path runs the whole workload; the fp64 oracle recomputes sampled
outputs one by one: SCA rows through their own window (gecko_oracle.sca_rows),
and the AWM of sampled heads (whole head, or streamed chunk by chunk with the
fp64 state propagated through every chunk for the 4M-token case).  Every
output of the run must also be finite.  Tolerances as elsewhere: bf16 max-abs
<= 2e-2 and rel-L2 <= 5e-3.
"""
import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import WORKLOADS, make_inputs
from oracle import gecko_oracle as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sequence_sca_b200 import build, lib
    build.build()
    lib.load()
    return lib


def _close(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= 2e-2 and rel <= 5e-3, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"


def _h(x, b, h):
    return x[b, h].double().cpu().numpy()


def _sample_rows(T, c, rng, per_chunk=6):
    rows = []
    for s in range(T // c):
        base = s * c
        fixed = [0, 1, c // 2, c - 1]
        rows += [base + r for r in fixed]
        rows += list(base + rng.integers(0, c, per_chunk - len(fixed)))
    return sorted(set(int(r) for r in rows))


def _run_and_check(L, w, heads, seed=0):
    x = make_inputs(w, device="cuda")
    o_sca, o_mem = L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    M, lz = L.awm_state(w.B, w.H, w.d)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    assert bool(torch.isfinite(o_sca).all()) and bool(torch.isfinite(o_mem).all())
    rng = np.random.default_rng(seed)
    for (b, h) in heads:
        q, k, v, qm, km = (_h(x[n], b, h) for n in ("q", "k", "v", "qm", "km"))
        rows = _sample_rows(w.T, w.c, rng)
        _close(o_sca[b, h, rows].double().cpu().numpy(), G.sca_rows(q, k, v, w.c, rows), f"out_sca b{b} h{h}")
        om, st, lzr = G.awm_head(qm, km, v, w.c, keep_states=False)
        _close(o_mem[b, h].double().cpu().numpy(), om, f"out_mem b{b} h{h}")
        _close(M[b, h].double().cpu().numpy(), st[-1], f"M b{b} h{h}")
        _close(lz[b, h].double().cpu().numpy(), lzr[-1], f"log z b{b} h{h}")


def test_headline_workload_sampled(L):
    w = WORKLOADS["bf16_h32_c4096"]
    _run_and_check(L, w, heads=[(0, 0), (0, 13), (0, 31)])


@pytest.mark.parametrize("c", [512, 1024, 2048, 4096])
def test_chunk_size_sweep_sampled(L, c):
    w = WORKLOADS[f"bf16_sweep_c{c}"]
    _run_and_check(L, w, heads=[(0, 0), (0, 21)], seed=c)


def test_four_million_tokens_stable_and_sampled(L):
    """4,194,304 tokens x 8 heads: every output finite; the AWM of one head is
    recomputed in fp64 through all 1024 chunks and 8 random chunks are
    compared in full, plus sampled SCA rows of those chunks."""
    w = WORKLOADS["bf16_4m_tokens"]
    x = make_inputs(w, device="cuda")
    o_sca, o_mem = L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    M, lz = L.awm_state(w.B, w.H, w.d)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    for t in (o_sca, o_mem, M, lz):
        assert bool(torch.isfinite(t).all())
    S, c = w.S, w.c
    rng = np.random.default_rng(5)
    want = sorted(set(int(s) for s in rng.choice(np.arange(3, S + 1), 8, replace=False)))
    h = 3
    chunk = lambda name: (x[name][0, h, (s - 1) * c: s * c].double().cpu().numpy() for s in range(1, S + 1))
    got, M_ref, lz_ref = G.awm_propagate(chunk("km"), chunk("v"), chunk("qm"), c, want_chunks=want)
    for s in want:
        _close(o_mem[0, h, (s - 1) * c: s * c].double().cpu().numpy(), got[s], f"out_mem chunk {s}")
        rows = [(s - 1) * c + int(r) for r in sorted(rng.choice(c, 8, replace=False))]
        lo = (s - 2) * c
        kk = x["k"][0, h, lo: s * c].double().cpu().numpy()
        vv = x["v"][0, h, lo: s * c].double().cpu().numpy()
        qq = x["q"][0, h, lo: s * c].double().cpu().numpy()
        ref = G.sca_rows(qq, kk, vv, c, [r - lo for r in rows])
        _close(o_sca[0, h, rows].double().cpu().numpy(), ref, f"out_sca chunk {s}")
    _close(M[0, h].double().cpu().numpy(), M_ref, "M after 1024 chunks")
    _close(lz[0, h].double().cpu().numpy(), lz_ref, "log z after 1024 chunks")
