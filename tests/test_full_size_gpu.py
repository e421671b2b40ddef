"""Parity at full workload sizes, in the launch configuration bench.py times.

Every output buffer is filled with NaN before the call, so a row that no work
unit writes (a unit dropped by the dynamic claim counter, or a ring slot
overwritten before it was read) fails the finiteness check.  At the
7B-layer-shaped headline workload (B=1, H=32, T=32768, d=128, c=4096) the
fp64 oracle then recomputes:
  * every SCA row of four heads: the first, one in the middle, and the two
    last ones (whose chunk-1 units are the last ones claimed), so all 128
    work units of each of those heads are compared element by element;
  * out_mem, M'_{S+1} and log z^S of all 32 heads;
and a bit-exact mask probe decodes the first and the last visible key of
every query of every head (Gecko digest, method step details, step 3: the
window is the current and the previous chunk).  The chunk-size sweep and the
4M-token run compare sampled SCA rows and whole AWM heads.  Tolerances as
elsewhere: bf16 max-abs <= 2e-2 and rel-L2 <= 5e-3; the probe bit-exact.
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


def _forward_nan_prefilled(L, x, c):
    """The forward into NaN-filled output buffers; every element must be
    written (finite) afterwards."""
    o_sca = torch.full_like(x["q"], float("nan"))
    o_mem = torch.full_like(x["q"], float("nan"))
    L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], c, out_sca=o_sca, out_mem=o_mem)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    assert bool(torch.isfinite(o_sca).all()), "out_sca: a row was never written"
    assert bool(torch.isfinite(o_mem).all()), "out_mem: a row was never written"
    return o_sca, o_mem


def _check_awm_heads(L, x, w, o_mem, heads):
    M, lz = L.awm_state(w.B, w.H, w.d)
    torch.cuda.synchronize()
    for (b, h) in heads:
        om, st, lzr = G.awm_head(_h(x["qm"], b, h), _h(x["km"], b, h), _h(x["v"], b, h), w.c, keep_states=False)
        _close(o_mem[b, h].double().cpu().numpy(), om, f"out_mem b{b} h{h}")
        _close(M[b, h].double().cpu().numpy(), st[-1], f"M b{b} h{h}")
        _close(lz[b, h].double().cpu().numpy(), lzr[-1], f"log z b{b} h{h}")


def test_headline_workload_every_row_of_four_heads(L):
    w = WORKLOADS["bf16_h32_c4096"]
    x = make_inputs(w, device="cuda")
    o_sca, o_mem = _forward_nan_prefilled(L, x, w.c)
    for h in (0, 13, w.H - 2, w.H - 1):
        want = G.sca_head(_h(x["q"], 0, h), _h(x["k"], 0, h), _h(x["v"], 0, h), w.c)
        _close(o_sca[0, h].double().cpu().numpy(), want, f"out_sca, every row of head {h}")
    _check_awm_heads(L, x, w, o_mem, [(0, h) for h in range(w.H)])


# ---------------------------------------------------- mask probe, full size --

def _probe_inputs(B, H, T, d, earliest: bool):
    """Q . K = -/+16 u makes the earliest / latest visible key u win by e^16;
    V holds u in binary, so each output row decodes the winning key.  All
    products are exact in bf16 inputs and fp32 accumulation (|16 u| < 2^24)."""
    nb = max(1, int(np.ceil(np.log2(T))))
    assert nb <= d
    u = torch.arange(T)
    bits = ((u[:, None] >> torch.arange(nb)[None, :]) & 1).float()
    k = torch.zeros(T, d)
    k[:, :nb] = bits
    q = torch.zeros(T, d)
    q[:, :nb] = (-16.0 if earliest else 16.0) * (2.0 ** torch.arange(nb).float())[None, :]
    v = torch.zeros(T, d)
    v[:, :nb] = bits
    rep = lambda a: a.to(torch.bfloat16).cuda()[None, None].expand(B, H, T, d).contiguous()
    z = torch.zeros(B, H, T, d, dtype=torch.bfloat16, device="cuda")
    return rep(q), rep(k), rep(v), z, z.clone(), nb


def test_mask_probe_bit_exact_at_headline_shape(L):
    """Window start max(0, (s-2)c) and end t of every query of all 32 heads at
    B=1, H=32, T=32768, c=4096, d=128, decoded exactly from the output."""
    B, H, T, d, c = 1, 32, 32768, 128, 4096
    t = torch.arange(T)
    want_lo = torch.clamp((t // c - 1) * c, min=0)
    for earliest, want in ((True, want_lo), (False, t)):
        q, k, v, qm, km, nb = _probe_inputs(B, H, T, d, earliest)
        o_sca = torch.full_like(q, float("nan"))
        L.sca_awm_forward(q, k, v, qm, km, c, out_sca=o_sca)
        torch.cuda.synchronize()
        assert L.device_status() == 0
        got = ((o_sca[0, :, :, :nb].float() > 0.5).long() << torch.arange(nb, device="cuda")).sum(-1).cpu()
        bad = (got != want[None, :]).nonzero()
        assert bad.numel() == 0, (earliest, bad[:5].tolist())
        del q, k, v, qm, km, o_sca


# ------------------------------------------------------ chunk-size sweep --

@pytest.mark.parametrize("c", [512, 1024, 2048, 4096])
def test_chunk_size_sweep_sampled(L, c):
    w = WORKLOADS[f"bf16_sweep_c{c}"]
    x = make_inputs(w, device="cuda")
    o_sca, o_mem = _forward_nan_prefilled(L, x, w.c)
    rng = np.random.default_rng(c)
    heads = [(0, 0), (0, 21), (0, w.H - 1)]
    for (b, h) in heads:
        rows = _sample_rows(w.T, w.c, rng)
        want = G.sca_rows(_h(x["q"], b, h), _h(x["k"], b, h), _h(x["v"], b, h), w.c, rows)
        _close(o_sca[b, h, rows].double().cpu().numpy(), want, f"out_sca b{b} h{h}")
    _check_awm_heads(L, x, w, o_mem, heads)


# ------------------------------------------------------------ 4M tokens --

def test_four_million_tokens_stable_and_sampled(L):
    """4,194,304 tokens x 8 heads into NaN-filled outputs: every output
    written and finite; the AWM of one head is recomputed in fp64 through all
    1024 chunks and 8 random chunks are compared in full, plus sampled SCA
    rows of those chunks."""
    w = WORKLOADS["bf16_4m_tokens"]
    x = make_inputs(w, device="cuda")
    o_sca, o_mem = _forward_nan_prefilled(L, x, w.c)
    M, lz = L.awm_state(w.B, w.H, w.d)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(M).all()) and bool(torch.isfinite(lz).all())
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
