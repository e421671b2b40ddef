"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.  Tolerances: fp32 max-abs <= 1e-4; bf16 max-abs <= 2e-2
and rel-L2 <= 5e-3 (fp32 accumulation); chunk indexing and masks bit-exact."""
import os

import numpy as np
import pytest
import torch

from long_context_sequence_sca_b200.inputs import WORKLOADS, Workload, make_inputs
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


def _np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


def _check(got, want, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want).max()
    tol = TOL[dtype]
    assert err <= tol["max_abs"], f"{what}: max-abs {err:.3e}"
    if "rel_l2" in tol:
        rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
        assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e}"


def _run(L, x, c):
    o_sca, o_mem = L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], c)
    B, H, T, d = x["q"].shape
    M, lz = L.awm_state(B, H, d)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return o_sca, o_mem, M, lz


def _full_parity(L, w: Workload, kernels=None, monkeypatch=None):
    if kernels and monkeypatch:
        monkeypatch.setenv("GECKO_KERNELS", kernels)
    x = make_inputs(w, device="cuda")
    o_sca, o_mem, M, lz = _run(L, x, w.c)
    r_sca, r_mem, r_M, r_lz = G.forward(*(_np(x[n]) for n in ("q", "k", "v", "qm", "km")), w.c)
    _check(_np(o_sca), r_sca, w.dtype, "out_sca")
    _check(_np(o_mem), r_mem, w.dtype, "out_mem")
    _check(_np(M), r_M, w.dtype, "M state")
    _check(_np(lz), r_lz, w.dtype, "log z")


SMALL = {
    "fp32_small": WORKLOADS["fp32_small"],
    "bf16_many_chunks": WORKLOADS["bf16_many_chunks"],
    # several query tiles, three chunks, d = 128
    "bf16_d128_c512": Workload("bf16_d128_c512", 11, "bf16", 1, 2, 1536, 128, 512),
    # odd number of 128-row tiles: the last work unit holds one query tile
    "bf16_ragged_c128": Workload("bf16_ragged_c128", 12, "bf16", 2, 1, 640, 128, 128),
    # c % 256 != 0: a work unit straddles a chunk boundary
    "bf16_c384": Workload("bf16_c384", 13, "bf16", 1, 2, 1152, 128, 384),
    "bf16_d64_c128": Workload("bf16_d64_c128", 14, "bf16", 1, 3, 1024, 64, 128),
    # a single chunk (T = c): no previous chunk, no memory readout
    "bf16_one_chunk": Workload("bf16_one_chunk", 15, "bf16", 1, 2, 256, 128, 256),
    # wide key offsets (exp-sum dynamic range)
    "bf16_wide_keys": Workload("bf16_wide_keys", 16, "bf16", 1, 2, 2048, 128, 256, key_offset_std=1.0),
    # c = 64 (SIMT kernels), bf16
    "bf16_c64": Workload("bf16_c64", 17, "bf16", 1, 2, 512, 64, 64),
    "fp32_d128": Workload("fp32_d128", 18, "f32", 1, 2, 768, 128, 128),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_parity_small(L, name):
    _full_parity(L, SMALL[name])


@pytest.mark.parametrize("name", ["bf16_d128_c512", "bf16_ragged_c128", "bf16_d64_c128"])
def test_parity_simt_kernels(L, name, monkeypatch):
    _full_parity(L, SMALL[name], kernels="simt", monkeypatch=monkeypatch)


# ---------------------------------------------------------- mask probes --

def _probe_inputs(B, H, T, d, c, dtype, earliest: bool):
    """Scores -/+16*u make the earliest / latest visible key win by e^16;
    V encodes the key index in binary, so the output decodes the winner."""
    nb = max(1, int(np.ceil(np.log2(T))))
    assert nb <= d
    u = torch.arange(T)
    bits = ((u[:, None] >> torch.arange(nb)[None, :]) & 1).float()
    k = torch.zeros(T, d)
    k[:, :nb] = bits
    q = torch.zeros(T, d)
    sign = -1.0 if earliest else 1.0
    q[:, :nb] = sign * 16.0 * (2.0 ** torch.arange(nb).float())[None, :]
    v = torch.zeros(T, d)
    v[:, :nb] = bits
    rep = lambda a: a[None, None].expand(B, H, T, d).contiguous().to(dtype).cuda()
    z = torch.zeros(B, H, T, d, dtype=dtype, device="cuda")
    return rep(q), rep(k), rep(v), z, z.clone(), nb


def _decode(o, nb):
    bits = (o[..., :nb].float().cpu() > 0.5).long()
    return (bits << torch.arange(nb)).sum(-1)


@pytest.mark.parametrize("T,c,d,dtype,kernels", [
    (2048, 256, 128, torch.bfloat16, None),
    (1536, 512, 64, torch.bfloat16, None),
    (1152, 384, 128, torch.bfloat16, None),
    (1024, 128, 128, torch.bfloat16, "simt"),
    (512, 64, 64, torch.float32, None),
])
def test_mask_probe_bit_exact(L, T, c, d, dtype, kernels, monkeypatch):
    if kernels:
        monkeypatch.setenv("GECKO_KERNELS", kernels)
    t = torch.arange(T)
    want_lo = torch.clamp((t // c - 1) * c, min=0)
    for earliest, want in ((True, want_lo), (False, t)):
        q, k, v, qm, km, nb = _probe_inputs(1, 2, T, d, c, dtype, earliest)
        o_sca, _ = L.sca_awm_forward(q, k, v, qm, km, c)
        torch.cuda.synchronize()
        got = _decode(o_sca, nb)
        for h in range(2):
            assert torch.equal(got[0, h], want), (earliest, (got[0, h] != want).nonzero()[:5])


# ------------------------------------------------------- state and errors --

def test_state_shape_mismatch_and_release(L):
    w = SMALL["bf16_one_chunk"]
    x = make_inputs(w, device="cuda")
    L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    with pytest.raises(L.GeckoError) as e:
        L.awm_state(w.B, w.H + 1, w.d)
    assert e.value.code == 1
    L.release()
    with pytest.raises(L.GeckoError) as e:
        L.awm_state(w.B, w.H, w.d)
    assert e.value.code == 6


def test_binding_rejects_mismatched_buffers(L):
    """The binding checks caller-given buffers before the C call: an output
    one row short, an output of another dtype, a state of the wrong size."""
    w = SMALL["bf16_one_chunk"]
    x = make_inputs(w, device="cuda")
    xs = [x[n] for n in ("q", "k", "v", "qm", "km")]
    short = torch.empty(w.B, w.H, w.T - 1, w.d, dtype=x["q"].dtype, device="cuda")
    with pytest.raises(ValueError):
        L.sca_awm_forward(*xs, w.c, out_sca=short)
    with pytest.raises(ValueError):
        L.sca_awm_forward(*xs, w.c, out_mem=torch.empty_like(x["q"], dtype=torch.float32))
    bad_state = torch.zeros(w.B, w.H, 2 * w.d * w.d, dtype=torch.float32, device="cuda")
    kv = [torch.cat([x[n][:, :, :w.c], x[n]], dim=2).contiguous() for n in ("k", "v")]
    with pytest.raises(ValueError):
        L.sca_awm_forward_segment(x["q"], kv[0], kv[1], x["qm"], x["km"], w.c, state_in=bad_state)
    with pytest.raises(ValueError):
        L.awm_segment_maps(x["km"], x["v"], torch.zeros(w.B, w.H, w.d, dtype=torch.float64, device="cuda"), w.c)


def test_injected_allocation_failure(L, monkeypatch):
    L.release()
    w = SMALL["bf16_one_chunk"]
    x = make_inputs(w, device="cuda")
    monkeypatch.setenv("GECKO_FAIL_ALLOC", "1")
    with pytest.raises(L.GeckoError) as e:
        L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    assert e.value.code == 4
    monkeypatch.delenv("GECKO_FAIL_ALLOC")
    L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    torch.cuda.synchronize()
    assert L.device_status() == 0


def test_repeat_calls_are_deterministic(L):
    w = SMALL["bf16_d128_c512"]
    x = make_inputs(w, device="cuda")
    a = [t.clone() for t in L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)]
    b = L.sca_awm_forward(x["q"], x["k"], x["v"], x["qm"], x["km"], w.c)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kernels,parts,d", [(None, None, 128), (None, "1", 128), ("simt", None, 128), (None, "1", 64)])
def test_awm_keys_growing_within_a_chunk(L, kernels, parts, d, monkeypatch):
    """K_m features whose values climb through each chunk (by up to 30 over
    the chunk, and one late spike of +40) and others that fall: the
    chunk-local exponentials of a feature cannot share one reference taken
    early in the chunk, so a kernel that tracks the per-feature maximum as
    it streams the chunk must raise it and rescale what it has accumulated.
    The chunk's log-sum-exp, the state and the readout still match the fp64
    oracle (step 4 of the method: Phi = exp(Km - log z), any real Km).
    parts="1" keeps one CTA per chunk, the form whose chunk kernel computes
    the chunk statistics itself (from the first tile's reference, every
    chunk here outgrowing it, so each is redone by the pass that raises
    its reference); by default this small problem shares each chunk among
    several CTAs after a separate statistics pass."""
    if kernels:
        monkeypatch.setenv("GECKO_KERNELS", kernels)
    if parts:
        monkeypatch.setenv("GECKO_CHUNK_PARTS", parts)
    w = Workload(f"bf16_growing_keys_d{d}", 19, "bf16", 1, 2, 1536, d, 512)
    x = make_inputs(w, device="cuda")
    c = w.c
    t = (torch.arange(w.T, device="cuda") % c).float() / c
    f = torch.arange(d, device="cuda")
    slope = torch.where(f % 4 == 0, 30.0 * (f.float() / d), torch.where(f % 4 == 1, -12.0, 0.0))
    km = x["km"].float() + t[:, None] * slope[None, :]
    spike = (torch.arange(w.T, device="cuda") % c) == c - 70
    km[..., spike, 2::8] += 40.0
    x["km"] = km.to(torch.bfloat16)
    o_sca, o_mem, M, lz = _run(L, x, w.c)
    r_sca, r_mem, r_M, r_lz = G.forward(*(_np(x[n]) for n in ("q", "k", "v", "qm", "km")), w.c)
    _check(_np(o_mem), r_mem, w.dtype, "out_mem")
    _check(_np(M), r_M, w.dtype, "M state")
    _check(_np(lz), r_lz, w.dtype, "log z")
    _check(_np(o_sca), r_sca, w.dtype, "out_sca")


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("growth", [15.0, 60.0])
def test_awm_keys_outgrowing_the_first_tile(L, d, growth, monkeypatch):
    """One CTA per chunk, the chunk statistics computed in the chunk kernel
    against a reference taken from each chunk's first tile.  A third of the
    K_m features climb by `growth` (natural-log units) through the second
    chunk only.  A climb of 15 keeps the exponentials within the 2^32 the
    first-tile reference allows, so no chunk is redone; a climb of 60 goes
    past it, so that chunk alone is redone with a running reference while
    the other chunks keep their first pass.  Either way the state, log z
    and both outputs match the fp64 oracle."""
    monkeypatch.setenv("GECKO_CHUNK_PARTS", "1")
    w = Workload(f"bf16_outgrow_d{d}", 29, "bf16", 1, 2, 2048, d, 512)
    x = make_inputs(w, device="cuda")
    c = w.c
    pos = torch.arange(w.T, device="cuda")
    ramp = ((pos // c) == 1).float() * (pos % c).float() / c * growth
    km = x["km"].float()
    km[..., 1::3] += ramp[:, None]
    x["km"] = km.to(torch.bfloat16)
    o_sca, o_mem, M, lz = _run(L, x, w.c)
    r_sca, r_mem, r_M, r_lz = G.forward(*(_np(x[n]) for n in ("q", "k", "v", "qm", "km")), w.c)
    _check(_np(o_mem), r_mem, w.dtype, "out_mem")
    _check(_np(M), r_M, w.dtype, "M state")
    _check(_np(lz), r_lz, w.dtype, "log z")
    _check(_np(o_sca), r_sca, w.dtype, "out_sca")


@pytest.mark.parametrize("name,parts", [("bf16_d128_c512", "1"), ("bf16_d128_c512", "3"), ("bf16_d128_c512", "8"),
                                        ("bf16_d64_c128", "2"), ("bf16_c384", "1"), ("bf16_c384", "6")])
def test_parity_chunk_parts(L, name, parts, monkeypatch):
    """The chunk products with k CTAs per chunk (each adding its share of
    the tiles into the products, ragged shares included) and with one CTA
    per chunk (at d = 128 with the statistics computed in the chunk kernel)
    against the oracle."""
    monkeypatch.setenv("GECKO_CHUNK_PARTS", parts)
    _full_parity(L, SMALL[name])
